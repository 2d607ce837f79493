"""Learned-coordinate scoring on the GPU (sparse_attn_dist_fwd / _bwd)
against the CPU oracle, element by element: s_ij = -scale |a_i - c_j|^2 over
the same neighbour lists ("SpatialLM-Mini ...", section "How tokens choose
whom to listen to").  Structured and CSR graphs (with empty rows), bf16 and
fp32 values, every supported head size, ragged tails; structured graphs
through the kernels that stage a block's rows in shared memory and, when
those do not fit, through the per-row kernels."""
import math

import numpy as np
import pytest
import torch

import synth
from gpu_util import compare, to_oracle

pytestmark = pytest.mark.gpu


def _wl(name, B, H, T, D, dtype, W, exps=(), seed=1, band=0, csr=False):
    return synth.Workload(name=name, B=B, H=H, T=T, D=D, dtype=dtype, W=W, exps=tuple(exps),
                          input_std=1.0, scale=0.5, seed=seed, band_hint=band, csr=csr)


def _csr_with_empty(T, seed):
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(T):
        n = 0 if i % 5 == 2 else int(rng.integers(1, 10))
        rows.append(list(rng.integers(0, i + 1, size=n)))
    rp = np.zeros(T + 1, np.int64)
    rp[1:] = np.cumsum([len(r) for r in rows])
    return rp, np.array([x for r in rows for x in r], np.int32)


CASES = [
    (_wl("dist_d64_bf16", 1, 2, 1000, 64, "bf16", 32, range(0, 10)), None),
    (_wl("dist_d32_fp32", 1, 2, 300, 32, "fp32", 8, range(0, 9)), None),
    (_wl("dist_d128_bf16", 2, 1, 333, 128, "bf16", 16, (4, 6, 8)), None),
    # fewer rows than one staged block, and one block plus a row (fp32: at a
    # handful of rows the bf16 out's rounding in Delta dominates da and dc)
    (_wl("dist_t5_fp32", 1, 2, 5, 64, "fp32", 4, (0, 1, 2)), None),
    (_wl("dist_t33_fp32", 1, 1, 33, 64, "fp32", 8, range(0, 6)), None),
    # a structured graph whose staged rows exceed the staged kernels' shared
    # memory (fp32, D = 128): the per-row kernels
    (_wl("dist_d128_fp32_unstaged", 1, 2, 700, 128, "fp32", 64, range(6, 10)), None),
    (_wl("dist_csr_empty_rows", 1, 2, 400, 64, "bf16", 0, csr=True), _csr_with_empty(400, 3)),
    (_wl("dist_csr_view", 1, 1, 1500, 64, "fp32", 0, csr=True, band=64),
     synth.csr_random_rows(1500, seed=5)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_dist_parity(case, oracle_lib):
    import sparse_graph_causal_b200 as sa
    w, csr = case
    o = oracle_lib
    if csr is None:
        g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
        rp, ci = o.structured(w.T, w.W, w.exps)
    else:
        g = sa.sparse_attn_graph_build_csr(torch.from_numpy(csr[0]).cuda(),
                                           torch.from_numpy(csr[1]).cuda(), band_hint=w.band_hint)
        rp, ci = o.normalize(*csr)
    a, c = synth.make_coords(w, device="cuda")
    x = synth.make_qkv(w, device="cuda")
    v, dout = x["v"], x["dout"]
    out, lse = sa.sparse_attn_dist_fwd(a, c, v, g, w.scale)
    da, dc, dv = sa.sparse_attn_dist_bwd(a, c, v, out, lse, dout, g, w.scale)
    sa.sparse_attn_check_device()
    BH = w.B * w.H
    for bh in range(BH):
        ah = a.view(BH, w.T, 3)[bh].cpu().numpy()
        chh = c.view(BH, w.T, 3)[bh].cpu().numpy()
        vh = to_oracle(v.view(BH, w.T, w.D)[bh], w.dtype)
        doh = to_oracle(dout.view(BH, w.T, w.D)[bh], w.dtype)
        r_out, r_lse = o.dist_fwd(ah, chh, vh, rp, ci, w.scale, dtype=w.dtype, cdtype="fp32")
        r_da, r_dc, r_dv = o.dist_bwd(ah, chh, vh, doh, rp, ci, w.scale, dtype=w.dtype,
                                      cdtype="fp32")
        tag = f"{w.name}[bh={bh}]"
        compare(out.view(BH, w.T, w.D)[bh], r_out, w.dtype, tag + " out")
        compare(lse.view(BH, w.T)[bh], r_lse, w.dtype, tag + " lse")
        # da and dc carry the coordinates' scale (2 scale |a - c| per edge),
        # not unit scale: bounded relative to their range (gpu_util.STRESS)
        compare(da.view(BH, w.T, 3)[bh], r_da, w.dtype, tag + " da", unit_range=1.0)
        compare(dc.view(BH, w.T, 3)[bh], r_dc, w.dtype, tag + " dc", unit_range=1.0)
        compare(dv.view(BH, w.T, w.D)[bh], r_dv, w.dtype, tag + " dv")


def test_dist_autograd_and_determinism():
    """The autograd wrapper returns the library's gradients; two backward
    calls give bitwise equal results."""
    import sparse_graph_causal_b200 as sa
    w = _wl("dist_autograd", 1, 2, 700, 64, "bf16", 32, range(0, 10))
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    a, c = synth.make_coords(w, device="cuda")
    x = synth.make_qkv(w, device="cuda")
    v, dout = x["v"], x["dout"]
    out, lse = sa.sparse_attn_dist_fwd(a, c, v, g, w.scale)
    r1 = sa.sparse_attn_dist_bwd(a, c, v, out, lse, dout, g, w.scale)
    r2 = sa.sparse_attn_dist_bwd(a, c, v, out, lse, dout, g, w.scale)
    for p, q in zip(r1, r2):
        assert torch.equal(p, q)
    ta, tc, tv = (t.clone().requires_grad_(True) for t in (a, c, v))
    y = sa.dist_attention(ta, tc, tv, g, w.scale)
    assert torch.equal(y, out)
    y.backward(dout)
    assert torch.equal(ta.grad, r1[0]) and torch.equal(tc.grad, r1[1])
    assert torch.equal(tv.grad, r1[2])
