"""sparse_attn_bwd_noalloc, the backward for callers that cannot allocate
device memory when they call it (a host under a fixed device-memory plan, or
code inside an allocator hook).  It is called through the C ABI and must give
the same gradients as sparse_attn_bwd and as the CPU oracle, within the
tolerance of the other parity tests, on two calls in a row (the second call
reuses the library's fixed scratch array left as the first call wrote it).
The cases reach each kernel family that reads that array: the tcgen05 band
kernels on a structured graph (distance links recomputed, no edge cache) and
on a CSR graph, and the CUDA-core gather kernels (fp32 inputs, and bf16
forced onto them).  This file is collected last so that a run stopping at
the first failure has run every other test."""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth
from gpu_util import compare, to_oracle

pytestmark = pytest.mark.gpu


def _call_noalloc(sa, q, k, v, out, lse, dout, g, scale, dq, dk, dv):
    ts = [sa._tensor(x, n) for x, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"),
                                        (dout, "dout"), (dq, "dq"), (dk, "dk"), (dv, "dv"))]
    r = [ctypes.byref(t) for t in ts]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sa._lib.sparse_attn_bwd_noalloc(r[0], r[1], r[2], r[3], lse.data_ptr(), r[4],
                                           g.handle, float(scale), r[5], r[6], r[7], stream)


def _wl(name, B, H, T, D, dtype, W, exps=(), std=1.0, seed=3, band=0, csr=False):
    return synth.Workload(name=name, B=B, H=H, T=T, D=D, dtype=dtype, W=W, exps=tuple(exps),
                          input_std=std, scale=1.0 / math.sqrt(D), seed=seed, band_hint=band,
                          csr=csr)


# (workload, kernel path): 0 = automatic choice, 1 = gather kernels only
CASES = [
    (_wl("band_links", 1, 4, 5000, 64, "bf16", 32, range(0, 13), std=0.125), 0),
    (_wl("band_csr", 1, 2, 1500, 64, "bf16", 0, band=64, csr=True), 0),
    (_wl("gather_fp32", 1, 2, 600, 64, "fp32", 16, range(0, 10)), 0),
    (_wl("gather_bf16", 1, 2, 900, 64, "bf16", 32, range(0, 10)), 1),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_bwd_noalloc_matches_bwd_and_oracle(case, oracle_lib):
    import sparse_graph_causal_b200 as sa
    w, path = case
    o = oracle_lib
    sa.sparse_attn_set_path(path)
    try:
        if w.csr:
            rp_raw, ci_raw = synth.csr_random_rows(w.T, seed=17)
            g = sa.sparse_attn_graph_build_csr(torch.from_numpy(rp_raw).cuda(),
                                               torch.from_numpy(ci_raw).cuda(),
                                               band_hint=w.band_hint)
            rp, ci = o.normalize(rp_raw, ci_raw)
        else:
            g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
            rp, ci = o.structured(w.T, w.W, w.exps)
        x = synth.make_qkv(w, device="cuda")
        out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
        ref = sa.sparse_attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale)
        ref = [t.double().cpu().numpy() for t in ref]
        got_calls = []
        for call in range(2):
            dq, dk, dv = (torch.full_like(x["q"], float("nan")) for _ in range(3))
            st = _call_noalloc(sa, x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale,
                               dq, dk, dv)
            assert st == sa.SA_OK, sa.sparse_attn_status_string(st)
            sa.sparse_attn_check_device()
            for got, r, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
                compare(got, r, w.dtype, f"{w.name} noalloc call {call} {name} vs bwd")
            got_calls.append((dq, dk, dv))
    finally:
        sa.sparse_attn_set_path(sa.SA_PATH_AUTO)
    # the oracle, on every (b, h) slice of the second call's gradients
    BH = w.B * w.H
    dq, dk, dv = got_calls[1]
    for bh in range(BH):
        sl = [to_oracle(x[n].view(BH, w.T, w.D)[bh], w.dtype) for n in ("q", "k", "v", "dout")]
        rdq, rdk, rdv = o.bwd(*sl, rp, ci, w.scale, dtype=w.dtype)
        for got, r, name in ((dq, rdq, "dq"), (dk, rdk, "dk"), (dv, rdv, "dv")):
            compare(got.view(BH, w.T, w.D)[bh], r, w.dtype, f"{w.name}[bh={bh}] noalloc {name}")


def test_bwd_noalloc_rejects_sizes_beyond_its_array():
    import sparse_graph_causal_b200 as sa
    T = sa.SA_NOALLOC_MAX_ROWS + 128
    g = sa.sparse_attn_graph_build_structured(T, 8, [])
    t = [torch.zeros(1, 1, T, 32, dtype=torch.bfloat16, device="cuda") for _ in range(7)]
    lse = torch.zeros(1, 1, T, dtype=torch.float32, device="cuda")
    before = sa.sparse_attn_launch_count()
    st = _call_noalloc(sa, t[0], t[1], t[2], t[3], lse, t[4], g, 1.0, t[5], t[6], t[0].clone())
    assert st == sa.SA_ERR_UNSUPPORTED
    assert sa.sparse_attn_launch_count() == before


def test_bwd_noalloc_checks_arguments_before_size():
    """A malformed argument is an argument error even when the size is also
    beyond the array, and nothing is launched."""
    import sparse_graph_causal_b200 as sa
    T = sa.SA_NOALLOC_MAX_ROWS + 128
    g = sa.sparse_attn_graph_build_structured(T, 8, [])
    t = [torch.zeros(1, 1, T, 32, dtype=torch.bfloat16, device="cuda") for _ in range(7)]
    lse = torch.zeros(1, 1, T, dtype=torch.float32, device="cuda")
    before = sa.sparse_attn_launch_count()
    st = _call_noalloc(sa, t[0], t[1], t[2], t[3], lse, t[4], g, float("nan"), t[5], t[6],
                       t[0].clone())
    assert st == sa.SA_ERR_INVALID_ARG
    assert sa.sparse_attn_launch_count() == before
