"""Grouped-query attention ("MiniGPT (Part 6)", introduction: grouped-query
attention shrinks the key-value cache): k and v carry Hkv heads, Hkv
dividing H, and query head h reads key/value head h / (H / Hkv).  GPU
forward and backward against the CPU oracle: out, lse and dq per query head
from the oracle on that head's key/value head; dk and dv of a key/value head
are the sums of the oracle's per-query-head gradients over its group."""
import math

import numpy as np
import pytest
import torch

import synth
from gpu_util import compare, to_oracle

pytestmark = pytest.mark.gpu


def _draw(shape, dtype, seed, std=1.0):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return (torch.empty(shape, dtype=torch.float32, device="cuda").normal_(
        0.0, std, generator=g)).to(dtype)


CASES = [
    # name, B, H, Hkv, T, D, dtype, W, exps, csr
    ("gqa2_d64_links", 2, 4, 2, 700, 64, torch.bfloat16, 32, range(0, 10), None),
    ("gqa4_d64_band", 1, 4, 1, 600, 64, torch.bfloat16, 128, (), None),
    ("gqa2_d128_links", 1, 4, 2, 520, 128, torch.bfloat16, 64, (6, 7, 8), None),
    ("gqa2_d32_fp32", 1, 4, 2, 300, 32, torch.float32, 8, range(0, 8), None),
    ("gqa2_csr", 1, 2, 1, 900, 64, torch.bfloat16, 0, (), synth.csr_random_rows(900, seed=31)),
]


@pytest.mark.parametrize("path", [0, 1], ids=["auto", "gather"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_gqa_parity(case, path, oracle_lib):
    import sparse_graph_causal_b200 as sa
    name, B, H, Hkv, T, D, dt, W, exps, csr = case
    o = oracle_lib
    dtype = "bf16" if dt == torch.bfloat16 else "fp32"
    scale = 1.0 / math.sqrt(D)
    sa.sparse_attn_set_path(path)
    try:
        if csr is None:
            g = sa.sparse_attn_graph_build_structured(T, W, list(exps))
            rp, ci = o.structured(T, W, exps)
        else:
            g = sa.sparse_attn_graph_build_csr(torch.from_numpy(csr[0]).cuda(),
                                               torch.from_numpy(csr[1]).cuda(), band_hint=64)
            rp, ci = o.normalize(*csr)
        q, dout = _draw((B, H, T, D), dt, 50), _draw((B, H, T, D), dt, 51)
        k, v = _draw((B, Hkv, T, D), dt, 52), _draw((B, Hkv, T, D), dt, 53)
        out, lse = sa.sparse_attn_fwd(q, k, v, g, scale)
        dq, dk, dv = sa.sparse_attn_bwd(q, k, v, out, lse, dout, g, scale)
        sa.sparse_attn_check_device()
    finally:
        sa.sparse_attn_set_path(sa.SA_PATH_AUTO)
    G = H // Hkv
    for b in range(B):
        for hk in range(Hkv):
            kh, vh = to_oracle(k[b, hk], dtype), to_oracle(v[b, hk], dtype)
            sdk = np.zeros((T, D))
            sdv = np.zeros((T, D))
            for h in range(hk * G, (hk + 1) * G):
                qh, doh = to_oracle(q[b, h], dtype), to_oracle(dout[b, h], dtype)
                r_out, r_lse = o.fwd(qh, kh, vh, rp, ci, scale, dtype=dtype)
                r_dq, r_dk, r_dv = o.bwd(qh, kh, vh, doh, rp, ci, scale, dtype=dtype)
                tag = f"{name}[b={b},h={h},path={path}]"
                compare(out[b, h], r_out, dtype, tag + " out")
                compare(lse[b, h], r_lse, dtype, tag + " lse")
                compare(dq[b, h], r_dq, dtype, tag + " dq")
                sdk += r_dk
                sdv += r_dv
            tag = f"{name}[b={b},kv head={hk},path={path}]"
            compare(dk[b, hk], sdk, dtype, tag + " dk (group sum)")
            compare(dv[b, hk], sdv, dtype, tag + " dv (group sum)")


def test_gqa_with_one_group_equals_repeated_heads():
    """Hkv < H gives the same forward as full multi-head attention on keys
    and values repeated per group (bitwise: same kernels, same operands)."""
    import sparse_graph_causal_b200 as sa
    B, H, Hkv, T, D = 1, 4, 2, 1000, 64
    g = sa.sparse_attn_graph_build_structured(T, 32, list(range(0, 10)))
    q = _draw((B, H, T, D), torch.bfloat16, 60)
    k, v = _draw((B, Hkv, T, D), torch.bfloat16, 61), _draw((B, Hkv, T, D), torch.bfloat16, 62)
    out, lse = sa.sparse_attn_fwd(q, k, v, g, 0.125)
    kr = k.repeat_interleave(H // Hkv, dim=1).contiguous()
    vr = v.repeat_interleave(H // Hkv, dim=1).contiguous()
    out2, lse2 = sa.sparse_attn_fwd(q, kr, vr, g, 0.125)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_gqa_shape_errors():
    import sparse_graph_causal_b200 as sa
    g = sa.sparse_attn_graph_build_structured(128, 8, [])
    q = torch.zeros(1, 4, 128, 64, dtype=torch.bfloat16, device="cuda")
    k3 = torch.zeros(1, 3, 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SparseAttentionError) as e:   # 3 does not divide 4
        sa.sparse_attn_fwd(q, k3, k3, g, 1.0)
    assert e.value.status == sa.SA_ERR_INVALID_ARG
