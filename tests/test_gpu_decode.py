"""Decode (one new query per batch row and head against a KV cache) on the
GPU against the CPU oracle: the query at position p attends to N(p) of the
graph, i.e. it is row p of the full computation, with query head h reading
cache head h / (H / Hkv).  Also checked against row p of the GPU forward on
the whole sequence, and for an out-of-range position (flagged on the device,
no fault)."""
import math

import numpy as np
import pytest
import torch

import synth
from gpu_util import compact, compare, to_oracle

pytestmark = pytest.mark.gpu


def _draw(shape, dtype, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.empty(shape, dtype=torch.float32, device="cuda").normal_(
        0.0, 1.0, generator=g).to(dtype)


CASES = [
    # name, B, H, Hkv, Tmax, D, dtype, W, exps, positions, csr
    ("dec_d64_gqa2", 3, 4, 2, 2000, 64, torch.bfloat16, 32, range(0, 11), (0, 777, 1999), None),
    ("dec_d64_mha", 2, 4, 4, 1500, 64, torch.bfloat16, 32, range(0, 11), (31, 1024), None),
    ("dec_d128_gqa4", 2, 8, 2, 3000, 128, torch.bfloat16, 256, (8, 9, 10, 11), (300, 2999), None),
    ("dec_d32_fp32", 2, 2, 1, 900, 32, torch.float32, 8, range(0, 9), (5, 640), None),
    ("dec_long_window", 1, 2, 2, 5000, 64, torch.bfloat16, 4096, (), (4999,), None),
    ("dec_csr", 2, 2, 1, 1200, 64, torch.bfloat16, 0, (), (0, 1100),
     synth.csr_random_rows(1200, seed=21)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_decode_parity(case, oracle_lib):
    import sparse_graph_causal_b200 as sa
    name, B, H, Hkv, Tmax, D, dt, W, exps, positions, csr = case
    o = oracle_lib
    dtype = "bf16" if dt == torch.bfloat16 else "fp32"
    scale = 1.0 / math.sqrt(D)
    if csr is None:
        g = sa.sparse_attn_graph_build_structured(Tmax, W, list(exps))
    else:
        g = sa.sparse_attn_graph_build_csr(torch.from_numpy(csr[0]).cuda(),
                                           torch.from_numpy(csr[1]).cuda(), band_hint=64)
        rp_n, ci_n = o.normalize(*csr)
    q = _draw((B, H, 1, D), dt, 11)
    kc = _draw((B, Hkv, Tmax, D), dt, 12)
    vc = _draw((B, Hkv, Tmax, D), dt, 13)
    pos = torch.tensor(positions, dtype=torch.int64, device="cuda")
    out, lse = sa.sparse_attn_decode(q, kc, vc, pos, g, scale)
    sa.sparse_attn_check_device()
    grp = H // Hkv
    for b in range(B):
        p = positions[b]
        if csr is None:
            rp, ci = o.structured_rows(np.array([p]), W, exps)
        else:
            rp = np.array([0, rp_n[p + 1] - rp_n[p]], np.int64)
            ci = ci_n[rp_n[p]:rp_n[p + 1]].astype(np.int32)
        keys, local = compact(rp, ci)
        for h in range(H):
            qh = to_oracle(q[b, h], dtype)
            kh = to_oracle(kc[b, h // grp][torch.as_tensor(keys, device="cuda")], dtype)
            vh = to_oracle(vc[b, h // grp][torch.as_tensor(keys, device="cuda")], dtype)
            r_out, r_lse = o.fwd(qh, kh, vh, rp, local, scale, dtype=dtype)
            tag = f"{name}[b={b},h={h},pos={p}]"
            compare(out[b, h], r_out, dtype, tag + " out")
            compare(lse[b, h:h + 1], r_lse, dtype, tag + " lse")


def test_decode_equals_row_of_full_forward():
    """Decoding position p gives row p of sparse_attn_fwd over the sequence
    whose rows are the cache (the query written at row p)."""
    import sparse_graph_causal_b200 as sa
    B, H, T, D, W, exps = 2, 4, 1024, 64, 32, range(0, 10)
    scale = 0.125
    g = sa.sparse_attn_graph_build_structured(T, W, list(exps))
    qs, ks, vs = (_draw((B, H, T, D), torch.bfloat16, 30 + n) for n in range(3))
    full, full_lse = sa.sparse_attn_fwd(qs, ks, vs, g, scale)
    positions = (700, 1023)
    q = torch.stack([qs[b, :, positions[b]:positions[b] + 1] for b in range(B)])
    pos = torch.tensor(positions, dtype=torch.int64, device="cuda")
    out, lse = sa.sparse_attn_decode(q, ks, vs, pos, g, scale)
    sa.sparse_attn_check_device()
    for b in range(B):
        p = positions[b]
        compare(out[b, :, 0], full[b, :, p].double().cpu().numpy(), "bf16", f"row {p} out")
        compare(lse[b], full_lse[b, :, p].double().cpu().numpy(), "bf16", f"row {p} lse")


def test_decode_position_out_of_range_is_flagged():
    import sparse_graph_causal_b200 as sa
    B, H, T, D = 2, 2, 256, 64
    g = sa.sparse_attn_graph_build_structured(T, 16, [4, 5])
    q = _draw((B, H, 1, D), torch.bfloat16, 40)
    kc = _draw((B, H, T, D), torch.bfloat16, 41)
    vc = _draw((B, H, T, D), torch.bfloat16, 42)
    pos = torch.tensor([100, T], dtype=torch.int64, device="cuda")
    out, lse = sa.sparse_attn_decode(q, kc, vc, pos, g, 0.125)
    with pytest.raises(sa.SparseAttentionError) as e:
        sa.sparse_attn_check_device()
    assert e.value.status == sa.SA_ERR_CUDA
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    assert torch.all(torch.isfinite(lse[0]))
    sa.sparse_attn_check_device()   # the flag was cleared; the context is usable
