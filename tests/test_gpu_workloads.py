"""The named workloads at their full sizes, in the launch configuration the
bench times: element-wise against the oracle where it finishes in seconds,
otherwise on sampled rows/keys the oracle computes one by one, plus
properties that hold at any size."""
import numpy as np
import pytest
import torch

import synth
from gpu_util import (compact, compare, local_rows, oracle_dkdv_keys, oracle_dq_rows,
                      oracle_fwd_rows, to_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    import sparse_graph_causal_b200 as m
    return m


def _fwd_bwd(sa, w, g, x, bwd=True):
    out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
    grads = None
    if bwd:
        grads = sa.sparse_attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale)
    sa.sparse_attn_check_device()
    return out, lse, grads


def test_spatiallm_16k_full(sa, oracle_lib):
    """B1 H4 T16384 D64 bf16, window 32 + 2^k (k = 0..13): every element."""
    w = synth.WORKLOADS["spatiallm_16k"]
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda")
    out, lse, (dq, dk, dv) = _fwd_bwd(sa, w, g, x)
    rp, ci = oracle_lib.structured(w.T, w.W, w.exps)
    BH = w.B * w.H
    for bh in range(BH):
        sl = [to_oracle(x[n].view(BH, w.T, w.D)[bh], w.dtype) for n in ("q", "k", "v", "dout")]
        rout, rlse = oracle_lib.fwd(*sl[:3], rp, ci, w.scale, dtype=w.dtype)
        rdq, rdk, rdv = oracle_lib.bwd(*sl, rp, ci, w.scale, dtype=w.dtype)
        for got, ref, nm in ((out, rout, "out"), (dq, rdq, "dq"), (dk, rdk, "dk"), (dv, rdv, "dv")):
            compare(got.view(BH, w.T, w.D)[bh], ref, w.dtype, f"{nm}[{bh}]")
        compare(lse.view(BH, w.T)[bh], rlse, w.dtype, f"lse[{bh}]")


def _band_sampled(sa, o, w, n_rows, key_blocks, bhs):
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda")
    out, lse, (dq, dk, dv) = _fwd_bwd(sa, w, g, x)
    BH = w.B * w.H
    for n, bh in enumerate(bhs):
        rows = synth.sample_rows(w.T, n_rows, seed=3000 + n)
        rp, ci = local_rows(o, rows, w.W, w.exps)
        rout, rlse = oracle_fwd_rows(o, x, bh, rows, rp, ci, w.scale, w.dtype)
        idx = torch.as_tensor(rows, device="cuda")
        compare(out.view(BH, w.T, w.D)[bh].index_select(0, idx), rout, w.dtype, f"out[{bh}]")
        compare(lse.view(BH, w.T)[bh].index_select(0, idx), rlse, w.dtype, f"lse[{bh}]")
        rdq = oracle_dq_rows(o, x, bh, rows, rp, ci, w.scale, w.dtype)
        compare(dq.view(BH, w.T, w.D)[bh].index_select(0, idx), rdq, w.dtype, f"dq[{bh}]")
    for n, (bh, k0, nk) in enumerate(key_blocks):
        keys = np.arange(k0, min(k0 + nk, w.T), dtype=np.int64)
        # every query that can list one of these keys: the window after it
        cand = np.arange(k0, min(w.T, k0 + nk + w.W - 1), dtype=np.int64)
        rp, ci = local_rows(o, cand, w.W, w.exps)
        rdk, rdv = oracle_dkdv_keys(o, x, bh, keys, cand, rp, ci, w.scale, w.dtype)
        idx = torch.as_tensor(keys, device="cuda")
        compare(dk.view(BH, w.T, w.D)[bh].index_select(0, idx), rdk, w.dtype, f"dk[{bh},{k0}]")
        compare(dv.view(BH, w.T, w.D)[bh].index_select(0, idx), rdv, w.dtype, f"dv[{bh},{k0}]")
    # properties at every size: sum_j dV_j = sum_i dO_i, sum_j dK_j = 0
    sdv = dv.double().sum(dim=2)
    sdo = x["dout"].double().sum(dim=2)
    rng = x["dout"].double().abs().sum(dim=2).max().item()
    assert (sdv - sdo).abs().max().item() <= 2e-3 * rng
    sdk = dk.double().sum(dim=2)
    assert sdk.abs().max().item() <= 2e-3 * dk.double().abs().sum(dim=2).max().item()
    return out, lse, x, g


def test_band_4k_full_causal(sa, oracle_lib):
    """B4 H32 T4096 D128, W = T: equals full causal attention (checked against
    the oracle on sampled rows and against torch's SDPA on every element)."""
    w = synth.WORKLOADS["band_4k_full"]
    out, lse, x, g = _band_sampled(sa, oracle_lib, w, 256, [(0, 0, 16), (77, 4000, 96)], [0, 127])
    ref = torch.nn.functional.scaled_dot_product_attention(x["q"], x["k"], x["v"], is_causal=True,
                                                           scale=w.scale)
    err = (out.float() - ref.float()).abs()
    assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3


def test_band_32k(sa, oracle_lib):
    """B4 H32 T32768 D128, W=4096: sampled rows and keys of a few slices."""
    w = synth.WORKLOADS["band_32k"]
    _band_sampled(sa, oracle_lib, w, 192, [(5, 0, 16), (100, 20000, 16)], [0, 64, 127])


def test_csr_1m_fwd(sa, oracle_lib):
    """B1 H8 T2^20 D64, raw CSR rows: one head in full, sampled rows of all."""
    w = synth.WORKLOADS["csr_1m"]
    rp_raw, ci_raw = synth.csr_random_rows(w.T, seed=w.graph_seed)
    g = sa.sparse_attn_graph_build_csr(torch.from_numpy(rp_raw).cuda(),
                                       torch.from_numpy(ci_raw).cuda(), band_hint=w.band_hint)
    x = synth.make_qkv(w, device="cuda", with_dout=False)
    out, lse, _ = _fwd_bwd(sa, w, g, x, bwd=False)
    rp, ci = oracle_lib.normalize(rp_raw, ci_raw)
    BH = w.B * w.H
    sl = [to_oracle(x[n].view(BH, w.T, w.D)[3], w.dtype) for n in ("q", "k", "v")]
    rout, rlse = oracle_lib.fwd(*sl, rp, ci, w.scale, dtype=w.dtype)
    compare(out.view(BH, w.T, w.D)[3], rout, w.dtype, "out[3]")
    compare(lse.view(BH, w.T)[3], rlse, w.dtype, "lse[3]")
    for bh in range(BH):
        rows = synth.sample_rows(w.T, 512, seed=4000 + bh)
        lrp, lci = local_rows(oracle_lib, rows, csr=(rp, ci))
        rout, rlse = oracle_fwd_rows(oracle_lib, x, bh, rows, lrp, lci, w.scale, w.dtype)
        idx = torch.as_tensor(rows, device="cuda")
        compare(out.view(BH, w.T, w.D)[bh].index_select(0, idx), rout, w.dtype, f"out[{bh}]")
        compare(lse.view(BH, w.T)[bh].index_select(0, idx), rlse, w.dtype, f"lse[{bh}]")


def test_extreme_128m_fwd(sa, oracle_lib):
    """B1 H1 T2^27 D64, window 32 + 2^k (k = 0..26), inputs drawn on the
    device: 4096 sampled rows against the oracle."""
    w = synth.WORKLOADS["extreme_128m"]
    torch.cuda.empty_cache()
    free, _ = torch.cuda.mem_get_info()
    need = 4 * w.T * w.D * 2 + 4 * w.T + (2 << 30)
    if free < need:
        pytest.skip(f"needs {need >> 30} GiB free on the device, has {free >> 30}")
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda", with_dout=False)
    out, lse, _ = _fwd_bwd(sa, w, g, x, bwd=False)
    rows = synth.sample_rows(w.T, 4096, seed=3005)
    rp, ci = local_rows(oracle_lib, rows, w.W, w.exps)
    rout, rlse = oracle_fwd_rows(oracle_lib, x, 0, rows, rp, ci, w.scale, w.dtype)
    idx = torch.as_tensor(rows, device="cuda")
    compare(out.view(w.T, w.D).index_select(0, idx), rout, w.dtype, "out")
    compare(lse.view(w.T).index_select(0, idx), rlse, w.dtype, "lse")
    del x, out, lse
    torch.cuda.empty_cache()


def test_gqa_16k_full(sa, oracle_lib):
    """B1 H8 over 2 key/value heads, T16384 D64 bf16, window 32 + 2^k
    (k = 0..13): every element.  out, lse and dq per query head from the
    oracle on its key/value head; dk and dv of a key/value head are the sums
    of the oracle's gradients over the 4 query heads of its group."""
    w = synth.WORKLOADS["gqa_16k"]
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda")
    out, lse, (dq, dk, dv) = _fwd_bwd(sa, w, g, x)
    rp, ci = oracle_lib.structured(w.T, w.W, w.exps)
    G = w.H // w.kv_heads
    for hk in range(w.kv_heads):
        kh, vh = to_oracle(x["k"][0, hk], w.dtype), to_oracle(x["v"][0, hk], w.dtype)
        sdk, sdv = np.zeros((w.T, w.D)), np.zeros((w.T, w.D))
        for h in range(hk * G, (hk + 1) * G):
            qh, doh = to_oracle(x["q"][0, h], w.dtype), to_oracle(x["dout"][0, h], w.dtype)
            rout, rlse = oracle_lib.fwd(qh, kh, vh, rp, ci, w.scale, dtype=w.dtype)
            rdq, rdk, rdv = oracle_lib.bwd(qh, kh, vh, doh, rp, ci, w.scale, dtype=w.dtype)
            compare(out[0, h], rout, w.dtype, f"out[h={h}]")
            compare(lse[0, h], rlse, w.dtype, f"lse[h={h}]")
            compare(dq[0, h], rdq, w.dtype, f"dq[h={h}]")
            sdk += rdk
            sdv += rdv
        compare(dk[0, hk], sdk, w.dtype, f"dk[kv head {hk}] (group sum)")
        compare(dv[0, hk], sdv, w.dtype, f"dv[kv head {hk}] (group sum)")


def test_dist_16k_full(sa, oracle_lib):
    """Learned-coordinate scores, B1 H4 T16384 D64 bf16 over the window 32 +
    2^k graph, coordinates N(0, 1), scale 0.5: every element of out, lse, da,
    dc and dv (da and dc carry the coordinates' scale and are bounded against
    their own range, as in the small learned-coordinate cases)."""
    w = synth.WORKLOADS["dist_16k"]
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    a, c = synth.make_coords(w, device="cuda")
    x = synth.make_qkv(w, device="cuda")
    v, dout = x["v"], x["dout"]
    out, lse = sa.sparse_attn_dist_fwd(a, c, v, g, w.scale)
    da, dc, dv = sa.sparse_attn_dist_bwd(a, c, v, out, lse, dout, g, w.scale)
    sa.sparse_attn_check_device()
    rp, ci = oracle_lib.structured(w.T, w.W, w.exps)
    BH = w.B * w.H
    for bh in range(BH):
        ah = a.view(BH, w.T, 3)[bh].cpu().numpy()
        ch = c.view(BH, w.T, 3)[bh].cpu().numpy()
        vh = to_oracle(v.view(BH, w.T, w.D)[bh], w.dtype)
        doh = to_oracle(dout.view(BH, w.T, w.D)[bh], w.dtype)
        rout, rlse = oracle_lib.dist_fwd(ah, ch, vh, rp, ci, w.scale, dtype=w.dtype,
                                         cdtype="fp32")
        rda, rdc, rdv = oracle_lib.dist_bwd(ah, ch, vh, doh, rp, ci, w.scale, dtype=w.dtype,
                                            cdtype="fp32")
        tag = f"dist_16k[bh={bh}]"
        compare(out.view(BH, w.T, w.D)[bh], rout, w.dtype, tag + " out")
        compare(lse.view(BH, w.T)[bh], rlse, w.dtype, tag + " lse")
        compare(da.view(BH, w.T, 3)[bh], rda, w.dtype, tag + " da", unit_range=1.0)
        compare(dc.view(BH, w.T, 3)[bh], rdc, w.dtype, tag + " dc", unit_range=1.0)
        compare(dv.view(BH, w.T, w.D)[bh], rdv, w.dtype, tag + " dv")


def test_decode_16k_full(sa, oracle_lib):
    """Decode as the bench times it: 64 sequences, 8 query heads over 2 cache
    heads, caches of 16384 rows (D64 bf16), positions drawn in [T/2, T), the
    window 32 + 2^k graph: every query against the oracle on its row p of
    the graph."""
    w = synth.WORKLOADS["decode_16k"]
    B, H, Hk, T, D = w.B, w.H, w.kv_heads, w.T, w.D
    gen = torch.Generator(device="cuda")
    gen.manual_seed(w.seed + 17)
    q = torch.empty((B, H, 1, D), dtype=torch.float32, device="cuda").normal_(
        generator=gen).to(w.torch_dtype)
    kc = torch.empty((B, Hk, T, D), dtype=torch.float32, device="cuda").normal_(
        generator=gen).to(w.torch_dtype)
    vc = torch.empty((B, Hk, T, D), dtype=torch.float32, device="cuda").normal_(
        generator=gen).to(w.torch_dtype)
    pos = torch.randint(T // 2, T, (B,), generator=gen, device="cuda", dtype=torch.int64)
    g = sa.sparse_attn_graph_build_structured(T, w.W, list(w.exps))
    out, lse = sa.sparse_attn_decode(q, kc, vc, pos, g, w.scale)
    sa.sparse_attn_check_device()
    grp = H // Hk
    for b, p in enumerate(pos.cpu().tolist()):
        rp, ci = oracle_lib.structured_rows(np.array([p]), w.W, w.exps)
        keys, local = compact(rp, ci)
        kidx = torch.as_tensor(keys, device="cuda")
        for hk in range(Hk):
            kh = to_oracle(kc[b, hk].index_select(0, kidx), w.dtype)
            vh = to_oracle(vc[b, hk].index_select(0, kidx), w.dtype)
            for h in range(hk * grp, (hk + 1) * grp):
                rout, rlse = oracle_lib.fwd(to_oracle(q[b, h], w.dtype), kh, vh, rp, local,
                                            w.scale, dtype=w.dtype)
                compare(out[b, h], rout, w.dtype, f"decode_16k[b={b},h={h},pos={p}] out")
                compare(lse[b, h:h + 1], rlse, w.dtype, f"decode_16k[b={b},h={h},pos={p}] lse")
