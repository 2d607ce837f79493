"""The forward's second pass over the long distance links of a structured
graph: the band kernel takes the window and the links shorter than 2^13
rows, the link pass the rest, class by class, and merges them into out and
lse.  The automatic choice takes it only when K and V hold 2 GiB or more,
1 GiB or more per slice (the extreme-length workloads); here SA_LINKS_SPLIT
forces it on sizes whose K and V are below that.  Checked against the gather kernels (every edge in one
pass) on every row, against the one-pass band kernel, and against the oracle
on sampled rows, for D = 32, 64, 128 and grouped heads."""
import math

import numpy as np
import pytest
import torch

import synth
from gpu_util import compact, compare, gather_rows, local_rows

pytestmark = pytest.mark.gpu


def _wl(name, H, Hkv, T, D, kmax, seed, B=1):
    return synth.Workload(name=name, B=B, H=H, T=T, D=D, dtype="bf16", W=32,
                          exps=tuple(range(0, kmax + 1)), input_std=1.0,
                          scale=1.0 / math.sqrt(D), seed=seed, Hkv=Hkv, bwd=False)


CASES = [
    _wl("links_d64", 1, 1, 1 << 19, 64, 18, 71),
    _wl("links_gqa", 2, 1, 1 << 19, 64, 18, 72),
    _wl("links_d32", 1, 1, 1 << 20, 32, 19, 73),
    _wl("links_d128", 1, 1, 1 << 18, 128, 17, 74),
    # ragged: the last tile partial, the last class one tile short
    _wl("links_ragged", 1, 1, (1 << 19) + 77, 64, 18, 75),
    # two batch rows of grouped heads: slice b * H + h reads K/V slice
    # b * Hkv + h / (H / Hkv)
    _wl("links_b2_gqa", 4, 2, 1 << 18, 64, 17, 77, B=2),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_link_pass_matches_one_pass_and_oracle(oracle_lib, w):
    import sparse_graph_causal_b200 as sa
    o = oracle_lib
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda", with_dout=False)
    sa.sparse_attn_set_link_pass(sa.SA_LINKS_SPLIT)
    try:
        sa.sparse_attn_profile_begin(True)
        out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
        prof = sa.sparse_attn_profile_end()
        sa.sparse_attn_check_device()
        assert set(prof) == {"band_fwd", "link_pass"}, prof
        # one pass (the automatic choice at this size)
        sa.sparse_attn_set_link_pass(sa.SA_LINKS_AUTO)
        sa.sparse_attn_profile_begin(True)
        out2, lse2 = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
        prof = sa.sparse_attn_profile_end()
        sa.sparse_attn_check_device()
        assert set(prof) == {"band_fwd"}, prof
    finally:
        sa.sparse_attn_set_link_pass(sa.SA_LINKS_AUTO)
    compare(out, out2.double().cpu().numpy(), w.dtype, f"{w.name} out vs band one pass")
    compare(lse, lse2.double().cpu().numpy(), w.dtype, f"{w.name} lse vs band one pass")
    del out2, lse2
    # every edge in one pass, on the gather kernels
    sa.sparse_attn_set_path(sa.SA_PATH_GATHER)
    try:
        out1, lse1 = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
        sa.sparse_attn_check_device()
    finally:
        sa.sparse_attn_set_path(sa.SA_PATH_AUTO)
    compare(out, out1.double().cpu().numpy(), w.dtype, f"{w.name} out vs one pass")
    compare(lse, lse1.double().cpu().numpy(), w.dtype, f"{w.name} lse vs one pass")
    # the oracle on sampled rows: random ones, the rows around the first long
    # link (2^13) and around the class boundaries of the second pass
    span = 1 << 13
    extra = [span - 1, span, span + 1, span + 127, span + 128, 2 * span - 1, 2 * span + 200,
             w.T - 129, w.T - 128]
    rows = np.unique(np.concatenate([synth.sample_rows(w.T, 768, seed=w.seed), extra]))
    rp, ci = local_rows(o, rows, w.W, w.exps)
    keys, local = compact(rp, ci)
    G = w.H // w.kv_heads
    BH = w.B * w.H
    for bh in range(BH):
        kvbh = (bh // w.H) * w.kv_heads + (bh % w.H) // G
        q = gather_rows(x["q"], bh, rows, w.dtype)
        k = gather_rows(x["k"], kvbh, keys, w.dtype)
        v = gather_rows(x["v"], kvbh, keys, w.dtype)
        rout, rlse = o.fwd(q, k, v, rp, local, w.scale, dtype=w.dtype)
        idx = torch.as_tensor(rows, device="cuda")
        compare(out.view(BH, w.T, w.D)[bh].index_select(0, idx), rout, w.dtype,
                f"{w.name}[{bh}] out")
        compare(lse.view(BH, w.T)[bh].index_select(0, idx), rlse, w.dtype,
                f"{w.name}[{bh}] lse")
    del x, out, lse, out1, lse1
    g.close()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("H,lg,expect", [(16, 20, {"band_fwd"}), (4, 22, {"band_fwd", "link_pass"})],
                         ids=["16x2^20_one_pass", "4x2^22_two_passes"])
def test_link_pass_automatic_choice(H, lg, expect):
    """The automatic choice follows the length of one slice, not the job's
    size: 16 slices of 2^20 rows (K and V 4 GiB in all, 256 MiB a slice) run
    one pass, 4 slices of 2^22 (4 GiB, 1 GiB a slice) two.  Checked by the
    kernels that ran; the output rows are finite and lse holds at least the
    row's own score (every row keeps itself)."""
    import sparse_graph_causal_b200 as sa
    w = _wl(f"auto_{H}x{lg}", H, H, 1 << lg, 64, lg - 1, 76)
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda", with_dout=False)
    sa.sparse_attn_set_link_pass(sa.SA_LINKS_AUTO)
    sa.sparse_attn_profile_begin(True)
    out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
    prof = sa.sparse_attn_profile_end()
    sa.sparse_attn_check_device()
    assert set(prof) == expect, prof
    rows = torch.as_tensor(synth.sample_rows(w.T, 256, seed=w.seed), device="cuda")
    o = out[0].index_select(1, rows).float()
    assert torch.isfinite(o).all()
    self_score = (x["q"][0].index_select(1, rows).float() * x["k"][0].index_select(1, rows).float()).sum(-1) * w.scale
    assert (lse[0].index_select(1, rows) >= self_score - 1e-2).all()
    del x, out, lse
    g.close()
    torch.cuda.empty_cache()
