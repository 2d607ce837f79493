"""GPU forward/backward against the CPU oracle, element by element, on
sizes the oracle finishes in seconds: several 128-row tiles, ragged tails,
every supported head size and dtype, structured and CSR graphs, and both
kernel paths (tcgen05 band tiles + gather, and gather only)."""
import math
from dataclasses import replace

import numpy as np
import pytest
import torch

import synth
from gpu_util import compare, to_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    import sparse_graph_causal_b200 as m
    return m


def _wl(name, B, H, T, D, dtype, W, exps=(), std=1.0, seed=1, csr=None, band=0, mult=1.0):
    w = synth.Workload(name=name, B=B, H=H, T=T, D=D, dtype=dtype, W=W, exps=tuple(exps),
                       input_std=std, scale=mult / math.sqrt(D), seed=seed, band_hint=band,
                       csr=csr is not None)
    return w, csr


def _random_csr_with_empty(T, seed):
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(T):
        n = 0 if i % 7 == 3 else int(rng.integers(1, 12))
        rows.append(list(rng.integers(0, i + 1, size=n)))
    rp = np.zeros(T + 1, np.int64)
    rp[1:] = np.cumsum([len(r) for r in rows])
    return rp, np.array([x for r in rows for x in r], np.int32)


CASES = [
    _wl("tiny", 1, 2, 256, 32, "fp32", 8, range(0, 8), seed=1001),
    _wl("tiny_full", 1, 2, 256, 32, "fp32", 256, (), seed=1001),
    _wl("t1", 1, 1, 1, 64, "bf16", 4, range(0, 3)),
    _wl("d64_ragged", 2, 2, 300, 64, "bf16", 32, range(0, 9)),
    _wl("d64_self_only", 1, 2, 129, 64, "bf16", 1, (0, 3, 5)),
    _wl("d64_full", 1, 1, 520, 64, "bf16", 520, ()),
    _wl("d64_small_values", 1, 4, 700, 64, "bf16", 32, range(0, 10), std=0.125),
    # scale 0: every kept score is 0 (uniform weights over each row's keys)
    _wl("d64_zero_scale", 1, 2, 300, 64, "bf16", 32, range(0, 9), mult=0.0),
    _wl("d128_w200", 1, 2, 1000, 128, "bf16", 200, (8, 9)),
    _wl("d128_band", 2, 1, 777, 128, "bf16", 256, ()),
    _wl("d32_bf16", 1, 2, 200, 32, "bf16", 16, range(0, 8)),
    # bf16 D = 32 runs on the D = 64 tensor-core tiles with zero-extended rows
    _wl("d32_links_ragged", 2, 2, 389, 32, "bf16", 32, range(0, 9)),
    _wl("d32_band_only", 1, 2, 600, 32, "bf16", 300, ()),
    _wl("csr_d32", 1, 2, 1500, 32, "bf16", 0, (), csr=synth.csr_random_rows(1500, seed=43),
        band=64),
    _wl("d64_fp32", 1, 2, 333, 64, "fp32", 40, range(0, 9)),
    _wl("d128_fp32", 1, 1, 150, 128, "fp32", 64, (7,)),
    _wl("csr_view_3000", 1, 2, 3000, 64, "bf16", 0, (),
        csr=synth.csr_random_rows(3000, seed=9), band=64),
    _wl("csr_empty_rows", 1, 2, 400, 64, "bf16", 0, (), csr=_random_csr_with_empty(400, 4)),
    _wl("csr_d128", 1, 1, 600, 128, "bf16", 0, (), csr=synth.csr_random_rows(600, seed=8), band=64),
    # CSR rows with a band but no shared key prefix, and with a prefix longer
    # than the band (the forward's dense prefix block: none, and 40 keys)
    _wl("csr_no_prefix", 1, 2, 2000, 64, "bf16", 0, (),
        csr=synth.csr_random_rows(2000, seed=41, n_global=0), band=64),
    _wl("csr_prefix40_band16", 1, 2, 1500, 64, "bf16", 0, (),
        csr=synth.csr_random_rows(1500, seed=42, window=16, n_global=40), band=16),
]


def build_graph(sa, o, w, csr):
    if csr is None:
        g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
        rp, ci = o.structured(w.T, w.W, w.exps)
    else:
        rp_raw, ci_raw = csr
        g = sa.sparse_attn_graph_build_csr(torch.from_numpy(rp_raw).cuda(),
                                           torch.from_numpy(ci_raw).cuda(), band_hint=w.band_hint)
        rp, ci = o.normalize(rp_raw, ci_raw)
    return g, rp, ci


def run_and_check(sa, o, w, csr, path, unit_range=None):
    sa.sparse_attn_set_path(path)
    try:
        g, rp, ci = build_graph(sa, o, w, csr)
        x = synth.make_qkv(w, device="cuda")
        out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
        dq, dk, dv = sa.sparse_attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale)
        sa.sparse_attn_check_device()
    finally:
        sa.sparse_attn_set_path(sa.SA_PATH_AUTO)
    BH = w.B * w.H
    for bh in range(BH):
        sl = [to_oracle(x[n].view(BH, w.T, w.D)[bh], w.dtype) for n in ("q", "k", "v", "dout")]
        rout, rlse = o.fwd(sl[0], sl[1], sl[2], rp, ci, w.scale, dtype=w.dtype)
        rdq, rdk, rdv = o.bwd(sl[0], sl[1], sl[2], sl[3], rp, ci, w.scale, dtype=w.dtype)
        tag = f"{w.name}[bh={bh},path={path}]"
        u = unit_range
        compare(out.view(BH, w.T, w.D)[bh], rout, w.dtype, tag + " out", unit_range=u)
        compare(lse.view(BH, w.T)[bh], rlse, w.dtype, tag + " lse", unit_range=u)
        compare(dq.view(BH, w.T, w.D)[bh], rdq, w.dtype, tag + " dq", unit_range=u)
        compare(dk.view(BH, w.T, w.D)[bh], rdk, w.dtype, tag + " dk", unit_range=u)
        compare(dv.view(BH, w.T, w.D)[bh], rdv, w.dtype, tag + " dv", unit_range=u)


@pytest.mark.parametrize("path", [0, 1], ids=["auto", "gather"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_parity_small(sa, oracle_lib, case, path):
    w, csr = case
    run_and_check(sa, oracle_lib, w, csr, path)


# Scores scaled by 2/sqrt(D) (or -2/sqrt(D)): spread of about 3 units of
# log2 per standard deviation, so a row's running max often grows by more than
# 2^8 after its first edges and the kernels' deferred rescaling of O and l runs
# (on both edge classes: some 60 distance-link and 200 band-block rescales over
# the 1100 rows of the first case's first head).  Gradients reach |x| ~ 8
# here, where the fixed max-abs bound of the unit-scale cases no longer
# applies: the comparison bounds max-abs relative to max|ref| instead and
# lets mean-abs grow beyond |x| = 4.
SHARP_CASES = [
    _wl("d64_sharp", 1, 2, 1100, 64, "bf16", 32, range(0, 11), seed=77, mult=2.0),
    _wl("d64_negative_scale", 1, 2, 1100, 64, "bf16", 32, range(0, 11), seed=77, mult=-2.0),
    _wl("d64_band_sharp", 1, 1, 900, 64, "bf16", 300, (), seed=78, mult=2.0),
    _wl("d128_sharp", 1, 1, 700, 128, "bf16", 200, (8, 9), seed=77, mult=2.0),
    _wl("d128_band_sharp", 1, 1, 777, 128, "bf16", 256, (), seed=79, mult=2.0),
    _wl("csr_sharp", 1, 1, 900, 64, "bf16", 0, (), csr=synth.csr_random_rows(900, seed=12),
        band=64, mult=2.0),
    _wl("d64_fp32_sharp", 1, 1, 333, 64, "fp32", 40, range(0, 9), seed=80, mult=2.0),
]


@pytest.mark.parametrize("path", [0, 1], ids=["auto", "gather"])
@pytest.mark.parametrize("case", SHARP_CASES, ids=lambda c: c[0].name)
def test_parity_sharp_softmax(sa, oracle_lib, case, path):
    w, csr = case
    run_and_check(sa, oracle_lib, w, csr, path, unit_range=4.0)


@pytest.mark.parametrize("path", [0, 1], ids=["auto", "gather"])
def test_causality_bitwise(sa, path):
    """Changing q/k/v at positions > i leaves rows <= i bitwise unchanged."""
    w = synth.WORKLOADS["spatiallm_16k"]
    w = replace(w, T=2000)
    sa.sparse_attn_set_path(path)
    try:
        g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
        x = synth.make_qkv(w, device="cuda", with_dout=False)
        out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
        i0 = 1234
        for n in ("q", "k", "v"):
            x[n][:, :, i0 + 1:] = torch.randn_like(x[n][:, :, i0 + 1:])
        out2, lse2 = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
    finally:
        sa.sparse_attn_set_path(0)
    assert torch.equal(out[:, :, : i0 + 1], out2[:, :, : i0 + 1])
    assert torch.equal(lse[:, :, : i0 + 1], lse2[:, :, : i0 + 1])
    assert not torch.equal(out[:, :, i0 + 1:], out2[:, :, i0 + 1:])


def test_backward_deterministic(sa):
    w = replace(synth.WORKLOADS["spatiallm_16k"], T=4096)
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda")
    out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
    r1 = sa.sparse_attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale)
    r2 = sa.sparse_attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale)
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)


def test_argument_errors(sa):
    w = replace(synth.WORKLOADS["spatiallm_16k"], T=256)
    g = sa.sparse_attn_graph_build_structured(300, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda", with_dout=False)
    with pytest.raises(sa.SparseAttentionError) as e:     # T mismatch
        sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    g = sa.sparse_attn_graph_build_structured(256, w.W, list(w.exps))
    with pytest.raises(sa.SparseAttentionError):           # non-finite scale
        sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, float("nan"))
    q48 = torch.zeros(1, 1, 256, 48, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SparseAttentionError) as e:      # head size
        sa.sparse_attn_fwd(q48, q48, q48, g, 1.0)
    assert e.value.status == sa.SA_ERR_UNSUPPORTED


def test_many_slices_on_tensor_cores(sa, oracle_lib):
    """B*H above 65,535 (short sequences, many heads) runs on the band
    kernels too: fwd and bwd of sampled slices against the oracle."""
    w = _wl("many_slices", 2, 32800, 130, 64, "bf16", 32, range(0, 8), seed=9)[0]
    o = oracle_lib
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    rp, ci = o.structured(w.T, w.W, w.exps)
    x = synth.make_qkv(w, device="cuda")
    n0 = sa.sparse_attn_launch_count()
    sa.sparse_attn_profile_begin(True)
    out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
    dq, dk, dv = sa.sparse_attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale)
    prof = sa.sparse_attn_profile_end()
    sa.sparse_attn_check_device()
    assert set(prof) == {"band_fwd", "band_bwd_dq", "band_bwd_dkdv"}, prof
    assert sa.sparse_attn_launch_count() - n0 == 3
    BH = w.B * w.H
    for bh in (0, 1, 40000, BH - 1):
        sl = [to_oracle(x[n].view(BH, w.T, w.D)[bh], w.dtype) for n in ("q", "k", "v", "dout")]
        rout, rlse = o.fwd(sl[0], sl[1], sl[2], rp, ci, w.scale, dtype=w.dtype)
        rdq, rdk, rdv = o.bwd(*sl, rp, ci, w.scale, dtype=w.dtype)
        for got, ref, n in ((out, rout, "out"), (dq, rdq, "dq"), (dk, rdk, "dk"), (dv, rdv, "dv")):
            compare(got.view(BH, w.T, w.D)[bh], ref, w.dtype, f"many_slices[{bh}] {n}")
        compare(lse.view(BH, w.T)[bh], rlse, w.dtype, f"many_slices[{bh}] lse")


@pytest.mark.parametrize("kind", ["links", "band", "csr"])
def test_d32_bf16_on_tensor_cores(sa, oracle_lib, kind):
    """bf16 with D = 32 takes the tcgen05 band kernels (not the gather
    kernels) for every graph kind, and matches the oracle there."""
    w, csr = {"links": _wl("d32_tc_links", 1, 2, 700, 32, "bf16", 32, range(0, 10), seed=5),
              "band": _wl("d32_tc_band", 1, 2, 700, 32, "bf16", 256, (), seed=6),
              "csr": _wl("d32_tc_csr", 1, 2, 900, 32, "bf16", 0, (),
                         csr=synth.csr_random_rows(900, seed=44), band=64)}[kind]
    o = oracle_lib
    g, rp, ci = build_graph(sa, o, w, csr)
    x = synth.make_qkv(w, device="cuda")
    sa.sparse_attn_profile_begin(True)
    out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
    dq, dk, dv = sa.sparse_attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale)
    prof = sa.sparse_attn_profile_end()
    sa.sparse_attn_check_device()
    assert set(prof) == {"band_fwd", "band_bwd_dq", "band_bwd_dkdv"}, prof
    BH = w.B * w.H
    for bh in range(BH):
        sl = [to_oracle(x[n].view(BH, w.T, w.D)[bh], w.dtype) for n in ("q", "k", "v", "dout")]
        rout, rlse = o.fwd(sl[0], sl[1], sl[2], rp, ci, w.scale, dtype=w.dtype)
        rdq, rdk, rdv = o.bwd(*sl, rp, ci, w.scale, dtype=w.dtype)
        for got, ref, n in ((out, rout, "out"), (dq, rdq, "dq"), (dk, rdk, "dk"), (dv, rdv, "dv")):
            compare(got.view(BH, w.T, w.D)[bh], ref, w.dtype, f"{w.name}[{bh}] {n}")
        compare(lse.view(BH, w.T)[bh], rlse, w.dtype, f"{w.name}[{bh}] lse")
