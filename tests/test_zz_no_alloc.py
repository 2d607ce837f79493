"""sparse_attn_bwd_noalloc, the backward for callers that cannot allocate
device memory when they call it (a host under a fixed device-memory plan, or
code inside an allocator hook).  It is called through the C ABI and must give
the same gradients as sparse_attn_bwd, within the tolerance of the other
parity tests, on two calls in a row (the second call reuses the library's
fixed scratch array left as the first call wrote it).  This file is collected
last so that a run stopping at the first failure has run every other test."""
import ctypes
from dataclasses import replace

import pytest
import torch

import synth
from gpu_util import compare

pytestmark = pytest.mark.gpu


def _call_noalloc(sa, q, k, v, out, lse, dout, g, scale, dq, dk, dv):
    ts = [sa._tensor(x, n) for x, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"),
                                        (dout, "dout"), (dq, "dq"), (dk, "dk"), (dv, "dv"))]
    r = [ctypes.byref(t) for t in ts]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return sa._lib.sparse_attn_bwd_noalloc(r[0], r[1], r[2], r[3], lse.data_ptr(), r[4],
                                           g.handle, float(scale), r[5], r[6], r[7], stream)


def test_bwd_noalloc_matches_bwd():
    import sparse_graph_causal_b200 as sa
    w = replace(synth.WORKLOADS["spatiallm_16k"], T=5000)
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    x = synth.make_qkv(w, device="cuda")
    out, lse = sa.sparse_attn_fwd(x["q"], x["k"], x["v"], g, w.scale)
    ref = sa.sparse_attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale)
    ref = [t.double().cpu().numpy() for t in ref]
    for call in range(2):
        dq, dk, dv = (torch.full_like(x["q"], float("nan")) for _ in range(3))
        st = _call_noalloc(sa, x["q"], x["k"], x["v"], out, lse, x["dout"], g, w.scale,
                           dq, dk, dv)
        assert st == sa.SA_OK, sa.sparse_attn_status_string(st)
        sa.sparse_attn_check_device()
        for got, r, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
            compare(got, r, w.dtype, f"noalloc call {call} {name}")


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
