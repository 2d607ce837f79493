"""The bounded-wait failure path on the GPU, without a fault: a wait that
nothing completes gives up after its limit, the host reads the timeout from
the device error word, and the context stays usable."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    import sparse_graph_causal_b200 as m
    return m


def test_bounded_wait_timeout_is_reported_and_cleared(sa):
    sa.sparse_attn_check_device()  # nothing pending
    sa.sparse_attn_selftest_wait_timeout(20_000_000)
    with pytest.raises(sa.SparseAttentionError) as e:
        sa.sparse_attn_check_device()
    assert e.value.status == sa.SA_ERR_DEVICE_TIMEOUT
    sa.sparse_attn_check_device()  # the word was cleared

    # the context still runs the attention kernels
    w = synth.WORKLOADS["tiny"]
    x = synth.make_qkv(w, device="cuda", with_dout=False)
    q, k, v = (x[n].to(torch.bfloat16) for n in ("q", "k", "v"))
    q, k, v = (t.repeat(1, 1, 1, 2).contiguous() for t in (q, k, v))  # D = 64
    g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
    out, lse = sa.sparse_attn_fwd(q, k, v, g, 0.125)
    sa.sparse_attn_check_device()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_selftest_limit_is_checked(sa):
    with pytest.raises(sa.SparseAttentionError) as e:
        sa.sparse_attn_selftest_wait_timeout(10)
    assert e.value.status == sa.SA_ERR_INVALID_ARG
