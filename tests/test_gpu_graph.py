"""Graph construction on the GPU against the oracle: bit-exact rowptr,
colidx and transpose lists; invalid graphs rejected."""
import math

import numpy as np
import pytest
import torch

import synth
from pins import closed_form_degree

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    import sparse_graph_causal_b200 as m
    return m


def _export(sa, g):
    return [t.cpu().numpy() for t in sa.sparse_attn_graph_export(g)]


@pytest.mark.parametrize("T,W,exps", [(1, 1, ()), (7, 1, (0, 1, 2)), (256, 8, range(0, 8)),
                                      (256, 256, ()), (1000, 17, (3, 5, 9)), (4097, 32, range(0, 13)),
                                      (16384, 32, range(0, 14)), (513, 600, ())])
def test_structured_graph_bit_exact(sa, oracle_lib, T, W, exps):
    g = sa.sparse_attn_graph_build_structured(T, W, list(exps), materialize=True)
    rp, ci, rrp, rci = _export(sa, g)
    orp, oci = oracle_lib.structured(T, W, exps)
    orr, orc = oracle_lib.reverse(orp, oci)
    assert np.array_equal(rp, orp) and np.array_equal(ci, oci)
    assert np.array_equal(rrp, orr) and np.array_equal(rci, orc)
    assert g.nnz == len(oci)


def test_structured_nnz_of_long_workloads(sa):
    """Implicit graphs (never materialised): nnz from the library equals the
    closed-form edge count."""
    for name, expect in (("band_32k", 125_831_168), ("extreme_128m", 7_113_539_120),
                         ("spatiallm_16k", 654_896)):
        w = synth.WORKLOADS[name]
        g = sa.sparse_attn_graph_build_structured(w.T, w.W, list(w.exps))
        assert g.nnz == expect, name


def _raw_csr_cases():
    rng = np.random.default_rng(11)
    T = 700
    rows = []
    for i in range(T):
        n = int(rng.integers(0, 9))
        r = list(rng.integers(0, i + 1, size=n))
        if i % 5 == 0:
            r += r[:2] + [i]
        rows.append(r)
    rp = np.zeros(T + 1, np.int64)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([x for r in rows for x in r], np.int32)
    return [("random_with_empty_rows", rp, ci, 0),
            ("graph_view_T5000", *synth.csr_random_rows(5000, seed=3), 64)]


@pytest.mark.parametrize("case", _raw_csr_cases(), ids=lambda c: c[0])
def test_csr_graph_bit_exact(sa, oracle_lib, case):
    name, rp, ci, band = case
    g = sa.sparse_attn_graph_build_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(),
                                       band_hint=band)
    nrp, nci, rrp, rci = _export(sa, g)
    orp, oci = oracle_lib.normalize(rp, ci)
    orr, orc = oracle_lib.reverse(orp, oci)
    assert np.array_equal(nrp, orp) and np.array_equal(nci, oci)
    assert np.array_equal(rrp, orr) and np.array_equal(rci, orc)


def test_csr_graph_view_1m_bit_exact(sa, oracle_lib):
    w = synth.WORKLOADS["csr_1m"]
    rp, ci = synth.csr_random_rows(w.T, seed=w.graph_seed)
    g = sa.sparse_attn_graph_build_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(),
                                       band_hint=w.band_hint)
    nrp, nci, rrp, rci = _export(sa, g)
    orp, oci = oracle_lib.normalize(rp, ci)
    assert np.array_equal(nrp, orp) and np.array_equal(nci, oci)
    orr, orc = oracle_lib.reverse(orp, oci)
    assert np.array_equal(rrp, orr) and np.array_equal(rci, orc)


@pytest.mark.parametrize("rows,status", [([[0], [2]], 2), ([[0], [-1]], 2), ([[0], [0, 1, 1]], 0)])
def test_csr_validation(sa, rows, status):
    rp = np.zeros(len(rows) + 1, np.int64)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([x for r in rows for x in r], np.int32)
    args = (torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda())
    if status == 0:
        g = sa.sparse_attn_graph_build_csr(*args)
        assert g.nnz == 3
    else:
        with pytest.raises(sa.SparseAttentionError) as e:
            sa.sparse_attn_graph_build_csr(*args)
        assert e.value.status == status


def test_csr_bad_rowptr_and_band(sa):
    rp = torch.tensor([0, 2, 1], dtype=torch.int64, device="cuda")
    ci = torch.tensor([0, 0], dtype=torch.int32, device="cuda")
    with pytest.raises(sa.SparseAttentionError) as e:
        sa.sparse_attn_graph_build_csr(rp, ci)
    assert e.value.status == 2
    rp, ci = synth.csr_random_rows(3000, seed=5, window=64)
    a = torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda()
    sa.sparse_attn_graph_build_csr(*a, band_hint=64)
    with pytest.raises(sa.SparseAttentionError) as e:
        sa.sparse_attn_graph_build_csr(*a, band_hint=65)
    assert e.value.status == 2


def test_bwd_workspace_size(sa):
    """Delta (4 bytes per query row) plus, for a structured graph with n
    distance links, the (p, dS) cache of its distance edges (8 n bytes per
    query row), each part rounded up to 256 bytes; CSR graphs and graphs
    without links need Delta only."""
    def up(x):
        return (x + 255) // 256 * 256

    B, H, T, D = 2, 3, 4097, 64
    q = torch.empty(B, H, T, D, dtype=torch.bfloat16, device="cuda")
    rows = B * H * T
    # window 32: links 2^0 .. 2^4 fall inside it, 2^5 and 2^9 remain
    g = sa.sparse_attn_graph_build_structured(T, 32, [0, 3, 5, 9])
    assert sa.sparse_attn_bwd_workspace_size(q, g) == up(4 * rows) + up(8 * 2 * rows)
    g_band = sa.sparse_attn_graph_build_structured(T, 32, [])
    assert sa.sparse_attn_bwd_workspace_size(q, g_band) == up(4 * rows)
    rp, ci = synth.csr_random_rows(T, seed=5, window=16, n_random=2, n_global=2)
    g_csr = sa.sparse_attn_graph_build_csr(torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda())
    assert sa.sparse_attn_bwd_workspace_size(q, g_csr) == up(4 * rows)
