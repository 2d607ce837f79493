"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle itself.  Each function takes an ``Oracle`` and
raises AssertionError on a mismatch, so the same pins also run against
deliberately broken builds of the oracle (test_oracle_mutants.py).

What pins what:
  graph     hand-enumerated lists (tests/golden), brute force from the dense
            mask rule, closed-form degrees, transpose identities, np.unique
  forward   hand-derived worked examples (tests/golden), full causal attention
            from torch's SDPA in float64 when W >= T, the dense numpy mask
            oracle, softmax invariants, causality
  backward  hand-derived gradients (tests/golden), central finite
            differences, torch autograd through the dense formulation,
            gradient invariants
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from oracle import OracleError
from oracle import dense

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _ev(x):
    env = {"log": math.log, "sqrt": math.sqrt}
    if isinstance(x, list):
        return np.array([_ev(e) for e in x], dtype=np.float64)
    return float(eval(x, {"__builtins__": {}}, env))


def _csr(rows):
    rowptr = np.zeros(len(rows) + 1, dtype=np.int64)
    rowptr[1:] = np.cumsum([len(r) for r in rows])
    colidx = np.array([j for r in rows for j in r], dtype=np.int32)
    return rowptr, colidx


def _csr_from_mask(mask):
    T = mask.shape[0]
    rowptr = np.zeros(T + 1, dtype=np.int64)
    rowptr[1:] = np.cumsum(mask.sum(axis=1))
    colidx = np.nonzero(mask)[1].astype(np.int32)   # row-major, ascending j
    return rowptr, colidx


def closed_form_degree(i, W, exps):
    """deg(i) = min(i+1, W) + #{distinct 2^k : W <= 2^k <= i}."""
    offs = {1 << k for k in exps}
    return min(i + 1, W) + sum(1 for o in offs if W <= o <= i)


def closed_form_in_degree(j, T, W, exps):
    """in-deg(j) = min(T-j, W) + #{distinct 2^k >= W : j + 2^k < T}."""
    offs = {1 << k for k in exps}
    return min(T - j, W) + sum(1 for o in offs if o >= W and j + o < T)


# ----------------------------------------------------------------- graph

def pin_graph_golden(o):
    g = _load("graph_T12_W3_k0-3.json")
    rowptr, colidx = o.structured(g["T"], g["W"], g["exps"])
    er, ec = _csr(g["rows"])
    assert int(rowptr[-1]) == g["nnz"]
    assert np.array_equal(rowptr, er) and np.array_equal(colidx, ec)


GRAPH_CASES = [(1, 1, ()), (7, 1, (0, 1, 2)), (64, 4, range(0, 6)), (256, 8, range(0, 8)),
               (300, 32, range(0, 9)), (1000, 17, (3, 5, 9)), (513, 600, ()), (129, 1, (0, 3, 3, 7))]


def pin_graph_bruteforce(o):
    for T, W, exps in GRAPH_CASES:
        rowptr, colidx = o.structured(T, W, exps)
        er, ec = _csr_from_mask(dense.structured_mask(T, W, exps))
        assert np.array_equal(rowptr, er), (T, W, exps)
        assert np.array_equal(colidx, ec), (T, W, exps)


def pin_graph_closed_forms(o):
    for T, W, exps in GRAPH_CASES:
        rowptr, colidx = o.structured(T, W, exps)
        deg = np.diff(rowptr)
        assert all(int(deg[i]) == closed_form_degree(i, W, exps) for i in range(T))
        rr, _ = o.reverse(rowptr, colidx)
        indeg = np.diff(rr)
        assert all(int(indeg[j]) == closed_form_in_degree(j, T, W, exps) for j in range(T))
    # edge counts of the named workloads, from the closed form summed by hand
    # (window part + distance part): tiny 2,020 + 1,032; 16k 523,792 + 131,104
    assert o.structured_nnz(256, 8, range(0, 8)) == 3052
    assert o.structured_nnz(256, 256, ()) == 256 * 257 // 2
    assert o.structured_nnz(16384, 32, range(0, 14)) == 654896


def pin_graph_rows_match_full(o):
    """Selected-row lists equal the same rows of the full graph."""
    for T, W, exps in GRAPH_CASES:
        rowptr, colidx = o.structured(T, W, exps)
        rows = np.array(sorted(set([0, T - 1, T // 2, T // 3])), dtype=np.int64)
        rr, rc = o.structured_rows(rows, W, exps)
        for n, i in enumerate(rows):
            assert np.array_equal(rc[rr[n]:rr[n + 1]], colidx[rowptr[i]:rowptr[i + 1]])


def pin_graph_reverse(o):
    for T, W, exps in GRAPH_CASES:
        rowptr, colidx = o.structured(T, W, exps)
        rr, rc = o.reverse(rowptr, colidx)
        er, ec = _csr_from_mask(dense.structured_mask(T, W, exps).T)
        assert np.array_equal(rr, er) and np.array_equal(rc, ec)
        r2, c2 = o.reverse(rr, rc)
        assert np.array_equal(r2, rowptr) and np.array_equal(c2, colidx)


def pin_graph_normalize(o):
    rng = np.random.default_rng(7)
    T = 200
    rows = []
    for i in range(T):
        n = int(rng.integers(0, 12))
        rows.append(list(rng.integers(0, i + 1, size=n)) + ([i] if i % 3 == 0 else []))
    rowptr, colidx = _csr(rows)
    nr, nc = o.normalize(rowptr, colidx)
    er, ec = _csr([sorted(set(int(x) for x in r)) for r in rows])
    assert np.array_equal(nr, er) and np.array_equal(nc, ec)
    # rejected graphs
    bad = [(_csr([[0], [2]]), "look-ahead edge"), (_csr([[0], [-1, 1]]), "negative key")]
    for (r, c), msg in bad:
        try:
            o.normalize(r, c)
        except OracleError as e:
            assert msg in str(e)
        else:
            raise AssertionError("invalid graph accepted: " + msg)
    try:
        o.normalize(np.array([0, 2, 1], dtype=np.int64), np.array([0, 0], dtype=np.int32))
    except OracleError as e:
        assert "rowptr" in str(e)
    else:
        raise AssertionError("decreasing rowptr accepted")


# --------------------------------------------------------------- forward

def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def pin_fwd_golden(o):
    for ex in _load("worked_attention.json")["examples"]:
        rowptr, colidx = _csr(ex["rows"])
        q, k, v = _ev(ex["q"]), _ev(ex["k"]), _ev(ex["v"])
        out, lse = o.fwd(q, k, v, rowptr, colidx, ex["scale"])
        assert np.allclose(out, _ev(ex["out"]), rtol=0, atol=1e-14), ex["name"]
        assert np.allclose(lse, _ev(ex["lse"]), rtol=0, atol=1e-14), ex["name"]


def pin_fwd_structured_rows_golden(o):
    """The second worked example's lists are the window-2 + distance-4 graph."""
    ex = _load("worked_attention.json")["examples"][1]
    rowptr, colidx = o.structured(5, 2, (2,))
    er, ec = _csr(ex["rows"])
    assert np.array_equal(rowptr, er) and np.array_equal(colidx, ec)


def pin_fwd_full_causal(o):
    """With W >= T and no links the method is full causal attention
    ('MiniGPT (Part 6)', section 'A mask is not enough', the check after the
    chunked_swa listing); torch's SDPA in float64 is the library routine."""
    for T, D, W, seed in [(1, 4, 1, 0), (37, 8, 37, 1), (128, 16, 200, 2)]:
        q, k, v = (_rand((T, D), seed + 10 * n) for n in range(3))
        scale = 1.0 / math.sqrt(D)
        rowptr, colidx = o.structured(T, W, ())
        out, lse = o.fwd(q, k, v, rowptr, colidx, scale)
        tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                               scale=scale)[0, 0].numpy()
        s = scale * (q @ k.T)
        s[np.triu_indices(T, 1)] = -np.inf
        ref_lse = torch.logsumexp(torch.from_numpy(s), dim=1).numpy()
        assert np.allclose(out, ref, rtol=0, atol=1e-12)
        assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def _random_csr(T, seed, max_extra=6):
    rng = np.random.default_rng(seed)
    rows = []
    for i in range(T):
        r = set(int(x) for x in rng.integers(0, i + 1, size=int(rng.integers(1, max_extra))))
        rows.append(sorted(r))
    return _csr(rows)


def pin_fwd_dense(o):
    """Neighbour-list oracle == dense masked softmax ('MiniGPT (Part 6)': 'with
    a real window it matches the masked version')."""
    cases = [("s", 64, 16, 4, range(0, 6)), ("s", 100, 8, 7, (0, 2, 5)), ("s", 33, 33, 1, ()),
             ("c", 90, 8, 0, ()), ("c", 17, 4, 0, ())]
    for n, (kind, T, D, W, exps) in enumerate(cases):
        if kind == "s":
            rowptr, colidx = o.structured(T, W, exps)
            mask = dense.structured_mask(T, W, exps)
        else:
            rowptr, colidx = _random_csr(T, 100 + n)
            mask = dense.mask_from_csr(T, rowptr, colidx)
        q, k, v = (_rand((T, D), 40 + 3 * n + m) for m in range(3))
        scale = 0.37
        out, lse = o.fwd(q, k, v, rowptr, colidx, scale)
        rout, rlse = dense.attention(q, k, v, mask, scale)
        assert np.allclose(out, rout, rtol=0, atol=1e-12), (kind, T)
        assert np.allclose(lse, rlse, rtol=0, atol=1e-12), (kind, T)


def pin_fwd_invariants(o):
    T, D, W, exps = 150, 8, 5, range(0, 8)
    rowptr, colidx = o.structured(T, W, exps)
    q, k, v = (_rand((T, D), 60 + m) for m in range(3))
    scale = 0.5
    out, lse = o.fwd(q, k, v, rowptr, colidx, scale)
    # constant values: every row of P sums to one, so out = c
    c = np.linspace(-2.0, 3.0, D)
    outc, _ = o.fwd(q, k, np.tile(c, (T, 1)), rowptr, colidx, scale)
    assert np.allclose(outc, np.tile(c, (T, 1)), rtol=0, atol=1e-13)
    # row 0 has only itself
    assert np.allclose(out[0], v[0], rtol=0, atol=1e-15)
    assert abs(lse[0] - scale * float(q[0] @ k[0])) < 1e-13
    # shifting every key by u: out unchanged, lse shifted by scale * q_i . u
    u = _rand((D,), 99)
    out2, lse2 = o.fwd(q, k + u, v, rowptr, colidx, scale)
    assert np.allclose(out2, out, rtol=0, atol=1e-12)
    assert np.allclose(lse2, lse + scale * (q @ u), rtol=0, atol=1e-12)
    # lse from its own definition on a few rows
    for i in (1, 17, 149):
        nb = colidx[rowptr[i]:rowptr[i + 1]]
        s = scale * (k[nb] @ q[i])
        assert abs(lse[i] - math.log(float(np.sum(np.exp(s))))) < 1e-12
    # causality: nothing at a position > i changes row i (bitwise)
    i0 = 70
    q3, k3, v3 = q.copy(), k.copy(), v.copy()
    q3[i0 + 1:] += 5.0
    k3[i0 + 1:] -= 3.0
    v3[i0 + 1:] *= -7.0
    out3, lse3 = o.fwd(q3, k3, v3, rowptr, colidx, scale)
    assert np.array_equal(out3[: i0 + 1], out[: i0 + 1])
    assert np.array_equal(lse3[: i0 + 1], lse[: i0 + 1])
    assert not np.array_equal(out3[i0 + 1:], out[i0 + 1:])


def pin_fwd_empty_rows(o):
    rowptr, colidx = _csr([[0], [], [0, 2], []])
    q, k, v = (_rand((4, 3), 70 + m) for m in range(3))
    out, lse = o.fwd(q, k, v, rowptr, colidx, 1.0)
    assert np.all(out[1] == 0) and np.all(out[3] == 0)
    assert lse[1] == -np.inf and lse[3] == -np.inf
    dq, dk, dv = o.bwd(q, k, v, _rand((4, 3), 80), rowptr, colidx, 1.0)
    assert np.all(dq[1] == 0) and np.all(dq[3] == 0)
    assert np.all(dk[1] == 0) and np.all(dv[1] == 0) and np.all(dk[3] == 0)


# -------------------------------------------------------------- backward

def pin_bwd_golden(o):
    ex = _load("worked_attention.json")["examples"][0]
    rowptr, colidx = _csr(ex["rows"])
    q, k, v, dout = (_ev(ex[n]) for n in ("q", "k", "v", "dout"))
    dq, dk, dv = o.bwd(q, k, v, dout, rowptr, colidx, ex["scale"])
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        assert np.allclose(got, _ev(ex[name]), rtol=0, atol=1e-14), name


def _loss(o, q, k, v, dout, rowptr, colidx, scale):
    out, _ = o.fwd(q, k, v, rowptr, colidx, scale)
    return float(np.sum(out * dout))


def pin_bwd_finite_differences(o):
    """Central differences of L = sum(dout * out), h = 1e-6, relative error
    below 1e-6, along random directions and on single coordinates."""
    T, D, W, exps = 256, 32, 8, range(0, 8)         # the tiny workload's graph
    rowptr, colidx = o.structured(T, W, exps)
    q, k, v, dout = (_rand((T, D), 200 + m) for m in range(4))
    scale = 1.0 / math.sqrt(D)
    dq, dk, dv = o.bwd(q, k, v, dout, rowptr, colidx, scale)
    h = 1e-6
    rng = np.random.default_rng(5)
    for which in range(4):
        uq, uk, uv = (rng.standard_normal((T, D)) * (which in (m, 3)) for m in range(3))
        lp = _loss(o, q + h * uq, k + h * uk, v + h * uv, dout, rowptr, colidx, scale)
        lm = _loss(o, q - h * uq, k - h * uk, v - h * uv, dout, rowptr, colidx, scale)
        fd = (lp - lm) / (2 * h)
        an = float(np.sum(dq * uq) + np.sum(dk * uk) + np.sum(dv * uv))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, fd, an)
    for name, g in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(6):
            i, d = int(rng.integers(0, T)), int(rng.integers(0, D))
            xs = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            xs[name][i, d] += h
            lp = _loss(o, xs["q"], xs["k"], xs["v"], dout, rowptr, colidx, scale)
            xs[name][i, d] -= 2 * h
            lm = _loss(o, xs["q"], xs["k"], xs["v"], dout, rowptr, colidx, scale)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[i, d]) <= 1e-6 * max(1.0, abs(g[i, d])), (name, i, d)


def pin_bwd_dense_autograd(o):
    """Gradients equal torch autograd through the dense masked formulation."""
    for n, (T, D, W, exps) in enumerate([(96, 8, 6, range(0, 7)), (40, 4, 40, ())]):
        rowptr, colidx = o.structured(T, W, exps)
        mask = torch.from_numpy(dense.structured_mask(T, W, exps))
        q, k, v, dout = (_rand((T, D), 300 + 4 * n + m) for m in range(4))
        scale = 0.29
        dq, dk, dv = o.bwd(q, k, v, dout, rowptr, colidx, scale)
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        s = (scale * tq @ tk.T).masked_fill(~mask, float("-inf"))
        out = torch.softmax(s, dim=1) @ tv
        out.backward(torch.from_numpy(dout))
        assert np.allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-12)


def pin_bwd_invariants(o):
    T, D, W, exps = 180, 8, 4, range(0, 8)
    rowptr, colidx = o.structured(T, W, exps)
    q, k, v, dout = (_rand((T, D), 400 + m) for m in range(4))
    dq, dk, dv = o.bwd(q, k, v, dout, rowptr, colidx, 0.7)
    # sum_j dV_j = sum_i dO_i, since every row of P sums to one
    assert np.allclose(dv.sum(axis=0), dout.sum(axis=0), rtol=0, atol=1e-11)
    # sum_j dK_j = 0, since every row of dS sums to zero
    assert np.allclose(dk.sum(axis=0), 0.0, rtol=0, atol=1e-11)
    # all keys equal: scores are constant along each row, dQ = 0
    kc = np.tile(k[3], (T, 1))
    dq2, _, _ = o.bwd(q, kc, v, dout, rowptr, colidx, 0.7)
    assert np.allclose(dq2, 0.0, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- learned
# coordinates: s_ij = -scale |a_i - c_j|^2 ("SpatialLM-Mini ...", section
# "How tokens choose whom to listen to": the closer the coordinates, the
# larger the weight)

def pin_dist_dense(o):
    """Equals the dense numpy statement on structured and random CSR graphs."""
    for n, (T, D) in enumerate([(120, 8), (64, 16)]):
        a, c = _rand((T, 3), 500 + n), _rand((T, 3), 510 + n)
        v = _rand((T, D), 520 + n)
        for rowptr, colidx in (o.structured(T, 5, range(0, 7)), _random_csr(T, 530 + n)):
            out, lse = o.dist_fwd(a, c, v, rowptr, colidx, 0.8)
            mask = dense.mask_from_csr(T, rowptr, colidx)
            r_out, r_lse = dense.dist_attention(a, c, v, mask, 0.8)
            assert np.allclose(out, r_out, rtol=0, atol=1e-12)
            fin = np.isfinite(r_lse)
            assert np.array_equal(np.isfinite(lse), fin)
            assert np.allclose(lse[fin], r_lse[fin], rtol=0, atol=1e-12)


def pin_dist_dot_product_identity(o):
    """-|a - c|^2 = 2 a.c - |c|^2 - |a|^2 and the last term is the same for
    every key of a row: with q' = (2a, -1) and k' = (c, |c|^2) the dot-product
    oracle (pinned on its own) gives the same out, an lse larger by
    scale |a|^2, and gradients related by the chain rule:
    da = 2 dq'[:3], dc = dk'[:3] + 2 c dk'[3]."""
    T, D, W, exps, scale = 150, 8, 6, range(0, 8), 0.45
    rowptr, colidx = o.structured(T, W, exps)
    a, c = _rand((T, 3), 540), _rand((T, 3), 541)
    v, dout = _rand((T, D), 542), _rand((T, D), 543)
    q2 = np.concatenate([2.0 * a, -np.ones((T, 1))], axis=1)
    k2 = np.concatenate([c, (c * c).sum(axis=1, keepdims=True)], axis=1)
    out, lse = o.dist_fwd(a, c, v, rowptr, colidx, scale)
    # the dot-product oracle's q, k, v share D: pad q' and k' with zeros
    pad = np.zeros((T, D - 4))
    qp, kp = np.concatenate([q2, pad], axis=1), np.concatenate([k2, pad], axis=1)
    r_out, r_lse = o.fwd(qp, kp, v, rowptr, colidx, scale)
    assert np.allclose(out, r_out, rtol=0, atol=1e-12)
    assert np.allclose(lse, r_lse - scale * (a * a).sum(axis=1), rtol=0, atol=1e-11)
    da, dc, dv = o.dist_bwd(a, c, v, dout, rowptr, colidx, scale)
    dqp, dkp, r_dv = o.bwd(qp, kp, v, dout, rowptr, colidx, scale)
    assert np.allclose(dv, r_dv, rtol=0, atol=1e-12)
    assert np.allclose(da, 2.0 * dqp[:, :3], rtol=0, atol=1e-11)
    assert np.allclose(dc, dkp[:, :3] + 2.0 * c * dkp[:, 3:4], rtol=0, atol=1e-11)


def pin_dist_invariants(o):
    """Moving every coordinate by the same vector changes nothing (distances
    are unchanged); row 0 sees only itself; constant V gives that constant;
    the closest key dominates when the scale is large."""
    T, D, W, exps = 100, 8, 4, range(0, 7)
    rowptr, colidx = o.structured(T, W, exps)
    a, c, v = _rand((T, 3), 550), _rand((T, 3), 551), _rand((T, D), 552)
    dout = _rand((T, D), 553)
    out, lse = o.dist_fwd(a, c, v, rowptr, colidx, 0.6)
    u = np.array([0.75, -2.5, 1.25])
    out2, lse2 = o.dist_fwd(a + u, c + u, v, rowptr, colidx, 0.6)
    assert np.allclose(out, out2, rtol=0, atol=1e-12)
    assert np.allclose(lse, lse2, rtol=0, atol=1e-12)
    g1 = o.dist_bwd(a, c, v, dout, rowptr, colidx, 0.6)
    g2 = o.dist_bwd(a + u, c + u, v, dout, rowptr, colidx, 0.6)
    for x, y in zip(g1, g2):
        assert np.allclose(x, y, rtol=0, atol=1e-11)
    assert np.allclose(out[0], v[0], rtol=0, atol=1e-15)
    assert abs(lse[0] + 0.6 * float(((a[0] - c[0]) ** 2).sum())) <= 1e-14
    cv = np.tile(np.arange(1.0, D + 1.0), (T, 1))
    out_c, _ = o.dist_fwd(a, c, cv, rowptr, colidx, 0.6)
    assert np.allclose(out_c, cv, rtol=0, atol=1e-12)
    # every query placed on its own key, other keys far: out_i -> v_i
    a3 = np.arange(T, dtype=np.float64)[:, None] * np.array([[10.0, 0.0, 0.0]])
    out_s, _ = o.dist_fwd(a3, a3.copy(), v, rowptr, colidx, 1.0)
    assert np.allclose(out_s, v, rtol=0, atol=1e-12)
    # sum_j dv_j = sum_i dO_i (rows of P sum to one); sum of da + dc is zero
    # (translation invariance of the loss)
    da, dc, dv = g1
    assert np.allclose(dv.sum(axis=0), dout.sum(axis=0), rtol=0, atol=1e-11)
    assert np.allclose(da.sum(axis=0) + dc.sum(axis=0), 0.0, rtol=0, atol=1e-11)


def _dist_loss(o, a, c, v, dout, rowptr, colidx, scale):
    out, _ = o.dist_fwd(a, c, v, rowptr, colidx, scale)
    return float(np.sum(out * dout))


def pin_dist_finite_differences(o):
    """Central differences of L = sum(dout * out) along random directions of
    a, c and v together and separately (h = 1e-6, relative error < 1e-6),
    and torch autograd through the dense formulation."""
    T, D, W, exps, scale = 130, 8, 6, range(0, 8), 0.35
    rowptr, colidx = o.structured(T, W, exps)
    a, c = _rand((T, 3), 560), _rand((T, 3), 561)
    v, dout = _rand((T, D), 562), _rand((T, D), 563)
    da, dc, dv = o.dist_bwd(a, c, v, dout, rowptr, colidx, scale)
    h = 1e-6
    rng = np.random.default_rng(6)
    for which in range(4):
        ua = rng.standard_normal((T, 3)) * (which in (0, 3))
        uc = rng.standard_normal((T, 3)) * (which in (1, 3))
        uv = rng.standard_normal((T, D)) * (which in (2, 3))
        lp = _dist_loss(o, a + h * ua, c + h * uc, v + h * uv, dout, rowptr, colidx, scale)
        lm = _dist_loss(o, a - h * ua, c - h * uc, v - h * uv, dout, rowptr, colidx, scale)
        fd = (lp - lm) / (2 * h)
        an = float(np.sum(da * ua) + np.sum(dc * uc) + np.sum(dv * uv))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, fd, an)
    mask = torch.from_numpy(dense.structured_mask(T, W, exps))
    ta, tc, tv = (torch.tensor(x, requires_grad=True) for x in (a, c, v))
    s = (-scale * ((ta[:, None, :] - tc[None, :, :]) ** 2).sum(-1)).masked_fill(~mask,
                                                                                float("-inf"))
    (torch.softmax(s, dim=1) @ tv).backward(torch.from_numpy(dout))
    assert np.allclose(da, ta.grad.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(dc, tc.grad.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-12)


ALL_PINS = [pin_graph_golden, pin_graph_bruteforce, pin_graph_closed_forms,
            pin_graph_rows_match_full, pin_graph_reverse,
            pin_graph_normalize, pin_fwd_golden, pin_fwd_structured_rows_golden,
            pin_fwd_full_causal, pin_fwd_dense, pin_fwd_invariants, pin_fwd_empty_rows,
            pin_bwd_golden, pin_bwd_finite_differences, pin_bwd_dense_autograd,
            pin_bwd_invariants, pin_dist_dense, pin_dist_dot_product_identity,
            pin_dist_invariants, pin_dist_finite_differences]
