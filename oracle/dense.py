"""TEST INFRASTRUCTURE ONLY: a dense fp64 statement of the same attention,
for tiny T.  Independent of ``oracle.c``: it never forms neighbour lists.

The mask follows "MiniGPT (Part 6)", section "A mask is not enough": key j is
kept for query i when j <= i and i - j < w.  The distance links follow
"SpatialLM-Mini ...", section "How tokens choose whom to listen to": query i
also sees position i - 2^k when that position exists.  Scores are
scale * (q . k) before the softmax, as in the chunked_swa listing of the same
MiniGPT section.
"""
from __future__ import annotations

import numpy as np


def structured_mask(T: int, W: int, exps) -> np.ndarray:
    """Boolean [T, T] mask: window of W keys including self, plus i - 2^k."""
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    keep = (j <= i) & (i - j < W)
    for k in set(int(e) for e in exps):
        keep |= (i - j) == (1 << k)
    return keep


def mask_from_csr(T: int, rowptr, colidx) -> np.ndarray:
    m = np.zeros((T, T), dtype=bool)
    for i in range(T):
        m[i, colidx[rowptr[i]:rowptr[i + 1]]] = True
    return m


def attention(q, k, v, mask, scale):
    """q, k, v: [T, D] float64; mask [T, T] bool.  Returns out [T, D], lse [T].
    Rows with no kept key give out = 0 and lse = -inf."""
    s = scale * (q @ k.T)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    empty = ~mask.any(axis=1)
    m = np.where(empty[:, None], 0.0, m)
    e = np.where(mask, np.exp(s - m), 0.0)
    l = e.sum(axis=1, keepdims=True)
    p = np.divide(e, l, out=np.zeros_like(e), where=l > 0)
    out = p @ v
    with np.errstate(divide="ignore"):
        lse = (m + np.log(l))[:, 0]
    lse = np.where(empty, -np.inf, lse)
    return out, lse


def dist_attention(a, c, v, mask, scale):
    """Learned-coordinate scoring, dense: s_ij = -scale * |a_i - c_j|^2 for
    kept (i, j) ("SpatialLM-Mini ...", section "How tokens choose whom to
    listen to": the closer the query and key coordinates, the larger the
    weight).  a, c: [T, 3]; v: [T, D]; mask [T, T] bool."""
    diff = a[:, None, :] - c[None, :, :]
    s = -scale * np.einsum("ijx,ijx->ij", diff, diff)
    s = np.where(mask, s, -np.inf)
    empty = ~mask.any(axis=1)
    m = np.where(empty[:, None], 0.0, s.max(axis=1, keepdims=True))
    e = np.where(mask, np.exp(s - m), 0.0)
    l = e.sum(axis=1, keepdims=True)
    p = np.divide(e, l, out=np.zeros_like(e), where=l > 0)
    with np.errstate(divide="ignore"):
        lse = (m + np.log(l))[:, 0]
    return p @ v, np.where(empty, -np.inf, lse)
