"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds workload shapes and random-number draws only; it contains
none of the attention arithmetic and none of the graph construction that the
library or the oracle performs (the CSR generator below emits *raw*,
unsorted neighbour lists with repeats; normalising them is the method's job).

Workloads (shapes from the pages' own experiments, values synthetic):
  tiny          B1 H2 T256 D32 fp32, window 8 + 2^k links k=0..7
  tiny_full     the same with window = T = 256 and no links (full causal)
  spatiallm_16k B1 H4 T16384 D64 bf16, window 32 + 2^k links k=0..13,
                inputs N(0,1)/sqrt(D) (the 16,384-token, 4-layer small LM of
                "SpatialLM-Mini ...")
  band_32k      B4 H32 T32768 D128 bf16, window 4096, no links (the
                Mistral-style window of "MiniGPT (Part 6)")
  band_4k_full  B4 H32 T4096 D128 bf16, window = T = 4096 (full causal check)
  band_32k_b1h8 B1 H8 T32768 D128 bf16, window 4096 (profiler-capture size)
  csr_1m        B1 H8 T2^20 D64 bf16, raw CSR rows: window 64 + 16 uniform
                draws from [0, i) + the first 16 tokens (graph view of
                "Longer Attention Span ...")
  csr_256k      B1 H4 T2^18 D64 bf16, the same rows (profiler-capture size of
                csr_1m: K and V still 256 MB, beyond L2)
  extreme_128m  B1 H1 T2^27 D64 bf16, window 32 + 2^k links k=0..26, inputs
                drawn on the device
  extreme_8m    B1 H1 T2^23 D64 bf16, window 32 + 2^k links k=0..22 (profiler-
                capture size of extreme_128m)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    D: int
    dtype: str            # "bf16" | "fp32"
    W: int                # window (keys including self); 0 for a CSR graph
    exps: tuple = ()      # distance links i - 2^k
    csr: bool = False     # neighbour lists drawn by csr_random_rows
    band_hint: int = 0    # window every CSR row is known to contain
    input_std: float = 1.0
    scale: float = 0.0
    seed: int = 0
    graph_seed: int = 0
    bwd: bool = True
    Hkv: int = 0          # key/value heads (grouped-query attention); 0: H
    kind: str = "attn"    # "attn", "dist" (learned coordinates) or "decode"

    @property
    def kv_heads(self) -> int:
        return self.Hkv or self.H

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_size(self) -> int:
        return 2 if self.dtype == "bf16" else 4


def _w(name, B, H, T, D, dtype, W, exps=(), std=1.0, seed=0, **kw):
    return Workload(name=name, B=B, H=H, T=T, D=D, dtype=dtype, W=W, exps=tuple(exps),
                    input_std=std, scale=1.0 / math.sqrt(D), seed=seed, **kw)


WORKLOADS = {
    "tiny": _w("tiny", 1, 2, 256, 32, "fp32", 8, range(0, 8), seed=1001),
    "tiny_full": _w("tiny_full", 1, 2, 256, 32, "fp32", 256, (), seed=1001),
    "spatiallm_16k": _w("spatiallm_16k", 1, 4, 16384, 64, "bf16", 32, range(0, 14),
                        std=1.0 / math.sqrt(64), seed=1002),
    "band_32k": _w("band_32k", 4, 32, 32768, 128, "bf16", 4096, (), seed=1003),
    "band_4k_full": _w("band_4k_full", 4, 32, 4096, 128, "bf16", 4096, (), seed=1003),
    # a quarter of band_32k (one batch row, 8 heads): the size used for
    # detailed profiler captures
    "band_32k_b1h8": _w("band_32k_b1h8", 1, 8, 32768, 128, "bf16", 4096, (), seed=1003),
    "csr_1m": _w("csr_1m", 1, 8, 1 << 20, 64, "bf16", 0, (), seed=1004, csr=True,
                 band_hint=64, graph_seed=2004, bwd=False),
    # a smaller csr_1m (a quarter of the rows, half the heads): the size used
    # for detailed profiler captures
    "csr_256k": _w("csr_256k", 1, 4, 1 << 18, 64, "bf16", 0, (), seed=1004, csr=True,
                   band_hint=64, graph_seed=2004, bwd=False),
    "extreme_128m": _w("extreme_128m", 1, 1, 1 << 27, 64, "bf16", 32, range(0, 27), seed=1005,
                       bwd=False),
    # a 1/16-length version of extreme_128m: the size used for profiler captures
    "extreme_8m": _w("extreme_8m", 1, 1, 1 << 23, 64, "bf16", 32, range(0, 23), seed=1005,
                     bwd=False),
    # the 16K layer with grouped-query attention: 8 query heads over 2 key/value heads
    "gqa_16k": _w("gqa_16k", 1, 8, 16384, 64, "bf16", 32, range(0, 14), std=1.0 / math.sqrt(64),
                  seed=1006, Hkv=2),
    # the 16K layer with learned-coordinate weights (coordinates N(0,1), scale 0.5)
    "dist_16k": Workload(name="dist_16k", B=1, H=4, T=16384, D=64, dtype="bf16", W=32,
                         exps=tuple(range(0, 14)), input_std=1.0, scale=0.5, seed=1007,
                         kind="dist"),
    # decode: one new token per sequence for 64 sequences against 16K caches
    # (8 query heads over 2 cache heads), positions drawn in [T/2, T)
    "decode_16k": _w("decode_16k", 64, 8, 16384, 64, "bf16", 32, range(0, 14), seed=1008,
                     Hkv=2, kind="decode", bwd=False),
}


def make_qkv(w: Workload, device="cpu", seed: int | None = None, with_dout: bool = True,
             std: float | None = None):
    """q, k, v (and dout) of shape [B, H, T, D] (k and v: [B, Hkv, T, D]),
    contiguous, N(0, std^2), drawn
    on ``device`` from a torch.Generator seeded with ``seed`` (default: the
    workload's).  Values are drawn in fp32 and rounded to the workload dtype."""
    seed = w.seed if seed is None else seed
    std = w.input_std if std is None else std
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    names = ["q", "k", "v"] + (["dout"] if with_dout else [])
    out = {}
    for n in names:
        shape = (w.B, w.kv_heads if n in ("k", "v") else w.H, w.T, w.D)
        t = torch.empty(shape, dtype=w.torch_dtype, device=dev)
        if w.torch_dtype == torch.float32:
            t.normal_(0.0, 1.0, generator=g)
            if std != 1.0:
                t.mul_(std)
        else:
            # draw in chunks to bound the fp32 temporary on very long sequences
            flat = t.view(-1)
            chunk = 1 << 28
            for s in range(0, flat.numel(), chunk):
                e = min(flat.numel(), s + chunk)
                tmp = torch.empty(e - s, dtype=torch.float32, device=dev)
                tmp.normal_(0.0, 1.0, generator=g)
                if std != 1.0:
                    tmp.mul_(std)
                flat[s:e].copy_(tmp)
                del tmp
        out[n] = t
    return out


def make_coords(w: Workload, device="cpu", seed: int | None = None, std: float = 1.0):
    """Query and key coordinates a, c of shape [B, H, T, 3], fp32,
    N(0, std^2), drawn on ``device`` from a torch.Generator (seed: the
    workload's + 7)."""
    seed = (w.seed + 7) if seed is None else seed
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    a = torch.empty((w.B, w.H, w.T, 3), dtype=torch.float32, device=dev).normal_(0.0, std,
                                                                                generator=g)
    c = torch.empty((w.B, w.H, w.T, 3), dtype=torch.float32, device=dev).normal_(0.0, std,
                                                                                generator=g)
    return a, c


def csr_random_rows(T: int, seed: int, window: int = 64, n_random: int = 16,
                    n_global: int = 16):
    """Raw neighbour lists, one row per query i, in this order and unsorted:
    n_random independent uniform draws from [0, i) (none for i = 0), the
    global keys 0 .. min(n_global, i + 1) - 1, then the window
    i, i - 1, ..., max(0, i - window + 1).  Repeats are left in.
    Returns (rowptr int64[T+1], colidx int32[nnz])."""
    rng = np.random.default_rng(seed)
    i = np.arange(T, dtype=np.int64)[:, None]
    u = rng.random((T, n_random))
    rand = np.floor(u * i).astype(np.int64)           # in [0, i) for i > 0
    rand_ok = np.broadcast_to(i > 0, rand.shape)
    glob = np.broadcast_to(np.arange(n_global, dtype=np.int64)[None, :], (T, n_global))
    glob_ok = glob <= i
    win = i - np.arange(window, dtype=np.int64)[None, :]
    win_ok = win >= 0
    cols = np.concatenate([rand, glob, win], axis=1)
    ok = np.concatenate([rand_ok, glob_ok, win_ok], axis=1)
    counts = ok.sum(axis=1)
    rowptr = np.zeros(T + 1, dtype=np.int64)
    np.cumsum(counts, out=rowptr[1:])
    colidx = cols[ok].astype(np.int32)
    return rowptr, colidx


def sample_rows(T: int, n: int, seed: int, include_edges: bool = True):
    """n distinct query positions in [0, T), sorted; always includes the first
    and last rows and the start of the sequence where neighbour lists are
    still growing."""
    rng = np.random.default_rng(seed)
    n = min(n, T)
    picks = set(rng.choice(T, size=n, replace=False).tolist())
    if include_edges:
        picks.update(x for x in (0, 1, 2, T - 1, T - 2) if 0 <= x < T)
    return np.array(sorted(picks)[: max(n, 1) + 5], dtype=np.int64)
