"""sparse_graph_causal_b200 -- Python binding of libsparse_attn.so.

Causal attention restricted to a fixed sparse neighbour graph on NVIDIA B200
(sm_100a).  Every computation runs in the library's CUDA kernels; this module
only marshals torch tensors (device memory) and the current CUDA stream into
the C ABI declared in include/sparse_attn.h, under the same names.  There is
no CPU fallback: the library is loaded on first use and every call raises
when it is not built or when it reports an error.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparse_attn.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_INVALID_GRAPH, SA_ERR_UNSUPPORTED = 0, 1, 2, 3
SA_ERR_OOM, SA_ERR_CUDA, SA_ERR_DEVICE_TIMEOUT = 4, 5, 6
SA_BF16, SA_FP32 = 0, 1
SA_PATH_AUTO, SA_PATH_GATHER = 0, 1
SA_LINKS_AUTO, SA_LINKS_SPLIT, SA_LINKS_ONE_PASS = 0, 1, 2

class SaTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("B", ctypes.c_int64),
                ("H", ctypes.c_int64), ("T", ctypes.c_int64), ("D", ctypes.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run `python -m sparse_graph_causal_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    i64, i32, vp, st = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int
    P = ctypes.POINTER
    sig = {
        "sparse_attn_graph_build_structured": (st, [i64, i32, vp, i32, i32, vp, P(vp)]),
        "sparse_attn_graph_build_csr": (st, [i64, vp, vp, i64, i32, vp, P(vp)]),
        "sparse_attn_graph_nnz": (st, [vp, P(i64), P(i64)]),
        "sparse_attn_graph_export": (st, [vp, vp, vp, vp, vp, vp]),
        "sparse_attn_graph_destroy": (st, [vp]),
        "sparse_attn_fwd": (st, [P(SaTensor), P(SaTensor), P(SaTensor), vp, ctypes.c_float,
                                 P(SaTensor), vp, vp]),
        "sparse_attn_bwd_workspace_size": (ctypes.c_size_t, [P(SaTensor), vp]),
        "sparse_attn_bwd": (st, [P(SaTensor), P(SaTensor), P(SaTensor), P(SaTensor), vp,
                                 P(SaTensor), vp, ctypes.c_float, P(SaTensor), P(SaTensor),
                                 P(SaTensor), vp, ctypes.c_size_t, vp]),
        "sparse_attn_status_string": (ctypes.c_char_p, [st]),
        "sparse_attn_set_path": (st, [i32]),
        "sparse_attn_set_link_pass": (st, [i32]),
        "sparse_attn_check_device": (st, [vp]),
        "sparse_attn_selftest_wait_timeout": (st, [i64, vp]),
        "sparse_attn_launch_count": (i64, []),
        "sparse_attn_last_error_message": (ctypes.c_char_p, []),
        "sparse_attn_bwd_noalloc": (st, [P(SaTensor), P(SaTensor), P(SaTensor), P(SaTensor), vp,
                                         P(SaTensor), vp, ctypes.c_float, P(SaTensor),
                                         P(SaTensor), P(SaTensor), vp]),
        "sparse_attn_decode": (st, [P(SaTensor), P(SaTensor), P(SaTensor), vp, vp,
                                    ctypes.c_float, P(SaTensor), vp, vp]),
        "sparse_attn_dist_fwd": (st, [P(SaTensor), P(SaTensor), P(SaTensor), vp,
                                      ctypes.c_float, P(SaTensor), vp, vp]),
        "sparse_attn_dist_bwd_workspace_size": (ctypes.c_size_t, [P(SaTensor), vp]),
        "sparse_attn_dist_bwd": (st, [P(SaTensor), P(SaTensor), P(SaTensor), P(SaTensor), vp,
                                      P(SaTensor), vp, ctypes.c_float, P(SaTensor),
                                      P(SaTensor), P(SaTensor), vp, ctypes.c_size_t, vp]),
        "sparse_attn_profile_begin": (st, [i32]),
        "sparse_attn_profile_end": (i32, [ctypes.c_char_p, i32, P(i32), P(ctypes.c_double), i32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


class _LazyLib:
    """The loaded library, opened on first attribute access."""

    def __init__(self):
        self._lib = None

    def __getattr__(self, name):
        if self._lib is None:
            self._lib = _load()
        return getattr(self._lib, name)


_lib = _LazyLib()


class SparseAttentionError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == SA_ERR_CUDA:
            detail = " [" + sparse_attn_last_error_message() + "]"
        super().__init__(f"{where}: {sparse_attn_status_string(status)} (status {status}){detail}")


def _check(status: int, where: str):
    if status != SA_OK:
        raise SparseAttentionError(status, where)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _tensor(t: torch.Tensor, name: str) -> SaTensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, H, T, D] tensor")
    if t.dtype == torch.bfloat16:
        dt = SA_BF16
    elif t.dtype == torch.float32:
        dt = SA_FP32
    else:
        raise ValueError(f"{name}: dtype {t.dtype} is not bf16 or fp32")
    B, H, T, D = t.shape
    return SaTensor(t.data_ptr(), dt, B, H, T, D)


# ------------------------------------------------------------------ graphs

class Graph:
    """Owner of an ``sa_graph`` handle (freed by :meth:`close` or on GC)."""

    def __init__(self, handle: int, T: int, kind: str, W: int = 0, exps=()):
        self.handle = ctypes.c_void_p(handle)
        self.T, self.kind, self.W, self.exps = T, kind, W, tuple(exps)

    @property
    def nnz(self) -> int:
        return sparse_attn_graph_nnz(self)[0]

    def close(self):
        if self.handle:
            sparse_attn_graph_destroy(self)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def sparse_attn_graph_build_structured(T: int, W: int, dil_exps=(), materialize: bool = False,
                                       stream=None) -> Graph:
    exps = (ctypes.c_int32 * max(len(dil_exps), 1))(*[int(e) for e in dil_exps])
    h = ctypes.c_void_p()
    _check(_lib.sparse_attn_graph_build_structured(int(T), int(W), exps, len(dil_exps),
                                                   int(bool(materialize)), _stream(stream),
                                                   ctypes.byref(h)),
           "sparse_attn_graph_build_structured")
    return Graph(h.value, T, "structured", W, dil_exps)


def sparse_attn_graph_build_csr(rowptr: torch.Tensor, colidx: torch.Tensor, band_hint: int = 0,
                                stream=None) -> Graph:
    """rowptr: CUDA int64 [T+1]; colidx: CUDA int32 [nnz] (rows may be
    unsorted and contain repeats)."""
    if rowptr.dtype != torch.int64 or colidx.dtype != torch.int32:
        raise ValueError("rowptr must be int64 and colidx int32")
    if not (rowptr.is_cuda and colidx.is_cuda and rowptr.is_contiguous()
            and colidx.is_contiguous()):
        raise ValueError("rowptr and colidx must be contiguous CUDA tensors")
    T = rowptr.numel() - 1
    h = ctypes.c_void_p()
    _check(_lib.sparse_attn_graph_build_csr(T, rowptr.data_ptr(),
                                            colidx.data_ptr() if colidx.numel() else None,
                                            colidx.numel(), int(band_hint), _stream(stream),
                                            ctypes.byref(h)),
           "sparse_attn_graph_build_csr")
    return Graph(h.value, T, "csr", band_hint)


def sparse_attn_graph_nnz(g: Graph):
    a, b = ctypes.c_int64(), ctypes.c_int64()
    _check(_lib.sparse_attn_graph_nnz(g.handle, ctypes.byref(a), ctypes.byref(b)),
           "sparse_attn_graph_nnz")
    return a.value, b.value


def sparse_attn_graph_export(g: Graph, stream=None, device=None):
    """Returns (rowptr int64[T+1], colidx int32[nnz], rev_rowptr, rev_colidx)
    as new CUDA tensors."""
    nnz, _ = sparse_attn_graph_nnz(g)
    dev = device or torch.device("cuda", torch.cuda.current_device())
    rp = torch.empty(g.T + 1, dtype=torch.int64, device=dev)
    ci = torch.empty(nnz, dtype=torch.int32, device=dev)
    rrp = torch.empty(g.T + 1, dtype=torch.int64, device=dev)
    rci = torch.empty(nnz, dtype=torch.int32, device=dev)
    _check(_lib.sparse_attn_graph_export(g.handle, rp.data_ptr(), ci.data_ptr() if nnz else None,
                                         rrp.data_ptr(), rci.data_ptr() if nnz else None,
                                         _stream(stream)),
           "sparse_attn_graph_export")
    return rp, ci, rrp, rci


def sparse_attn_graph_destroy(g: Graph):
    h, g.handle = g.handle, ctypes.c_void_p()
    if h:
        _check(_lib.sparse_attn_graph_destroy(h), "sparse_attn_graph_destroy")


# --------------------------------------------------------------- attention

def sparse_attn_fwd(q, k, v, g: Graph, scale: float, out=None, lse=None, stream=None):
    """Returns (out [B,H,T,D] in q's dtype, lse fp32 [B,H,T])."""
    B, H, T, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or lse.shape != (B, H, T):
        raise ValueError("lse must be a contiguous fp32 [B, H, T] tensor")
    tq, tk, tv, to = (_tensor(x, n) for x, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")))
    _check(_lib.sparse_attn_fwd(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), g.handle,
                                float(scale), ctypes.byref(to), lse.data_ptr(), _stream(stream)),
           "sparse_attn_fwd")
    return out, lse


def sparse_attn_bwd_workspace_size(q, g: Graph) -> int:
    tq = _tensor(q, "q")
    return int(_lib.sparse_attn_bwd_workspace_size(ctypes.byref(tq), g.handle))


def sparse_attn_bwd(q, k, v, out, lse, dout, g: Graph, scale: float, dq=None, dk=None, dv=None,
                    workspace=None, stream=None):
    """Returns (dq, dk, dv)."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws_bytes = sparse_attn_bwd_workspace_size(q, g)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32")
    ts = [_tensor(x, n) for x, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout"),
                                     (dq, "dq"), (dk, "dk"), (dv, "dv"))]
    r = [ctypes.byref(t) for t in ts]
    _check(_lib.sparse_attn_bwd(r[0], r[1], r[2], r[3], lse.data_ptr(), r[4], g.handle,
                                float(scale), r[5], r[6], r[7], workspace.data_ptr(),
                                workspace.numel() * workspace.element_size(), _stream(stream)),
           "sparse_attn_bwd")
    return dq, dk, dv


def sparse_attn_bwd_noalloc(q, k, v, out, lse, dout, g: Graph, scale: float, dq=None, dk=None,
                            dv=None, stream=None):
    """sparse_attn_bwd without a workspace: for callers that cannot allocate
    device memory when they call it.  The library keeps its scratch in a
    fixed device array (B*H*T <= SA_NOALLOC_MAX_ROWS); calls that overlap on
    the GPU race on it.  Output tensors passed in are written, not
    allocated; the defaults below allocate them here, in Python, for
    convenience."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32")
    ts = [_tensor(x, n) for x, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout"),
                                     (dq, "dq"), (dk, "dk"), (dv, "dv"))]
    r = [ctypes.byref(t) for t in ts]
    _check(_lib.sparse_attn_bwd_noalloc(r[0], r[1], r[2], r[3], lse.data_ptr(), r[4], g.handle,
                                        float(scale), r[5], r[6], r[7], _stream(stream)),
           "sparse_attn_bwd_noalloc")
    return dq, dk, dv


SA_NOALLOC_MAX_ROWS = 1 << 20


# ------------------------------------------------------------------ decode

def sparse_attn_decode(q, k_cache, v_cache, pos, g: Graph, scale: float, out=None, lse=None,
                       stream=None):
    """q [B, H, 1, D]; caches [B, Hkv, Tmax, D]; pos: CUDA int64 [B] (the
    query's own key/value already at cache row pos[b]).  Returns (out
    [B, H, 1, D], lse fp32 [B, H])."""
    B, H, _, D = q.shape
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or lse.shape != (B, H):
        raise ValueError("lse must be a contiguous fp32 [B, H] tensor")
    if pos.dtype != torch.int64 or not pos.is_cuda or pos.numel() != B:
        raise ValueError("pos must be a CUDA int64 tensor of B positions")
    tq, tk, tv, to = (_tensor(x, n) for x, n in ((q, "q"), (k_cache, "k_cache"),
                                                  (v_cache, "v_cache"), (out, "out")))
    _check(_lib.sparse_attn_decode(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv),
                                   pos.data_ptr(), g.handle, float(scale), ctypes.byref(to),
                                   lse.data_ptr(), _stream(stream)),
           "sparse_attn_decode")
    return out, lse


# ------------------------------------------------ learned-coordinate scoring

def _coords(t: torch.Tensor, name: str) -> SaTensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32:
        raise ValueError(f"{name} must be a CUDA fp32 tensor")
    if t.dim() != 4 or t.shape[3] != 3 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, H, T, 3] tensor")
    B, H, T, _ = t.shape
    return SaTensor(t.data_ptr(), SA_FP32, B, H, T, 3)


def sparse_attn_dist_fwd(a, c, v, g: Graph, scale: float, out=None, lse=None, stream=None):
    """s_ij = -scale |a_i - c_j|^2 over the graph's lists; a, c fp32
    [B, H, T, 3].  Returns (out [B, H, T, D] in v's dtype, lse fp32 [B, H, T])."""
    B, H, T, D = v.shape
    out = torch.empty_like(v) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=v.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or lse.shape != (B, H, T):
        raise ValueError("lse must be a contiguous fp32 [B, H, T] tensor")
    ta, tc = _coords(a, "a"), _coords(c, "c")
    tv, to = _tensor(v, "v"), _tensor(out, "out")
    _check(_lib.sparse_attn_dist_fwd(ctypes.byref(ta), ctypes.byref(tc), ctypes.byref(tv),
                                     g.handle, float(scale), ctypes.byref(to), lse.data_ptr(),
                                     _stream(stream)),
           "sparse_attn_dist_fwd")
    return out, lse


def sparse_attn_dist_bwd_workspace_size(v, g: Graph) -> int:
    tv = _tensor(v, "v")
    return int(_lib.sparse_attn_dist_bwd_workspace_size(ctypes.byref(tv), g.handle))


def sparse_attn_dist_bwd(a, c, v, out, lse, dout, g: Graph, scale: float, da=None, dc=None,
                         dv=None, workspace=None, stream=None):
    """Returns (da, dc, dv)."""
    da = torch.empty_like(a) if da is None else da
    dc = torch.empty_like(c) if dc is None else dc
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(sparse_attn_dist_bwd_workspace_size(v, g), dtype=torch.uint8,
                                device=v.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32")
    ta, tc, tda, tdc = _coords(a, "a"), _coords(c, "c"), _coords(da, "da"), _coords(dc, "dc")
    tv, to, tdo, tdv = (_tensor(x, n) for x, n in ((v, "v"), (out, "out"), (dout, "dout"),
                                                    (dv, "dv")))
    _check(_lib.sparse_attn_dist_bwd(ctypes.byref(ta), ctypes.byref(tc), ctypes.byref(tv),
                                     ctypes.byref(to), lse.data_ptr(), ctypes.byref(tdo),
                                     g.handle, float(scale), ctypes.byref(tda), ctypes.byref(tdc),
                                     ctypes.byref(tdv), workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(),
                                     _stream(stream)),
           "sparse_attn_dist_bwd")
    return da, dc, dv


# ---------------------------------------------------------------- utilities

def sparse_attn_status_string(status: int) -> str:
    return _lib.sparse_attn_status_string(int(status)).decode()


def sparse_attn_set_path(path: int):
    _check(_lib.sparse_attn_set_path(int(path)), "sparse_attn_set_path")


def sparse_attn_set_link_pass(mode: int):
    _check(_lib.sparse_attn_set_link_pass(int(mode)), "sparse_attn_set_link_pass")


def sparse_attn_check_device(stream=None):
    _check(_lib.sparse_attn_check_device(_stream(stream)), "sparse_attn_check_device")


def sparse_attn_selftest_wait_timeout(limit_ns: int = 20_000_000, stream=None):
    """Enqueue a wait that nothing completes and that gives up after
    limit_ns; the next sparse_attn_check_device raises with status
    SA_ERR_DEVICE_TIMEOUT."""
    _check(_lib.sparse_attn_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "sparse_attn_selftest_wait_timeout")


def sparse_attn_last_error_message() -> str:
    return (_lib.sparse_attn_last_error_message() or b"").decode()


def sparse_attn_launch_count() -> int:
    return int(_lib.sparse_attn_launch_count())


def sparse_attn_profile_begin(enable: bool = True):
    _check(_lib.sparse_attn_profile_begin(int(bool(enable))), "sparse_attn_profile_begin")


def sparse_attn_profile_end(max_kernels: int = 64):
    """Returns {kernel name: (launches, total event-timed ms)} since
    sparse_attn_profile_begin()."""
    name_len = 64
    names = ctypes.create_string_buffer(name_len * max_kernels)
    counts = (ctypes.c_int32 * max_kernels)()
    ms = (ctypes.c_double * max_kernels)()
    n = _lib.sparse_attn_profile_end(names, name_len, counts, ms, max_kernels)
    if n < 0:
        raise SparseAttentionError(SA_ERR_CUDA, "sparse_attn_profile_end")
    out = {}
    for k in range(n):
        nm = names.raw[k * name_len:(k + 1) * name_len].split(b"\0", 1)[0].decode()
        out[nm] = (int(counts[k]), float(ms[k]))
    return out


class _SparseAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, graph, scale):
        out, lse = sparse_attn_fwd(q, k, v, graph, scale)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.graph, ctx.scale = graph, scale
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = sparse_attn_bwd(q, k, v, out, lse, dout.contiguous(), ctx.graph, ctx.scale)
        return dq, dk, dv, None, None


class _DistAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, a, c, v, graph, scale):
        out, lse = sparse_attn_dist_fwd(a, c, v, graph, scale)
        ctx.save_for_backward(a, c, v, out, lse)
        ctx.graph, ctx.scale = graph, scale
        return out

    @staticmethod
    def backward(ctx, dout):
        a, c, v, out, lse = ctx.saved_tensors
        da, dc, dv = sparse_attn_dist_bwd(a, c, v, out, lse, dout.contiguous(), ctx.graph,
                                          ctx.scale)
        return da, dc, dv, None, None


def dist_attention(a, c, v, graph: Graph, scale: float):
    """Differentiable learned-coordinate attention on the graph:
    softmax over N(i) of -scale |a_i - c_j|^2, applied to v."""
    return _DistAttention.apply(a, c, v, graph, scale)


def attention(q, k, v, graph: Graph, scale: float):
    """Differentiable sparse-graph causal attention (forward and backward in
    the library's kernels)."""
    return _SparseAttention.apply(q, k, v, graph, scale)


__all__ = [n for n in dir() if n.startswith("sparse_attn_")] + [
    "Graph", "attention", "dist_attention", "SparseAttentionError", "LIB_PATH"]
