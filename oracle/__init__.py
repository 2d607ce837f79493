"""TEST INFRASTRUCTURE ONLY: the CPU oracle for sparse-graph causal attention.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library under
``sparse_graph_causal_b200`` never does, and this package imports nothing
from it.

Two independent statements of the method live here:

* ``oracle.c`` (loaded through ctypes by :class:`Oracle`): plain,
  single-threaded fp64 C that loops over each query's neighbour list.
* :mod:`oracle.dense`: a dense T x T masked softmax in numpy fp64, for tiny
  T only, written from the window-mask rule of "MiniGPT (Part 6)", section
  "A mask is not enough", plus the 2^k distance links of "SpatialLM-Mini ...",
  section "How tokens choose whom to listen to".

The two share no code; the tests pin each against the other and against
closed forms and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

STATUS = {0: "ok", 1: "bad rowptr", 2: "look-ahead edge", 3: "negative key",
          4: "bad argument", 5: "out of memory"}

DTYPE_CODE = {"bf16": 0, "fp32": 1, "f64": 2}


def build(src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    """Compile the C oracle with gcc (-O2, IEEE arithmetic, no fast-math)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(lib: str, src: str) -> bool:
    return (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(src)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


class OracleError(RuntimeError):
    pass


class Oracle:
    """ctypes front of ``oracle.c``.  ``lib_path`` selects another build of
    the same source (the pin tests load deliberately broken copies)."""

    def __init__(self, lib_path: str | None = None):
        if lib_path is None:
            if _needs_build(_LIB, _SRC):
                build()
            lib_path = _LIB
        self.lib = ctypes.CDLL(lib_path)
        L = self.lib
        i64, i32, vp, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_double
        L.oracle_graph_structured_nnz.restype = i64
        L.oracle_graph_structured_nnz.argtypes = [i64, i32, vp, i32]
        L.oracle_graph_structured.restype = ctypes.c_int
        L.oracle_graph_structured.argtypes = [i64, i32, vp, i32, vp, vp]
        L.oracle_graph_structured_rows.restype = ctypes.c_int
        L.oracle_graph_structured_rows.argtypes = [i64, vp, i32, vp, i32, vp, vp]
        L.oracle_graph_normalize.restype = ctypes.c_int
        L.oracle_graph_normalize.argtypes = [i64, vp, vp, vp, vp, vp]
        L.oracle_graph_reverse.restype = ctypes.c_int
        L.oracle_graph_reverse.argtypes = [i64, vp, vp, vp, vp]
        L.oracle_attn_fwd.restype = ctypes.c_int
        L.oracle_attn_fwd.argtypes = [i64, i32, ctypes.c_int, vp, vp, vp, vp, vp, dbl, vp, vp]
        L.oracle_attn_bwd.restype = ctypes.c_int
        L.oracle_attn_bwd.argtypes = [i64, i64, i32, ctypes.c_int, vp, vp, vp, vp, vp, vp, dbl,
                                      vp, vp, vp]
        L.oracle_dist_fwd.restype = ctypes.c_int
        L.oracle_dist_fwd.argtypes = [i64, i32, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp,
                                      dbl, vp, vp]
        L.oracle_dist_bwd.restype = ctypes.c_int
        L.oracle_dist_bwd.argtypes = [i64, i64, i32, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp,
                                      vp, vp, dbl, vp, vp, vp]

    # ---------------- graph ----------------
    def structured_nnz(self, T: int, W: int, exps) -> int:
        e = np.ascontiguousarray(np.asarray(list(exps), dtype=np.int32))
        return int(self.lib.oracle_graph_structured_nnz(T, W, _ptr(e), len(e)))

    def structured(self, T: int, W: int, exps):
        """CSR (rowptr int64[T+1], colidx int32[nnz]) of the window + 2^k graph."""
        e = np.ascontiguousarray(np.asarray(list(exps), dtype=np.int32))
        nnz = self.structured_nnz(T, W, exps)
        rowptr = np.zeros(T + 1, dtype=np.int64)
        colidx = np.zeros(max(nnz, 1), dtype=np.int32)
        st = self.lib.oracle_graph_structured(T, W, _ptr(e), len(e), _ptr(rowptr), _ptr(colidx))
        if st:
            raise OracleError(STATUS[st])
        return rowptr, colidx[:nnz]

    def structured_rows(self, rows, W: int, exps):
        """Neighbour lists of the given query positions only (any T):
        (rowptr int64[len(rows)+1], colidx int32[...])."""
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        e = np.ascontiguousarray(np.asarray(list(exps), dtype=np.int32))
        rowptr = np.zeros(len(rows) + 1, dtype=np.int64)
        st = self.lib.oracle_graph_structured_rows(len(rows), _ptr(rows), W, _ptr(e), len(e),
                                                   _ptr(rowptr), None)
        if st:
            raise OracleError(STATUS[st])
        colidx = np.zeros(max(int(rowptr[-1]), 1), dtype=np.int32)
        st = self.lib.oracle_graph_structured_rows(len(rows), _ptr(rows), W, _ptr(e), len(e),
                                                   _ptr(rowptr), _ptr(colidx))
        if st:
            raise OracleError(STATUS[st])
        return rowptr, colidx[: int(rowptr[-1])]

    def normalize(self, rowptr, colidx):
        """Sort + deduplicate every row; raises OracleError on an invalid graph."""
        rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
        colidx = np.ascontiguousarray(colidx, dtype=np.int32)
        T = len(rowptr) - 1
        out_r = np.zeros(T + 1, dtype=np.int64)
        out_c = np.zeros(max(len(colidx), 1), dtype=np.int32)
        nnz = np.zeros(1, dtype=np.int64)
        st = self.lib.oracle_graph_normalize(T, _ptr(rowptr), _ptr(colidx), _ptr(out_r),
                                             _ptr(out_c), _ptr(nnz))
        if st:
            raise OracleError(STATUS[st])
        return out_r, out_c[: int(nnz[0])]

    def reverse(self, rowptr, colidx):
        rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
        colidx = np.ascontiguousarray(colidx, dtype=np.int32)
        T = len(rowptr) - 1
        rr = np.zeros(T + 1, dtype=np.int64)
        rc = np.zeros(max(len(colidx), 1), dtype=np.int32)
        st = self.lib.oracle_graph_reverse(T, _ptr(rowptr), _ptr(colidx), _ptr(rr), _ptr(rc))
        if st:
            raise OracleError(STATUS[st])
        return rr, rc[: int(rowptr[-1])]

    # ---------------- attention ----------------
    @staticmethod
    def _as_input(x: np.ndarray, dtype: str) -> np.ndarray:
        if dtype == "bf16":
            assert x.dtype == np.uint16, "bf16 inputs are passed as raw uint16 bits"
        elif dtype == "fp32":
            x = x.astype(np.float32, copy=False)
        else:
            x = x.astype(np.float64, copy=False)
        return np.ascontiguousarray(x)

    def fwd(self, q, k, v, rowptr, colidx, scale: float, dtype: str = "f64"):
        """q [nq, D]; k, v [nk, D]; neighbour lists index k/v rows.
        Returns out [nq, D] (fp64) and lse [nq] (fp64, natural log)."""
        q, k, v = (self._as_input(x, dtype) for x in (q, k, v))
        nq, D = q.shape
        rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
        colidx = np.ascontiguousarray(colidx, dtype=np.int32)
        assert len(rowptr) == nq + 1
        if len(colidx):
            assert colidx.min() >= 0 and colidx.max() < k.shape[0]
        out = np.zeros((nq, D), dtype=np.float64)
        lse = np.zeros(nq, dtype=np.float64)
        st = self.lib.oracle_attn_fwd(nq, D, DTYPE_CODE[dtype], _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(rowptr), _ptr(colidx), float(scale), _ptr(out), _ptr(lse))
        if st:
            raise OracleError(STATUS[st])
        return out, lse

    def bwd(self, q, k, v, dout, rowptr, colidx, scale: float, dtype: str = "f64"):
        """Gradients of sum(dout * out) w.r.t. q [nq, D], k and v [nk, D]."""
        q, k, v, dout = (self._as_input(x, dtype) for x in (q, k, v, dout))
        nq, D = q.shape
        nk = k.shape[0]
        rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
        colidx = np.ascontiguousarray(colidx, dtype=np.int32)
        if len(colidx):
            assert colidx.min() >= 0 and colidx.max() < nk
        dq = np.zeros((nq, D), dtype=np.float64)
        dk = np.zeros((nk, D), dtype=np.float64)
        dv = np.zeros((nk, D), dtype=np.float64)
        st = self.lib.oracle_attn_bwd(nq, nk, D, DTYPE_CODE[dtype], _ptr(q), _ptr(k), _ptr(v),
                                      _ptr(dout), _ptr(rowptr), _ptr(colidx), float(scale),
                                      _ptr(dq), _ptr(dk), _ptr(dv))
        if st:
            raise OracleError(STATUS[st])
        return dq, dk, dv


    # ---------------- learned-coordinate (distance) scoring ----------------
    @staticmethod
    def _coords(x: np.ndarray, cdtype: str) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float32 if cdtype == "fp32" else np.float64)
        assert x.ndim == 2 and x.shape[1] == 3, "coordinates are [n, 3]"
        return x

    def dist_fwd(self, a, c, v, rowptr, colidx, scale: float, dtype: str = "f64",
                 cdtype: str = "f64"):
        """s_ij = -scale * |a_i - c_j|^2 over the lists.  a [nq, 3] query
        coordinates; c [nk, 3] key coordinates; v [nk, D].  Returns out
        [nq, D] and lse [nq] (fp64, natural log)."""
        a, c = self._coords(a, cdtype), self._coords(c, cdtype)
        v = self._as_input(v, dtype)
        nq, D = a.shape[0], v.shape[1]
        rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
        colidx = np.ascontiguousarray(colidx, dtype=np.int32)
        assert len(rowptr) == nq + 1
        if len(colidx):
            assert colidx.min() >= 0 and colidx.max() < c.shape[0] and c.shape[0] == v.shape[0]
        out = np.zeros((nq, D), dtype=np.float64)
        lse = np.zeros(nq, dtype=np.float64)
        st = self.lib.oracle_dist_fwd(nq, D, DTYPE_CODE[cdtype], DTYPE_CODE[dtype], _ptr(a),
                                      _ptr(c), _ptr(v), _ptr(rowptr), _ptr(colidx), float(scale),
                                      _ptr(out), _ptr(lse))
        if st:
            raise OracleError(STATUS[st])
        return out, lse

    def dist_bwd(self, a, c, v, dout, rowptr, colidx, scale: float, dtype: str = "f64",
                 cdtype: str = "f64"):
        """Gradients of sum(dout * out) w.r.t. a [nq, 3], c [nk, 3], v [nk, D]."""
        a, c = self._coords(a, cdtype), self._coords(c, cdtype)
        v, dout = self._as_input(v, dtype), self._as_input(dout, dtype)
        nq, nk, D = a.shape[0], c.shape[0], v.shape[1]
        rowptr = np.ascontiguousarray(rowptr, dtype=np.int64)
        colidx = np.ascontiguousarray(colidx, dtype=np.int32)
        if len(colidx):
            assert colidx.min() >= 0 and colidx.max() < nk
        da = np.zeros((nq, 3), dtype=np.float64)
        dc = np.zeros((nk, 3), dtype=np.float64)
        dv = np.zeros((nk, D), dtype=np.float64)
        st = self.lib.oracle_dist_bwd(nq, nk, D, DTYPE_CODE[cdtype], DTYPE_CODE[dtype], _ptr(a),
                                      _ptr(c), _ptr(v), _ptr(dout), _ptr(rowptr), _ptr(colidx),
                                      float(scale), _ptr(da), _ptr(dc), _ptr(dv))
        if st:
            raise OracleError(STATUS[st])
        return da, dc, dv


_default: Oracle | None = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
