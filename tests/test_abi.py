"""The C-ABI library loads and exports every entry point that
include/*.h declares; host-side argument checks reject bad calls before any
CUDA work.  No GPU needed."""
import ctypes
import glob
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"\b(sparse_attn_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("sparse_attn_graph_build_structured", "sparse_attn_graph_build_csr",
              "sparse_attn_fwd", "sparse_attn_bwd", "sparse_attn_bwd_workspace_size",
              "sparse_attn_graph_export", "sparse_attn_graph_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import sparse_graph_causal_b200 as sa
    lib = ctypes.CDLL(sa.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_python_binding_has_the_same_names():
    import sparse_graph_causal_b200 as sa
    for n in declared_functions():
        assert hasattr(sa, n), n


def test_host_side_rejections():
    import sparse_graph_causal_b200 as sa
    lib = sa._lib
    h = ctypes.c_void_p()
    assert lib.sparse_attn_launch_count() >= 0
    # bad sizes are rejected before any CUDA call
    assert lib.sparse_attn_graph_build_structured(0, 4, None, 0, 0, None, ctypes.byref(h)) == 1
    assert lib.sparse_attn_graph_build_structured(16, 0, None, 0, 0, None, ctypes.byref(h)) == 1
    exps = (ctypes.c_int32 * 1)(70)
    assert lib.sparse_attn_graph_build_structured(16, 2, exps, 1, 0, None, ctypes.byref(h)) == 1
    assert lib.sparse_attn_graph_build_csr(0, None, None, 0, 0, None, ctypes.byref(h)) == 1
    assert lib.sparse_attn_fwd(None, None, None, None, 1.0, None, None, None) == 1
    assert lib.sparse_attn_set_path(7) == 1
    assert lib.sparse_attn_set_link_pass(3) == 1 and lib.sparse_attn_set_link_pass(-1) == 1
    assert sa.sparse_attn_status_string(2) == "invalid graph"


def test_cpu_tensors_are_refused():
    import sparse_graph_causal_b200 as sa
    x = torch.zeros(1, 1, 8, 32)
    with pytest.raises(ValueError):
        sa._tensor(x, "q")
