"""The C-ABI library: it loads without a GPU, exports exactly what include/sfnn.h
declares, and rejects bad arguments with a status code before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import activation_sparse_ffn_threshold_b200 as sf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sfnn.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^SFNN_API\s+[^;(]*?\b(sfnn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("sfnn_create", "sfnn_predict", "sfnn_forward", "sfnn_forward_batch", "sfnn_destroy"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = sf.load_library()
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", sf.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted(l.split()[-1] for l in out.splitlines() if " T " in l)
    assert exported == _declared()


def test_status_strings():
    lib = sf.load_library()
    for code in range(6):
        assert lib.sfnn_status_str(code)
    assert lib.sfnn_status_str(99) == b"unknown status"


def test_null_and_invalid_arguments_return_status():
    lib = sf.load_library()
    h = ctypes.c_void_p()
    assert lib.sfnn_create(None, None, ctypes.byref(h)) == 1
    assert lib.sfnn_create(None, None, None) == 1
    desc = sf.LayerDesc(0, 16, 8, 1, 0, 1, 1, None, 1, 1, 1, 1, 1, None)
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 1 and not h.value
    desc = sf.LayerDesc(12, 16, 8, 1, 0, 1, 1, None, 1, 1, 1, 1, 1, None)  # d not a multiple of 8 (fp16)
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 1
    desc = sf.LayerDesc(16, 16, 8, 1, 1, 1, 1, None, 1, 1, 1, 1, 1, None)  # ReGLU without w_gate
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 1
    desc = sf.LayerDesc(16, 16, 8, 33, 0, 1, 1, None, 1, 1, 1, 1, 1, None)  # batch above 32
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 4
    desc = sf.LayerDesc(16, 16, 8, 1, 5, 1, 1, None, 1, 1, 1, 1, 1, None)  # bad activation
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 1
    desc = sf.LayerDesc(16, 16, 8, 1, 0, 0, 1, None, 1, 1, 1, 1, 1, None, sf.I8)  # int8 rows of fp32 weights
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 4
    desc = sf.LayerDesc(24, 16, 8, 1, 0, 1, 1, None, 1, 1, 1, 1, 1, None, sf.I8)  # int8 rows, d % 16 != 0
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 4
    desc = sf.LayerDesc(32, 16, 8, 1, 0, 0, 1, None, 1, 1, 1, 1, 1, None, sf.I4)  # int4 rows of fp32 weights
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 4
    desc = sf.LayerDesc(48, 16, 8, 1, 0, 1, 1, None, 1, 1, 1, 1, 1, None, sf.I4)  # int4 rows, d % 32 != 0
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 4
    desc = sf.LayerDesc(16, 16, 8, 1, 0, 1, 1, None, 1, 1, 1, 1, 1, None, 0, 7)  # unknown storage order
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 1
    assert lib.sfnn_set_hot_prefix(None, 1) == 1
    assert lib.sfnn_set_fused_quota(None, 1) == 1
    assert lib.sfnn_set_batch_quota(None, 1) == 1
    assert lib.sfnn_tune_batch_paths(None, None, None) == 1
    assert lib.sfnn_set_batch_depths(None, 6, 4, 2, 4) == 1
    assert lib.sfnn_set_batch_tc_shape(None, 2, 1, 1) == 1
    assert lib.sfnn_set_fused_depths(None, 4, 8, 2, 8) == 1
    assert lib.sfnn_forward(None, 1, None, None, 1, None) == 1
    assert lib.sfnn_predict(None, 1, 1, 1, None) == 1
    assert lib.sfnn_forward_batch(None, 1, 1, 1, None, None, None) == 1
    assert lib.sfnn_forward_stack(None, 1, 1, 1, 1, None, None, None) == 1
    assert lib.sfnn_forward_stack_lookahead(None, 1, 1, 1, 1, None, None, None) == 1
    assert lib.sfnn_destroy(None) == 0
    assert lib.sfnn_get_error(None) == 1
    assert lib.sfnn_set_batch_path(None, 0) == 1
    assert lib.sfnn_query(None, None) == 1


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU error path")
def test_create_without_gpu_reports_cuda_error():
    lib = sf.load_library()
    h = ctypes.c_void_p()
    desc = sf.LayerDesc(16, 16, 8, 1, 0, 1, 1, None, 1, 1, 1, 1, 1, None)
    assert lib.sfnn_create(ctypes.byref(desc), None, ctypes.byref(h)) == 2 and not h.value


def test_hotness_order_host_logic():
    hot = np.array([0.1, 0.9, np.nan, 0.9, 0.5, 0.0], np.float32)
    assert sf.hotness_order(hot).tolist() == [1, 3, 4, 0, 5, 2]
    rng = np.random.default_rng(0)
    h = rng.random(1000).astype(np.float32)
    perm = sf.hotness_order(h)
    assert sorted(perm.tolist()) == list(range(1000))
    assert np.all(np.diff(h[perm]) <= 0)
