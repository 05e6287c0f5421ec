"""The C ABI without a GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from recurrent_memory_transformer_diag_b200 import armt
from recurrent_memory_transformer_diag_b200.inputs import CONFIGS

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "armt.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(armt_[a-z_]+)\s*\(", src)))


def test_header_declarations_match_binding():
    assert _declared() == sorted(armt.EXPORTS)


def test_library_exports_every_declared_symbol(libarmt):
    for name in _declared():
        assert hasattr(libarmt, name), name


def test_status_strings(libarmt):
    for code in range(9):
        s = libarmt.armt_status_string(code)
        assert s and s != b"unknown status"
    assert libarmt.armt_status_string(99) == b"unknown status"


def _cfg(**kw):
    c = armt.make_c_config(CONFIGS["tiny"])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,status", [
    ("n_layers", 0, 1), ("d_model", -1, 1), ("n_mem", -1, 1), ("max_segments", 0, 1),
    ("write_gate", 2, 1), ("gamma_unclamped", -1, 1),
    ("n_kv_heads", 3, 1), ("head_dim", 15, 1), ("dtype", 7, 1), ("schedule", 5, 1),
    ("mem_eps", 0.0, 1), ("rope_theta", -1.0, 1), ("dpfp_nu", 40, 1),
    ("head_dim", 48, 7), ("n_mem", 40, 7), ("d_key", 600, 7),
])
def test_create_rejects_bad_config_before_device(libarmt, field, value, status):
    c = _cfg(**{field: value})
    h = ctypes.c_void_p(123)
    assert libarmt.armt_create(ctypes.byref(c), ctypes.byref(h)) == status
    assert h.value is None


def test_null_arguments(libarmt):
    assert libarmt.armt_create(None, None) == 1
    h = ctypes.c_void_p()
    assert libarmt.armt_create(None, ctypes.byref(h)) == 1
    assert libarmt.armt_destroy(None) == 0
    assert libarmt.armt_set_schedule(None, 0) == 1
    assert libarmt.armt_forward(None, None, 1, 1, None, None, None, None) == 1
    assert libarmt.armt_load_weights(None, None) == 1
    n = ctypes.c_int()
    assert libarmt.armt_launch_count(None, 1, ctypes.byref(n)) == 1
    idx = (ctypes.c_int * 1)(0)
    assert libarmt.armt_grouped_gemm(1, 0, 8, 16, 16, None, None, 1, idx, None, None) == 1
    assert libarmt.armt_memory_write(0, 8, 2, 1, 1e-5, None, None, None, None, None, None) == 1
    assert libarmt.armt_forward_ex(None, None, 1, 1, None, None, None, 0, None) == 1


def test_bf16_requires_aligned_dims(libarmt):
    c = armt.make_c_config(CONFIGS["small"])
    c.d_ffn = 690
    h = ctypes.c_void_p()
    assert libarmt.armt_create(ctypes.byref(c), ctypes.byref(h)) == 7


def test_create_without_device_reports_cuda_error(libarmt):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    c = _cfg()
    h = ctypes.c_void_p()
    assert libarmt.armt_create(ctypes.byref(c), ctypes.byref(h)) == 5
