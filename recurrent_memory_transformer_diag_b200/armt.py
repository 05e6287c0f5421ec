"""ctypes binding of libarmt.so (include/armt.h): argument marshalling only.

Every step of the forward runs in the library's CUDA kernels.  PyTorch is
used only to own device buffers and streams (``tensor.data_ptr()`` and
``torch.cuda.current_stream().cuda_stream`` are handed to the C ABI).  There
is no CPU or PyTorch fallback: if the library is missing or a call fails,
an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np

from .inputs import ArmtConfig

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libarmt.so")

ARMT_FP32, ARMT_BF16, ARMT_F16, ARMT_TF32 = 0, 1, 2, 3
SCHED = {"diagonal": 0, "sequential": 1}

STATUS = {
    0: "ARMT_OK", 1: "ARMT_ERR_INVALID_ARG", 2: "ARMT_ERR_NOT_LOADED", 3: "ARMT_ERR_SHAPE",
    4: "ARMT_ERR_OOM", 5: "ARMT_ERR_CUDA", 6: "ARMT_ERR_DEVICE_TIMEOUT", 7: "ARMT_ERR_UNSUPPORTED",
    8: "ARMT_ERR_NUMERIC_RANGE",
}

# Every symbol the header declares (checked by the CPU tests).
EXPORTS = (
    "armt_create", "armt_load_weights", "armt_set_schedule", "armt_set_graph", "armt_forward",
    "armt_forward_host", "armt_device_status", "armt_launch_count", "armt_destroy",
    "armt_status_string", "armt_last_error", "armt_grouped_gemm", "armt_memory_write",
    "armt_kernel_kinds", "armt_kernel_kind_name", "armt_profile_forward", "armt_memory_write_static",
    "armt_forward_ex", "armt_test_bounded_wait", "armt_stage_wave",
)


class ArmtError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name}" + (f" ({detail})" if detail else ""))


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim",
                                            "d_ffn", "n_mem", "d_key", "dpfp_nu")] + \
               [("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float), ("mem_eps", ctypes.c_float),
                ("dtype", ctypes.c_int), ("schedule", ctypes.c_int),
                ("max_seg_len", ctypes.c_int), ("max_segments", ctypes.c_int),
                ("write_gate", ctypes.c_int), ("gamma_unclamped", ctypes.c_int)]


_WEIGHT_FIELDS = ("mem_emb", "attn_norm", "mlp_norm", "wq", "wk", "wv", "wo", "w_gate", "w_up",
                  "w_down", "wq_mem", "wk_mem", "wv_mem", "w_beta")


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _WEIGHT_FIELDS]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libarmt.so (built in-tree by ``python -m recurrent_memory_transformer_diag_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libarmt.so is not built ({LIB_PATH}); run "
                           "`python -m recurrent_memory_transformer_diag_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    c_int, c_float, vp = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
    L.armt_create.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(vp)]
    L.armt_load_weights.argtypes = [vp, ctypes.POINTER(_Weights)]
    L.armt_set_schedule.argtypes = [vp, c_int]
    L.armt_set_graph.argtypes = [vp, c_int]
    L.armt_forward.argtypes = [vp, vp, c_int, c_int, vp, vp, vp, vp]
    L.armt_forward_ex.argtypes = [vp, vp, c_int, c_int, vp, vp, vp, c_int, vp]
    L.armt_forward_host.argtypes = [vp, vp, c_int, c_int, vp, vp, vp, vp]
    L.armt_device_status.argtypes = [vp, vp]
    L.armt_launch_count.argtypes = [vp, c_int, ctypes.POINTER(c_int)]
    L.armt_destroy.argtypes = [vp]
    L.armt_status_string.argtypes = [c_int]
    L.armt_status_string.restype = ctypes.c_char_p
    L.armt_last_error.argtypes = [vp]
    L.armt_last_error.restype = ctypes.c_char_p
    L.armt_grouped_gemm.argtypes = [c_int, c_int, c_int, c_int, c_int, vp, vp, c_int,
                                    ctypes.POINTER(c_int), vp, vp]
    L.armt_memory_write.argtypes = [c_int, c_int, c_int, c_int, c_float, vp, vp, vp, vp, vp, vp]
    L.armt_memory_write_static.argtypes = [c_int, c_int, c_int, c_int, c_float, vp, vp, vp, vp, vp, vp]
    L.armt_test_bounded_wait.argtypes = [vp]
    L.armt_stage_wave.argtypes = [vp, c_int, c_int, c_int, c_int, c_int, vp, vp, vp, vp, vp, vp, c_int, vp]
    L.armt_kernel_kinds.argtypes = []
    L.armt_kernel_kind_name.argtypes = [c_int]
    L.armt_kernel_kind_name.restype = ctypes.c_char_p
    L.armt_profile_forward.argtypes = [vp, vp, c_int, c_int, vp, vp, vp, vp,
                                       ctypes.POINTER(ctypes.c_double), ctypes.POINTER(c_int)]
    for name in EXPORTS:
        if name not in ("armt_status_string", "armt_last_error", "armt_kernel_kind_name"):
            getattr(L, name).restype = c_int
    _lib = L
    return L


def _check(status: int, where: str, ctx=None):
    if status != 0:
        detail = ""
        if ctx is not None:
            detail = (lib().armt_last_error(ctx) or b"").decode()
        raise ArmtError(status, where, detail)


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t) -> Optional[int]:
    if t is None:
        return None   # NULL
    return t.data_ptr() if hasattr(t, "data_ptr") else t.ctypes.data


def make_c_config(cfg: ArmtConfig, max_segments: Optional[int] = None, max_seg_len: Optional[int] = None,
                  schedule: str = "diagonal") -> _Config:
    c = _Config()
    for n in ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "d_ffn", "n_mem", "d_key", "dpfp_nu"):
        setattr(c, n, getattr(cfg, n))
    c.rope_theta, c.rms_eps, c.mem_eps = cfg.rope_theta, cfg.rms_eps, cfg.mem_eps
    c.dtype = ARMT_BF16 if cfg.dtype == "bf16" else ARMT_FP32
    c.schedule = SCHED[schedule]
    c.max_seg_len = max_seg_len or cfg.seg_len
    c.max_segments = max_segments or cfg.n_segments
    c.write_gate = int(bool(getattr(cfg, "write_gate", False)))
    c.gamma_unclamped = int(not getattr(cfg, "gamma_clamp", True))
    return c


class Armt:
    """One library context (weights + workspace) on the current CUDA device."""

    def __init__(self, cfg: ArmtConfig, max_segments: Optional[int] = None, max_seg_len: Optional[int] = None,
                 schedule: str = "diagonal"):
        self.cfg = cfg
        self._c = make_c_config(cfg, max_segments, max_seg_len, schedule)
        h = ctypes.c_void_p()
        _check(lib().armt_create(ctypes.byref(self._c), ctypes.byref(h)), "armt_create")
        self._h = h

    # -- lifecycle
    def close(self):
        if getattr(self, "_h", None):
            lib().armt_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    # -- calls
    def load_weights(self, weights: Dict[str, np.ndarray]):
        keep = {k: np.ascontiguousarray(weights[k], dtype=np.float32) for k in _WEIGHT_FIELDS if k in weights}
        w = _Weights(**{k: v.ctypes.data for k, v in keep.items()})
        _check(lib().armt_load_weights(self._h, ctypes.byref(w)), "armt_load_weights", self._h)

    def set_schedule(self, schedule: str):
        _check(lib().armt_set_schedule(self._h, SCHED[schedule]), "armt_set_schedule", self._h)

    def set_graph(self, enable: bool):
        _check(lib().armt_set_graph(self._h, int(bool(enable))), "armt_set_graph", self._h)

    def forward(self, emb, n_segments: int, seg_len: int, out_hidden, out_A, out_z, stream=None):
        """Device buffers (torch tensors): see armt_forward in include/armt.h."""
        _check(lib().armt_forward(self._h, _ptr(emb), n_segments, seg_len, _ptr(out_hidden), _ptr(out_A),
                                  _ptr(out_z), _stream_handle(stream)), "armt_forward", self._h)

    def forward_ex(self, emb, n_segments: int, seg_len: int, out_hidden, A, z, carry_state: bool,
                   stream=None):
        """armt_forward_ex: with carry_state, A and z (device) hold the state to
        start from and are updated in place (streaming a long input across calls)."""
        _check(lib().armt_forward_ex(self._h, _ptr(emb), n_segments, seg_len, _ptr(out_hidden), _ptr(A),
                                     _ptr(z), int(bool(carry_state)), _stream_handle(stream)),
               "armt_forward_ex", self._h)

    def stage_wave(self, n_segments: int, seg_len: int, wave: int, layer_offset: int, total_layers: int,
                   emb, in_rows, out_rows, out_hidden, A, z, carry_state: bool = False, stream=None):
        """armt_stage_wave: one global wave of a layer-pipelined forward for this
        context's layer block (device buffers; None where the wave needs none)."""
        _check(lib().armt_stage_wave(self._h, n_segments, seg_len, wave, layer_offset, total_layers,
                                     _ptr(emb), _ptr(in_rows), _ptr(out_rows), _ptr(out_hidden), _ptr(A),
                                     _ptr(z), int(bool(carry_state)), _stream_handle(stream)),
               "armt_stage_wave", self._h)

    def forward_host(self, emb, n_segments: int, seg_len: int, out_hidden, out_A, out_z, stream=None):
        """Host buffers (numpy arrays or pinned CPU tensors): see armt_forward_host."""
        _check(lib().armt_forward_host(self._h, _ptr(emb), n_segments, seg_len, _ptr(out_hidden),
                                       _ptr(out_A), _ptr(out_z), _stream_handle(stream)),
               "armt_forward_host", self._h)

    def profile_forward(self, emb, n_segments: int, seg_len: int, out_hidden, out_A, out_z, stream=None):
        """One un-graphed forward with CUDA events around every launch:
        returns {kernel kind: (device ms, launches)}."""
        L = lib()
        n = L.armt_kernel_kinds()
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int * n)()
        _check(L.armt_profile_forward(self._h, _ptr(emb), n_segments, seg_len, _ptr(out_hidden), _ptr(out_A),
                                      _ptr(out_z), _stream_handle(stream), ms, cnt), "armt_profile_forward", self._h)
        return {L.armt_kernel_kind_name(k).decode(): (ms[k], cnt[k]) for k in range(n) if cnt[k]}

    def device_status(self, stream=None):
        _check(lib().armt_device_status(self._h, _stream_handle(stream)), "armt_device_status", self._h)

    def launch_count(self, n_segments: int) -> int:
        n = ctypes.c_int()
        _check(lib().armt_launch_count(self._h, n_segments, ctypes.byref(n)), "armt_launch_count", self._h)
        return n.value


def grouped_gemm(A, B, bidx, C, stream=None, tf32: bool = False):
    """C[g] = A[g] @ B[bidx[g]]^T on device tensors; bf16/fp16 -> tcgen05 kernel, fp32 -> SIMT
    (fp32 with tf32=True -> tcgen05 kind::tf32)."""
    import torch
    dtype = {torch.bfloat16: ARMT_BF16, torch.float16: ARMT_F16}.get(A.dtype, ARMT_FP32)
    if tf32:
        assert A.dtype == torch.float32 and B.dtype == torch.float32
        dtype = ARMT_TF32
    G, m, k = A.shape
    num_b, n, _ = B.shape
    idx = (ctypes.c_int * G)(*[int(i) for i in bidx])
    _check(lib().armt_grouped_gemm(dtype, G, m, n, k, _ptr(A), _ptr(B), num_b, idx, _ptr(C),
                                   _stream_handle(stream)), "armt_grouped_gemm")


def memory_write_static(m, wk, wv, A, z, nu: int, eps: float, stream=None):
    """armt_memory_write_static: the same write with the library's fixed
    device scratch, for callers that cannot allocate device memory."""
    M, d = m.shape
    dk = wk.shape[0]
    _check(lib().armt_memory_write_static(M, d, dk, nu, eps, _ptr(m), _ptr(wk), _ptr(wv), _ptr(A), _ptr(z),
                                          _stream_handle(stream)), "armt_memory_write_static")


def memory_write(m, wk, wv, A, z, nu: int, eps: float, stream=None):
    """Delta-rule write of one node on device fp32 tensors (A, z updated in place)."""
    M, d = m.shape
    dk = wk.shape[0]
    _check(lib().armt_memory_write(M, d, dk, nu, eps, _ptr(m), _ptr(wk), _ptr(wv), _ptr(A), _ptr(z),
                                   _stream_handle(stream)), "armt_memory_write")
