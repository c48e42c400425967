"""ctypes mirror of include/gdla.h and the loader of libgdla.so.

Loading fails loudly (RuntimeError) when the native library is missing: there
is no Python or CPU fallback for any step of the layer.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdla.so")

GDLA_OK, GDLA_ERR_INVALID_ARG, GDLA_ERR_UNSUPPORTED, GDLA_ERR_CUDA, GDLA_ERR_TIMEOUT, GDLA_ERR_SCRATCH_LIMIT = range(6)
GDLA_DECODE_NOALLOC_SCRATCH_BYTES = 32 << 20
GDLA_MASK_CAUSAL, GDLA_MASK_SLIDING = 0, 1
GDLA_BF16, GDLA_FP32 = 0, 1

_vp = ctypes.c_void_p
_fp = ctypes.POINTER(ctypes.c_float)
_ip = ctypes.POINTER(ctypes.c_int)


class ExpandArgs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "L", "d_c", "d_rope", "n_kv", "d_nope", "d_v")] + [
        ("dtype", ctypes.c_int), ("rms_eps", ctypes.c_float), ("rope_max_pos", ctypes.c_int),
        ("c_kv", _vp), ("gamma", _vp), ("k_rope", _vp), ("w_ukv", _vp), ("rope_cos", _vp), ("rope_sin", _vp),
        ("kv_out", _vp), ("k_rope_out", _vp), ("c_hat_out", _vp)]


class PrefillArgs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "L", "d_c", "d_rope", "n_kv", "d_nope", "d_v", "n_noise", "g")] + [
        ("mask", ctypes.c_int), ("window", ctypes.c_int), ("softmax_scale", ctypes.c_float),
        ("rms_eps", ctypes.c_float), ("dtype", ctypes.c_int), ("rope_max_pos", ctypes.c_int),
        ("c_kv", _vp), ("gamma", _vp), ("k_rope", _vp), ("q", _vp), ("w_ukv", _vp), ("rope_cos", _vp),
        ("rope_sin", _vp), ("lam_logits", _vp), ("gate_logits", _vp), ("out", _vp), ("cache_c_hat", _vp),
        ("cache_k_rope", _vp), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class AttendArgs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "L", "d_rope", "n_kv", "d_nope", "d_v", "n_noise", "g")] + [
        ("mask", ctypes.c_int), ("window", ctypes.c_int), ("softmax_scale", ctypes.c_float),
        ("dtype", ctypes.c_int), ("rope_max_pos", ctypes.c_int),
        ("q", _vp), ("kv", _vp), ("k_rope_rot", _vp), ("rope_cos", _vp), ("rope_sin", _vp), ("lam_logits", _vp),
        ("gate_logits", _vp), ("out", _vp), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
        ("q_len", ctypes.c_int), ("q_start", ctypes.c_int)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "T_max", "d_c", "d_rope", "n_kv", "d_nope", "d_v", "n_noise", "g")] + [
        ("mask", ctypes.c_int), ("window", ctypes.c_int), ("softmax_scale", ctypes.c_float),
        ("dtype", ctypes.c_int), ("rope_max_pos", ctypes.c_int),
        ("seqlens", _vp), ("c_cache", _vp), ("kr_cache", _vp), ("q", _vp), ("w_ukv", _vp), ("rope_cos", _vp),
        ("rope_sin", _vp), ("lam_logits", _vp), ("gate_logits", _vp), ("out", _vp), ("workspace", _vp),
        ("workspace_bytes", ctypes.c_size_t)]


class GatesArgs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "L", "d_q", "d_x", "n_signal", "d_v")] + [
        ("dtype", ctypes.c_int), ("rms_eps", ctypes.c_float),
        ("c_q", _vp), ("gamma_q", _vp), ("w_g", _vp), ("x", _vp), ("w_lambda", _vp), ("gate_logits", _vp),
        ("lam_logits", _vp), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


# Every symbol include/gdla.h declares.
EXPORTED = ("gdla_latent_expand", "gdla_prefill_workspace_size", "gdla_prefill", "gdla_prefill_host_workspace_size",
            "gdla_prefill_host", "gdla_attend", "gdla_decode_workspace_size", "gdla_decode", "gdla_decode_noalloc",
            "gdla_gates_workspace_size", "gdla_gates", "gdla_status_string", "gdla_workspace_status",
            "gdla_build_info", "gdla_diag_wait_timeout", "gdla_rope_tables", "gdla_yarn_rope_tables",
            "gdla_yarn_mscale")

_lock = threading.Lock()
_lib = None


def load(path: str = LIB_PATH):
    """Load libgdla.so and declare its signatures (once)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"libgdla.so not found at {path}: build it with "
                "`python -m differential_latent_attention_gdla_b200.build` (there is no fallback path)")
        lib = ctypes.CDLL(path)
        lib.gdla_latent_expand.argtypes = [ctypes.POINTER(ExpandArgs), _vp]
        lib.gdla_latent_expand.restype = ctypes.c_int
        lib.gdla_prefill_workspace_size.argtypes = [ctypes.POINTER(PrefillArgs)]
        lib.gdla_prefill_workspace_size.restype = ctypes.c_size_t
        lib.gdla_prefill.argtypes = [ctypes.POINTER(PrefillArgs), _vp]
        lib.gdla_prefill.restype = ctypes.c_int
        lib.gdla_prefill_host_workspace_size.argtypes = [ctypes.POINTER(PrefillArgs), ctypes.c_int]
        lib.gdla_prefill_host_workspace_size.restype = ctypes.c_size_t
        lib.gdla_prefill_host.argtypes = [ctypes.POINTER(PrefillArgs), ctypes.c_int, _vp]
        lib.gdla_prefill_host.restype = ctypes.c_int
        lib.gdla_attend.argtypes = [ctypes.POINTER(AttendArgs), _vp]
        lib.gdla_attend.restype = ctypes.c_int
        lib.gdla_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeArgs)]
        lib.gdla_decode_workspace_size.restype = ctypes.c_size_t
        lib.gdla_decode.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
        lib.gdla_decode.restype = ctypes.c_int
        lib.gdla_decode_noalloc.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
        lib.gdla_decode_noalloc.restype = ctypes.c_int
        lib.gdla_gates_workspace_size.argtypes = [ctypes.POINTER(GatesArgs)]
        lib.gdla_gates_workspace_size.restype = ctypes.c_size_t
        lib.gdla_gates.argtypes = [ctypes.POINTER(GatesArgs), _vp]
        lib.gdla_gates.restype = ctypes.c_int
        lib.gdla_status_string.argtypes = [ctypes.c_int]
        lib.gdla_status_string.restype = ctypes.c_char_p
        lib.gdla_workspace_status.argtypes = [_vp, _vp]
        lib.gdla_diag_wait_timeout.argtypes = [_vp, _vp]
        lib.gdla_diag_wait_timeout.restype = ctypes.c_int
        lib.gdla_workspace_status.restype = ctypes.c_int
        lib.gdla_build_info.argtypes = []
        lib.gdla_build_info.restype = ctypes.c_char_p
        lib.gdla_rope_tables.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, _fp, _fp]
        lib.gdla_rope_tables.restype = ctypes.c_int
        lib.gdla_yarn_rope_tables.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                              ctypes.c_int, ctypes.c_double, ctypes.c_double, _fp, _fp]
        lib.gdla_yarn_rope_tables.restype = ctypes.c_int
        lib.gdla_yarn_mscale.argtypes = [ctypes.c_double]
        lib.gdla_yarn_mscale.restype = ctypes.c_double
        _lib = lib
        return lib


class GdlaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = load().gdla_status_string(code).decode()
        super().__init__(f"{what}: {msg}")


def check(code: int, what: str):
    if code != GDLA_OK:
        raise GdlaError(code, what)
