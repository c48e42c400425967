"""B200-native GDLA forward: Python binding of libgdla.so.

Grouped Differential Latent Attention ("Motif 3: Technical Report",
Architecture). The functions below only check tensors and marshal pointers and
sizes into the C ABI of ``include/gdla.h``; every step of the layer runs in the
library's CUDA kernels. PyTorch supplies device memory and streams.

    prefill(...)        whole forward for B sequences of L tokens
    decode(...)         one new token per sequence over the latent cache
    latent_expand(...)  latent RMSNorm + W_UKV expansion + rotary-key RoPE
    rope_tables(...)    the cos/sin tables the kernels read (set-up, like weights)
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _abi
from ._abi import GDLA_BF16, GDLA_FP32, GDLA_MASK_CAUSAL, GDLA_MASK_SLIDING, GdlaError  # noqa: F401

__all__ = ["prefill", "prefill_host", "prefill_host_workspace_size", "gates", "attend", "decode", "decode_noalloc", "latent_expand", "rope_tables", "yarn_rope_tables",
           "yarn_mscale", "prefill_workspace_size", "decode_workspace_size", "workspace_status", "diag_wait_timeout",
           "build_info", "GdlaError"]

_DT = {torch.bfloat16: GDLA_BF16, torch.float32: GDLA_FP32}


def _lib():
    return _abi.load()


def build_info() -> str:
    return _lib().gdla_build_info().decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("GDLA tensors must be CUDA device tensors")
    if not t.is_contiguous():
        raise ValueError("GDLA tensors must be contiguous (row-major)")
    return t.data_ptr()


def _host_ptr(t) -> int:
    if t.is_cuda:
        raise ValueError("prefill_host takes its activations as CPU tensors (page-locked for copy overlap)")
    if not t.is_contiguous():
        raise ValueError("GDLA tensors must be contiguous (row-major)")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype(t) -> int:
    if t.dtype not in _DT:
        raise ValueError(f"unsupported dtype {t.dtype}; GDLA takes bfloat16 or float32")
    return _DT[t.dtype]


def _mask(mask: str) -> int:
    if mask not in ("causal", "sliding"):
        raise ValueError("mask must be 'causal' or 'sliding'")
    return GDLA_MASK_CAUSAL if mask == "causal" else GDLA_MASK_SLIDING


def _tables(fill, max_pos: int, d_rope: int, device):
    cos = torch.empty((max_pos, d_rope // 2), dtype=torch.float32)
    sin = torch.empty_like(cos)
    fp = ctypes.POINTER(ctypes.c_float)
    _abi.check(fill(ctypes.cast(cos.data_ptr(), fp), ctypes.cast(sin.data_ptr(), fp)), "RoPE tables")
    return cos.to(device), sin.to(device)


def rope_tables(max_pos: int, d_rope: int, base: float = 10000.0, device="cuda"):
    """cos/sin tables [max_pos, d_rope/2] (fp32) of the rotate-half RoPE with
    frequencies theta_k = base^(-2k/d_rope), built by the library
    (gdla_rope_tables) on the host and moved to ``device``. Model set-up,
    computed once like any other constant input (a YaRN variant only changes
    these tables)."""
    return _tables(lambda c, s: _lib().gdla_rope_tables(int(max_pos), int(d_rope), float(base), c, s), max_pos,
                   d_rope, device)


def yarn_rope_tables(max_pos: int, d_rope: int, factor: float, original_max_pos: int, base: float = 10000.0,
                     beta_fast: float = 32.0, beta_slow: float = 1.0, device="cuda"):
    """cos/sin tables [max_pos, d_rope/2] (fp32) of RoPE with YaRN frequency scaling
    ("Open-Source Frontier Models: Architecture and Benchmarks of Rnj-1 and
    Motif-2", section 2, the Scale(i) equation), built by the library
    (gdla_yarn_rope_tables). Pair them with
    ``softmax_scale = yarn_mscale(factor)**2 / sqrt(d_qk)``."""
    return _tables(lambda c, s: _lib().gdla_yarn_rope_tables(int(max_pos), int(d_rope), float(base), float(factor),
                                                             int(original_max_pos), float(beta_fast),
                                                             float(beta_slow), c, s), max_pos, d_rope, device)


def yarn_mscale(factor: float) -> float:
    """YaRN's attention temperature m = 1 + 0.1 ln(factor) (1 for factor <= 1),
    from the library (gdla_yarn_mscale); the logits are multiplied by m^2, which
    the caller folds into softmax_scale."""
    return float(_lib().gdla_yarn_mscale(float(factor)))


# ------------------------------------------------------------------- expansion
def latent_expand(c_kv, gamma, k_rope, w_ukv, rope_cos, rope_sin, *, n_kv: int, d_nope: int, d_v: int,
                  rms_eps: float = 0.0, kv_out=None, k_rope_out=None, c_hat_out=None, stream=None):
    """Latent RMSNorm, W_UKV expansion and rotary-key RoPE. Returns
    (kv [B,L,n_kv,d_nope+d_v], k_rope_rot [B,L,d_rope], c_hat [B,L,d_c])."""
    B, L, d_c = c_kv.shape
    d_rope = k_rope.shape[-1]
    if kv_out is None:
        kv_out = torch.empty((B, L, n_kv, d_nope + d_v), dtype=c_kv.dtype, device=c_kv.device)
    if k_rope_out is None:
        k_rope_out = torch.empty((B, L, d_rope), dtype=c_kv.dtype, device=c_kv.device)
    if c_hat_out is None:
        c_hat_out = torch.empty((B, L, d_c), dtype=c_kv.dtype, device=c_kv.device)
    a = _abi.ExpandArgs(B, L, d_c, d_rope, n_kv, d_nope, d_v, _dtype(c_kv), rms_eps, rope_cos.shape[0],
                        _ptr(c_kv), _ptr(gamma), _ptr(k_rope), _ptr(w_ukv), _ptr(rope_cos), _ptr(rope_sin),
                        _ptr(kv_out), _ptr(k_rope_out), _ptr(c_hat_out))
    _abi.check(_lib().gdla_latent_expand(ctypes.byref(a), _stream(stream)), "gdla_latent_expand")
    return kv_out, k_rope_out, c_hat_out


# --------------------------------------------------------------------- prefill
def _prefill_args(c_kv, gamma, k_rope, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, out, g, mask, window,
                  softmax_scale, rms_eps, cache_c_hat, cache_k_rope, workspace, act_ptr=_ptr):
    B, L, d_c = c_kv.shape
    d_rope = k_rope.shape[-1]
    H_q, d_qk = q.shape[2], q.shape[3]
    if H_q % (g + 1):
        raise ValueError("q must hold g*n_noise signal heads followed by n_noise noise heads")
    n_noise = H_q // (g + 1)
    d_nope = d_qk - d_rope
    d_v = w_ukv.shape[1] // n_noise - d_nope
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _abi.PrefillArgs(B, L, d_c, d_rope, n_noise, d_nope, d_v, n_noise, g, _mask(mask), int(window),
                            float(softmax_scale), float(rms_eps), _dtype(c_kv), rope_cos.shape[0],
                            act_ptr(c_kv), _ptr(gamma), act_ptr(k_rope), act_ptr(q), _ptr(w_ukv), _ptr(rope_cos),
                            _ptr(rope_sin), act_ptr(lam_logits), act_ptr(gate_logits), act_ptr(out),
                            _ptr(cache_c_hat), _ptr(cache_k_rope), ws_ptr, ws_bytes)


def prefill_workspace_size(*, B, L, d_c, d_rope, n_kv, d_nope, d_v, g, dtype=torch.bfloat16) -> int:
    a = _abi.PrefillArgs()
    a.B, a.L, a.d_c, a.d_rope, a.n_kv, a.d_nope, a.d_v, a.n_noise, a.g = B, L, d_c, d_rope, n_kv, d_nope, d_v, n_kv, g
    a.dtype = _DT[dtype]
    return int(_lib().gdla_prefill_workspace_size(ctypes.byref(a)))


def prefill(c_kv, gamma, k_rope, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, *, g: int,
            mask: str = "causal", window: int = 0, softmax_scale: float = 0.0, rms_eps: float = 0.0, out=None,
            workspace=None, cache_c_hat=None, cache_k_rope=None, stream=None):
    """GDLA forward for B sequences of L tokens; returns Y [B, L, n_signal, d_v].

    Shapes: c_kv [B,L,d_c], gamma [d_c], k_rope [B,L,d_rope] (pre-RoPE),
    q [B,L,n_signal+n_noise,d_nope+d_rope] (signal heads first; rotary part
    pre-RoPE), w_ukv [d_c, n_kv*(d_nope+d_v)], lam_logits [B,L,n_signal] fp32,
    gate_logits [B,L,n_signal,d_v]. ``workspace`` is a uint8 CUDA tensor of at
    least prefill_workspace_size() bytes (allocated here when omitted)."""
    B, L = c_kv.shape[:2]
    n_signal = lam_logits.shape[-1]
    d_v_guess = gate_logits.shape[-1]
    if out is None:
        out = torch.empty((B, L, n_signal, d_v_guess), dtype=c_kv.dtype, device=c_kv.device)
    a = _prefill_args(c_kv, gamma, k_rope, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, out, g, mask,
                      window, softmax_scale, rms_eps, cache_c_hat, cache_k_rope, workspace)
    if workspace is None:
        need = int(_lib().gdla_prefill_workspace_size(ctypes.byref(a)))
        workspace = torch.empty(need, dtype=torch.uint8, device=c_kv.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), need
    _abi.check(_lib().gdla_prefill(ctypes.byref(a), _stream(stream)), "gdla_prefill")
    return out


def prefill_host_workspace_size(*, B, L, d_c, d_rope, n_kv, d_nope, d_v, g, chunk_tokens=0,
                                dtype=torch.bfloat16) -> int:
    a = _abi.PrefillArgs()
    a.B, a.L, a.d_c, a.d_rope, a.n_kv, a.d_nope, a.d_v, a.n_noise, a.g = B, L, d_c, d_rope, n_kv, d_nope, d_v, n_kv, g
    a.dtype = _DT[dtype]
    return int(_lib().gdla_prefill_host_workspace_size(ctypes.byref(a), int(chunk_tokens)))


def prefill_host(c_kv, gamma, k_rope, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, *, g: int,
                 mask: str = "causal", window: int = 0, softmax_scale: float = 0.0, rms_eps: float = 0.0,
                 chunk_tokens: int = 0, out=None, workspace=None, cache_c_hat=None, cache_k_rope=None, stream=None):
    """prefill() for activations in host memory: c_kv, k_rope, q, lam_logits,
    gate_logits and the returned Y are CPU tensors (page-locked ones let the
    copies overlap the kernels); gamma, w_ukv, the RoPE tables, the workspace
    and the optional decode-cache outputs are CUDA tensors. The inputs travel
    to the GPU in chunks of ``chunk_tokens`` tokens (0 = the library default)
    while earlier chunks compute. Asynchronous like every call: synchronise
    ``stream`` before reading Y."""
    B, L = c_kv.shape[:2]
    n_signal, d_v_guess = lam_logits.shape[-1], gate_logits.shape[-1]
    if out is None:
        out = torch.empty((B, L, n_signal, d_v_guess), dtype=c_kv.dtype, pin_memory=True)
    a = _prefill_args(c_kv, gamma, k_rope, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, out, g, mask,
                      window, softmax_scale, rms_eps, cache_c_hat, cache_k_rope, workspace, act_ptr=_host_ptr)
    if workspace is None:
        need = int(_lib().gdla_prefill_host_workspace_size(ctypes.byref(a), int(chunk_tokens)))
        workspace = torch.empty(need, dtype=torch.uint8, device=gamma.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), need
    _abi.check(_lib().gdla_prefill_host(ctypes.byref(a), int(chunk_tokens), _stream(stream)), "gdla_prefill_host")
    return out


def attend(q, kv, k_rope_rot, rope_cos, rope_sin, lam_logits, gate_logits, *, g: int, mask: str = "causal",
           window: int = 0, softmax_scale: float = 0.0, q_start: int = 0, out=None, status=None, stream=None):
    """Steps 3-8 over an expanded latent (the output of latent_expand); returns
    Y [B, q_len, n_signal, d_v]. The query side (q, lam_logits, gate_logits)
    holds q_len = q.shape[1] rows per sequence at positions q_start ..
    q_start + q_len - 1; kv and k_rope_rot hold all L key positions. ``status``
    is an optional 256-byte uint8 CUDA tensor that receives the device status word."""
    B, q_len, H_q, d_qk = q.shape
    L, n_kv, dkv = kv.shape[1], kv.shape[2], kv.shape[3]
    d_rope = k_rope_rot.shape[-1]
    d_nope = d_qk - d_rope
    d_v = dkv - d_nope
    if out is None:
        out = torch.empty((B, q_len, lam_logits.shape[-1], d_v), dtype=q.dtype, device=q.device)
    if status is None:
        status = torch.empty(256, dtype=torch.uint8, device=q.device)
    a = _abi.AttendArgs(B, L, d_rope, n_kv, d_nope, d_v, H_q // (g + 1), g, _mask(mask), int(window),
                        float(softmax_scale), _dtype(q), rope_cos.shape[0], _ptr(q), _ptr(kv), _ptr(k_rope_rot),
                        _ptr(rope_cos), _ptr(rope_sin), _ptr(lam_logits), _ptr(gate_logits), _ptr(out), _ptr(status),
                        status.numel(), int(q_len), int(q_start))
    _abi.check(_lib().gdla_attend(ctypes.byref(a), _stream(stream)), "gdla_attend")
    return out


# ----------------------------------------------------------------------- gates
def gates(c_q=None, gamma_q=None, w_g=None, x=None, w_lambda=None, *, n_signal: int, d_v: int = 0,
          rms_eps: float = 0.0, gate_out=None, lam_out=None, workspace=None, stream=None):
    """Gate and lambda logits from the layer's activations: gate_logits =
    RMSNorm(c_q; gamma_q) @ w_g as [*, n_signal, d_v] (dtype of c_q) and
    lam_logits = x @ w_lambda as [*, n_signal] fp32, where * is the leading
    [B, L] (or [B]) of c_q / x. Pass only (c_q, gamma_q, w_g) or only
    (x, w_lambda) to compute one of them. Returns (gate_logits, lam_logits),
    None for the half not computed."""
    if c_q is None and x is None:
        raise ValueError("gates needs c_q (gate) and/or x (lambda)")
    ref = c_q if c_q is not None else x
    lead = tuple(ref.shape[:-1])
    B, L = (lead[0], lead[1]) if len(lead) == 2 else (lead[0], 1)
    d_q = c_q.shape[-1] if c_q is not None else 0
    d_x = x.shape[-1] if x is not None else 0
    if c_q is not None:
        if d_v <= 0:
            d_v = w_g.shape[1] // n_signal
        if gate_out is None:
            gate_out = torch.empty(lead + (n_signal, d_v), dtype=c_q.dtype, device=c_q.device)
    if x is not None and lam_out is None:
        lam_out = torch.empty(lead + (n_signal,), dtype=torch.float32, device=x.device)
    a = _abi.GatesArgs(B, L, d_q, d_x, n_signal, d_v, _dtype(ref), float(rms_eps), _ptr(c_q), _ptr(gamma_q),
                       _ptr(w_g), _ptr(x), _ptr(w_lambda), _ptr(gate_out), _ptr(lam_out), None, 0)
    need = int(_lib().gdla_gates_workspace_size(ctypes.byref(a)))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=ref.device)
    a.workspace, a.workspace_bytes = _ptr(workspace), workspace.numel()
    _abi.check(_lib().gdla_gates(ctypes.byref(a), _stream(stream)), "gdla_gates")
    return (gate_out if c_q is not None else None), (lam_out if x is not None else None)


# ---------------------------------------------------------------------- decode
def _decode_args(c_cache, kr_cache, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, seqlens, out, g, mask,
                 window, softmax_scale, workspace):
    B, T_max, d_c = c_cache.shape
    d_rope = kr_cache.shape[-1]
    H_q, d_qk = q.shape[1], q.shape[2]
    if H_q % (g + 1):
        raise ValueError("q must hold g*n_noise signal heads followed by n_noise noise heads")
    n_noise = H_q // (g + 1)
    d_nope = d_qk - d_rope
    d_v = w_ukv.shape[1] // n_noise - d_nope
    if seqlens.dtype != torch.int32:
        raise ValueError("seqlens must be int32")
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return _abi.DecodeArgs(B, T_max, d_c, d_rope, n_noise, d_nope, d_v, n_noise, g, _mask(mask), int(window),
                           float(softmax_scale), _dtype(c_cache), rope_cos.shape[0], _ptr(seqlens), _ptr(c_cache),
                           _ptr(kr_cache), _ptr(q), _ptr(w_ukv), _ptr(rope_cos), _ptr(rope_sin), _ptr(lam_logits),
                           _ptr(gate_logits), _ptr(out), ws_ptr, ws_bytes)


def decode_workspace_size(*, B, T_max, d_c, d_rope, n_kv, d_nope, d_v, g, dtype=torch.bfloat16) -> int:
    a = _abi.DecodeArgs()
    a.B, a.T_max, a.d_c, a.d_rope, a.n_kv, a.d_nope, a.d_v, a.n_noise, a.g = B, T_max, d_c, d_rope, n_kv, d_nope, d_v, n_kv, g
    a.dtype = _DT[dtype]
    return int(_lib().gdla_decode_workspace_size(ctypes.byref(a)))


def decode(c_cache, kr_cache, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, seqlens, *, g: int,
           mask: str = "causal", window: int = 0, softmax_scale: float = 0.0, out=None, workspace=None, stream=None):
    """One decode step per sequence; returns Y [B, n_signal, d_v].

    c_cache [B,T_max,d_c] normalised latent, kr_cache [B,T_max,d_rope] rotated
    rotary key, q [B,n_signal+n_noise,d_nope+d_rope] (rotary part pre-RoPE, at
    position seqlens[b]-1), lam_logits [B,n_signal] fp32, gate_logits
    [B,n_signal,d_v], seqlens [B] int32 on the device."""
    B = c_cache.shape[0]
    if out is None:
        out = torch.empty((B, lam_logits.shape[-1], gate_logits.shape[-1]), dtype=c_cache.dtype,
                          device=c_cache.device)
    a = _decode_args(c_cache, kr_cache, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, seqlens, out, g,
                     mask, window, softmax_scale, workspace)
    if workspace is None:
        need = int(_lib().gdla_decode_workspace_size(ctypes.byref(a)))
        workspace = torch.empty(need, dtype=torch.uint8, device=c_cache.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), need
    _abi.check(_lib().gdla_decode(ctypes.byref(a), _stream(stream)), "gdla_decode")
    return out


def decode_noalloc(c_cache, kr_cache, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, seqlens, *, g: int,
                   mask: str = "causal", window: int = 0, softmax_scale: float = 0.0, out=None, stream=None):
    """decode() for callers that cannot provide device scratch: the library's
    own fixed 32 MiB array is used instead of a workspace (see
    gdla_decode_noalloc in include/gdla.h: calls on one device share it and
    must not overlap; the first call on a device should come before any stream
    capture). Raises GdlaError (GDLA_ERR_SCRATCH_LIMIT) for a batch too large
    for the array."""
    B = c_cache.shape[0]
    if out is None:
        out = torch.empty((B, lam_logits.shape[-1], gate_logits.shape[-1]), dtype=c_cache.dtype,
                          device=c_cache.device)
    a = _decode_args(c_cache, kr_cache, q, w_ukv, rope_cos, rope_sin, lam_logits, gate_logits, seqlens, out, g,
                     mask, window, softmax_scale, None)
    _abi.check(_lib().gdla_decode_noalloc(ctypes.byref(a), _stream(stream)), "gdla_decode_noalloc")
    return out


def diag_wait_timeout(status_word, stream=None) -> None:
    """Diagnostic: run one device wait that can never complete; it ends at its
    limit and records GDLA_ERR_TIMEOUT in ``status_word`` (a 256-byte uint8 CUDA
    tensor), readable with ``workspace_status``."""
    _abi.check(_lib().gdla_diag_wait_timeout(_ptr(status_word), _stream(stream)), "gdla_diag_wait_timeout")


def workspace_status(workspace, stream=None) -> int:
    """Device status word of the last call that used ``workspace`` (0 = OK)."""
    return int(_lib().gdla_workspace_status(_ptr(workspace), _stream(stream)))


def _mask_const(mask: str) -> int:
    return _mask(mask)


def default_scale(d_nope: int, d_rope: int) -> float:
    return 1.0 / math.sqrt(d_nope + d_rope)
