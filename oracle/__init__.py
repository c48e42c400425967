"""fp64 CPU oracle for the GDLA forward pass -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package. The product path (the CUDA
library under ``differential_latent_attention_gdla_b200``) never does; the two
share no code, header, table or helper. The arithmetic lives in
``gdla_oracle.c`` (plain loops in double precision, one function per step of
the layer as stated in "Motif 3: Technical Report", section "Architecture");
this module only marshals numpy float64 arrays into it.

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, invariants, brute force and independent numpy formulations.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdla_oracle.c")
_LIB = os.path.join(_HERE, "libgdla_oracle.so")
_lock = threading.Lock()
_lib = None

MASK_CAUSAL = 0
MASK_SLIDING = 1
DEFAULT_EPS = 1e-6
DEFAULT_ROPE_BASE = 10000.0

_dp = ctypes.POINTER(ctypes.c_double)
_lp = ctypes.POINTER(ctypes.c_long)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile gdla_oracle.c into libgdla_oracle.so (gcc, OpenMP) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            lib.gdla_oracle_num_threads.restype = ctypes.c_int
            lib.gdla_oracle_latent_norm.argtypes = [_dp, _dp, ctypes.c_long, ctypes.c_int, ctypes.c_double, _dp]
            lib.gdla_oracle_project.argtypes = [_dp, ctypes.c_long, ctypes.c_int, _dp, ctypes.c_int, _dp]
            lib.gdla_oracle_expand_head.argtypes = [_dp, _dp, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp]
            lib.gdla_oracle_rope.argtypes = [_dp, ctypes.c_long, ctypes.c_int, ctypes.c_double, _dp]
            lib.gdla_oracle_rope_table.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_double, _dp, _dp]
            lib.gdla_oracle_yarn_inv_freq.argtypes = [ctypes.c_int] + [ctypes.c_double] * 5 + [_dp]
            lib.gdla_oracle_attend_row.argtypes = [_dp, _dp, _dp, ctypes.c_long, _dp, ctypes.c_long, _dp,
                                                   ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_long, ctypes.c_int, ctypes.c_long, ctypes.c_double,
                                                   _dp, _dp]
            lib.gdla_oracle_differential_gate.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                                          ctypes.c_int, _dp]
            lib.gdla_oracle_prefill_rows.restype = ctypes.c_int
            lib.gdla_oracle_prefill_rows.argtypes = (
                [ctypes.c_int, ctypes.c_long] + [ctypes.c_int] * 6 + [ctypes.c_int, ctypes.c_long]
                + [ctypes.c_double] * 3 + [_dp] * 5 + [ctypes.c_long, _lp, _lp] + [_dp] * 3 + [_ip] + [_dp] * 2)
            lib.gdla_oracle_decode_seq.restype = ctypes.c_int
            lib.gdla_oracle_decode_seq.argtypes = (
                [ctypes.c_long] + [ctypes.c_int] * 6 + [ctypes.c_int, ctypes.c_long, ctypes.c_double,
                                                       ctypes.c_double] + [_dp] * 7 + [_ip, _dp, _dp])
            _lib = lib
    return _lib


def _d(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().gdla_oracle_num_threads())


def default_scale(d_n: int, d_R: int) -> float:
    """1/sqrt(d_qk), the scaled dot-product factor with d_qk = d_n + d_R."""
    return 1.0 / np.sqrt(d_n + d_R)


# ---------------------------------------------------------------------------- steps
def latent_norm(c, gamma, eps: float = DEFAULT_EPS) -> np.ndarray:
    """Step 1: RMS normalisation of the latent rows of ``c`` [T, d_c]."""
    c = _d(c)
    gamma = _d(gamma)
    T, d_c = c.shape
    out = np.empty_like(c)
    _load().gdla_oracle_latent_norm(_p(c), _p(gamma), T, d_c, eps, _p(out))
    return out


def project(a, w) -> np.ndarray:
    """out [T, N] = a [T, K] @ w [K, N], summed in increasing k (plain loops)."""
    a = _d(a)
    w = _d(w)
    T, K = a.shape
    N = w.shape[1]
    out = np.empty((T, N))
    _load().gdla_oracle_project(_p(a), T, K, _p(w), N, _p(out))
    return out


def gate_logits(c_q, gamma_q, w_g, eps: float = DEFAULT_EPS) -> np.ndarray:
    """Gate logits G [T, n_S * d_v] from the query latent c_q [T, d_q]: the latent is
    RMS-normalised (the same normalisation as step 1, with its own gain gamma_q) and
    projected by W_G [d_q, n_S * d_v] ("Motif 3: Technical Report", section
    "Architecture": the gate is computed from the normalised query latent)."""
    return project(latent_norm(c_q, gamma_q, eps), w_g)


def lambda_logits(x, w_lam) -> np.ndarray:
    """lambda logits [T, n_S] = x [T, d_x] @ W_lambda [d_x, n_S] ("Motif 3: Technical
    Report", section "Architecture": lambda_t = sigmoid(x_t W_lambda))."""
    return project(x, w_lam)


def expand_head(c_hat, w_ukv, n_kv: int, d_n: int, d_v: int, h: int):
    """Step 2 for KV head ``h``: returns (k_nope [T, d_n], v [T, d_v])."""
    c_hat = _d(c_hat)
    w_ukv = _d(w_ukv)
    T, d_c = c_hat.shape
    k = np.empty((T, d_n))
    v = np.empty((T, d_v))
    _load().gdla_oracle_expand_head(_p(c_hat), _p(w_ukv), T, d_c, n_kv, d_n, d_v, h, _p(k), _p(v))
    return k, v


def rope(x, pos: int, base: float = DEFAULT_ROPE_BASE) -> np.ndarray:
    """Step 3: rotate-half RoPE of one vector ``x`` [d_R] at position ``pos``."""
    x = _d(x)
    y = np.empty_like(x)
    _load().gdla_oracle_rope(_p(x), int(pos), x.shape[0], base, _p(y))
    return y


def rope_table(max_pos: int, d_R: int, base: float = DEFAULT_ROPE_BASE):
    """The oracle's own fp64 cos/sin table, [max_pos, d_R/2] each."""
    c = np.empty((max_pos, d_R // 2))
    s = np.empty((max_pos, d_R // 2))
    _load().gdla_oracle_rope_table(max_pos, d_R, base, _p(c), _p(s))
    return c, s


def rope_freqs(d_R: int, base: float = DEFAULT_ROPE_BASE) -> np.ndarray:
    """The plain RoPE frequencies theta_k = base^(-2k/d_R), k < d_R/2 (fp64)."""
    return base ** (-2.0 * np.arange(d_R // 2) / d_R)


def yarn_inv_freq(d_R: int, factor: float, original_max_pos: float, base: float = DEFAULT_ROPE_BASE,
                  beta_fast: float = 32.0, beta_slow: float = 1.0) -> np.ndarray:
    """RoPE frequencies rescaled by YaRN ("Open-Source Frontier Models: Architecture and Benchmarks of Rnj-1 and Motif-2",
    section 2, the Scale(i) equation): kept where the wavelength is below original_max_pos/beta_fast,
    divided by ``factor`` above original_max_pos/beta_slow, blended linearly in the
    wavelength in between (computed by the C oracle)."""
    out = np.empty(d_R // 2)
    _load().gdla_oracle_yarn_inv_freq(d_R, base, factor, original_max_pos, beta_fast, beta_slow, _p(out))
    return out


def yarn_mscale(factor: float) -> float:
    """YaRN's attention temperature: the factor 1 + 0.1 ln(s) by which the pages'
    listing scales both rotated vectors, i.e. a factor m^2 on the logits (1 for
    s <= 1). The pages' prose gives sqrt(1 + 0.1 ln s) instead; the listing's
    value is the one used here (a reading)."""
    return 1.0 + 0.1 * math.log(factor) if factor > 1.0 else 1.0


def rope_table_freq(max_pos: int, inv_freq) -> tuple[np.ndarray, np.ndarray]:
    """cos/sin tables [max_pos, d_R/2] for explicit frequencies (fp64)."""
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * _d(inv_freq)[None, :]
    return np.cos(ang), np.sin(ang)


def attend_row(q_n, q_r_rot, k_n, k_r_rot, v, i: int, mask: int = MASK_CAUSAL, window: int = 0,
               scale: float | None = None, want_p: bool = False):
    """Steps 4-6 for one query row ``i`` of one head over keys/values [T, *].

    ``q_r_rot`` and ``k_r_rot`` are already rotated. Returns H [d_v], and the
    probabilities [i+1] when ``want_p``.
    """
    q_n, q_r_rot, k_n, k_r_rot, v = map(_d, (q_n, q_r_rot, k_n, k_r_rot, v))
    d_n, d_R, d_v = q_n.shape[0], q_r_rot.shape[0], v.shape[1]
    if scale is None:
        scale = default_scale(d_n, d_R)
    h = np.empty(d_v)
    p = np.empty(i + 1) if want_p else None
    _load().gdla_oracle_attend_row(_p(q_n), _p(q_r_rot), _p(k_n), d_n, _p(k_r_rot), d_R, _p(v), d_v,
                                   d_n, d_R, d_v, i, mask, window, scale, _p(h),
                                   _p(p) if want_p else None)
    return (h, p) if want_p else h


def differential_gate(h_s, h_n, lam_logits, gate_logits, g: int) -> np.ndarray:
    """Steps 7-8 for one token: h_s [n_S, d_v], h_n [n_N, d_v] -> Y [n_S, d_v]."""
    h_s, h_n, lam, gate = map(_d, (h_s, h_n, lam_logits, gate_logits))
    n_S, d_v = h_s.shape
    y = np.empty_like(h_s)
    _load().gdla_oracle_differential_gate(_p(h_s), _p(h_n), _p(lam), _p(gate), n_S, g, d_v, _p(y))
    return y


# ------------------------------------------------------------------------- composites
def prefill_rows(*, c_kv, gamma, k_rope, w_ukv, q_rows, lam_rows, gate_rows, row_b, row_i, g: int,
                 d_n: int, d_v: int, mask: int = MASK_CAUSAL, window: int = 0, scale: float | None = None,
                 eps: float = DEFAULT_EPS, rope_base: float = DEFAULT_ROPE_BASE, want_heads: bool = False,
                 kv_sel=None, inv_freq=None):
    """Output rows Y [nrows, n_S, d_v] of the prefill for query tokens (row_b, row_i).
    With ``kv_sel`` (a list of KV group indices) only those groups are computed
    and the other groups' rows are NaN. ``inv_freq`` [d_R/2] replaces the RoPE
    frequencies rope_base^(-2k/d_R) (e.g. with ``yarn_inv_freq``).

    c_kv [B, L, d_c], k_rope [B, L, d_R], w_ukv [d_c, n_kv*(d_n+d_v)], gamma [d_c]
    cover the whole batch; q_rows [nrows, n_S+n_N, d_n+d_R], lam_rows
    [nrows, n_S] and gate_rows [nrows, n_S, d_v] only the selected rows.
    """
    c_kv, gamma, k_rope, w_ukv = map(_d, (c_kv, gamma, k_rope, w_ukv))
    q_rows, lam_rows, gate_rows = map(_d, (q_rows, lam_rows, gate_rows))
    B, L, d_c = c_kv.shape
    d_R = k_rope.shape[2]
    n_kv = w_ukv.shape[1] // (d_n + d_v)
    n_S = g * n_kv
    H_q = n_S + n_kv
    nrows = len(row_b)
    assert q_rows.shape == (nrows, H_q, d_n + d_R), q_rows.shape
    assert lam_rows.shape == (nrows, n_S) and gate_rows.shape == (nrows, n_S, d_v)
    if scale is None:
        scale = default_scale(d_n, d_R)
    rb = np.ascontiguousarray(row_b, dtype=np.int64)
    ri = np.ascontiguousarray(row_i, dtype=np.int64)
    y = np.empty((nrows, n_S, d_v))
    heads = np.empty((nrows, H_q, d_v)) if want_heads else None
    sel = None
    if kv_sel is not None:
        sel = np.zeros(n_kv, dtype=np.int32)
        sel[np.asarray(kv_sel, dtype=np.int64)] = 1
    inv = None if inv_freq is None else _d(inv_freq)
    assert inv is None or inv.shape == (d_R // 2,)
    rc = _load().gdla_oracle_prefill_rows(
        B, L, d_c, d_R, n_kv, d_n, d_v, g, mask, window, scale, eps, rope_base, _p(inv) if inv is not None else None,
        _p(c_kv), _p(gamma), _p(k_rope), _p(w_ukv), nrows, rb.ctypes.data_as(_lp), ri.ctypes.data_as(_lp),
        _p(q_rows), _p(lam_rows), _p(gate_rows), sel.ctypes.data_as(_ip) if sel is not None else None, _p(y),
        _p(heads) if want_heads else None)
    if rc != 0:
        raise ValueError("oracle prefill_rows rejected its arguments")
    if sel is not None:
        for h in range(n_kv):
            if not sel[h]:
                y[:, h * g:(h + 1) * g] = np.nan
    return (y, heads) if want_heads else y


def decode_seq(*, c_hat, k_r_rot, q, w_ukv, lam, gate, g: int, d_n: int, d_v: int, mask: int = MASK_CAUSAL,
               window: int = 0, scale: float | None = None, rope_base: float = DEFAULT_ROPE_BASE,
               kv_sel=None, want_heads: bool = False, inv_freq=None):
    """Decode of one token at position T-1 over one sequence's latent cache.

    c_hat [T, d_c] (normalised latent), k_r_rot [T, d_R] (rotated key),
    q [n_S+n_N, d_n+d_R] (rotary part pre-RoPE), lam [n_S], gate [n_S, d_v].
    Returns Y [n_S, d_v]; rows of KV groups excluded by ``kv_sel`` are NaN.
    ``inv_freq`` [d_R/2] replaces the RoPE frequencies of the query rotation.
    """
    c_hat, k_r_rot, q, w_ukv, lam, gate = map(_d, (c_hat, k_r_rot, q, w_ukv, lam, gate))
    T, d_c = c_hat.shape
    d_R = k_r_rot.shape[1]
    n_kv = w_ukv.shape[1] // (d_n + d_v)
    n_S = g * n_kv
    if scale is None:
        scale = default_scale(d_n, d_R)
    y = np.full((n_S, d_v), np.nan)
    heads = np.full((n_S + n_kv, d_v), np.nan) if want_heads else None
    sel = None
    if kv_sel is not None:
        sel = np.zeros(n_kv, dtype=np.int32)
        sel[np.asarray(kv_sel, dtype=np.int64)] = 1
    inv = None if inv_freq is None else _d(inv_freq)
    assert inv is None or inv.shape == (d_R // 2,)
    rc = _load().gdla_oracle_decode_seq(
        T, d_c, d_R, n_kv, d_n, d_v, g, mask, window, scale, rope_base, _p(inv) if inv is not None else None,
        _p(c_hat), _p(k_r_rot), _p(q),
        _p(w_ukv), _p(lam), _p(gate), sel.ctypes.data_as(_ip) if sel is not None else None, _p(y),
        _p(heads) if want_heads else None)
    if rc != 0:
        raise ValueError("oracle decode_seq rejected its arguments")
    return (y, heads) if want_heads else y
