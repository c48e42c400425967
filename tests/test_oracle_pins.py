"""Pins for the fp64 oracle (CPU only).

Each test ties one step of the oracle to something other than itself: a closed
form, an invariant of attention or of the rotation, brute force against an
independent numpy matrix formulation, or a special case that reduces to a
textbook routine. The steps follow "Motif 3: Technical Report", section
"Architecture" (GDLA), and the attention/RoPE/sliding-window definitions of
"Open-Source Frontier Models: Architecture and Benchmarks of Rnj-1 and
Motif-2", sections 1 and 2.
"""
import math

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(1234)


# ------------------------------------------------------------------ independent forms
def np_rope_complex(x, pos, base=10000.0, theta=None):
    """RoPE as multiplication of (x_k + i x_{k+d/2}) by exp(i pos theta_k)."""
    d = x.shape[-1]
    h = d // 2
    if theta is None:
        theta = base ** (-2.0 * np.arange(h) / d)
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * pos * theta)
    return np.concatenate([z.real, z.imag], axis=-1)


def np_attention_matrix(Q, K, V, scale, mask, window):
    """softmax(scale * Q K^T + M) V with an additive -inf mask, all rows."""
    T = Q.shape[0]
    S = scale * (Q @ K.T)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = j <= i
    if mask == oracle.MASK_SLIDING:
        vis &= j > i - window
    S = np.where(vis, S, -np.inf)
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(axis=1, keepdims=True)
    return P @ V, P


def np_gdla_prefill(c, gamma, k_rope, q, w, lam, gate, g, d_n, d_v, mask, window, eps=1e-6, base=10000.0,
                    theta=None, scale=None):
    """The whole layer in numpy matrix form (one sequence): normalise, expand,
    rotate (complex form), attend per head, differential, gate."""
    L, d_c = c.shape
    d_R = k_rope.shape[1]
    n_kv = w.shape[1] // (d_n + d_v)
    n_S = g * n_kv
    chat = gamma * c / np.sqrt((c * c).mean(axis=1, keepdims=True) + eps)
    KV = (chat @ w).reshape(L, n_kv, d_n + d_v)
    pos = np.arange(L)[:, None]
    kr = np_rope_complex(k_rope, pos, base, theta)
    H = np.zeros((L, n_S + n_kv, d_v))
    if scale is None:
        scale = 1.0 / math.sqrt(d_n + d_R)
    for head in range(n_S + n_kv):
        kvh = head // g if head < n_S else head - n_S
        qn = q[:, head, :d_n]
        qr = np_rope_complex(q[:, head, d_n:], pos, base, theta)
        Qf = np.concatenate([qn, qr], axis=1)
        Kf = np.concatenate([KV[:, kvh, :d_n], kr], axis=1)
        H[:, head], _ = np_attention_matrix(Qf, Kf, KV[:, kvh, d_n:], scale, mask, window)
    lam_s = 1.0 / (1.0 + np.exp(-lam))
    HN_rep = np.repeat(H[:, n_S:], g, axis=1)
    D = H[:, :n_S] - lam_s[:, :, None] * HN_rep
    return D / (1.0 + np.exp(-gate)), H


def tiny_inputs(B=2, L=11, d_c=8, d_R=4, n_kv=2, d_n=6, d_v=5, g=3, rng=RNG):
    n_S = g * n_kv
    return dict(
        c_kv=rng.standard_normal((B, L, d_c)),
        gamma=1 + 0.1 * rng.standard_normal(d_c),
        k_rope=rng.standard_normal((B, L, d_R)),
        w_ukv=rng.standard_normal((d_c, n_kv * (d_n + d_v))) / math.sqrt(d_c),
        q=rng.standard_normal((B, L, n_S + n_kv, d_n + d_R)),
        lam=rng.standard_normal((B, L, n_S)),
        gate=rng.standard_normal((B, L, n_S, d_v)),
        g=g, d_n=d_n, d_v=d_v,
    )


def run_all_rows(inp, mask=oracle.MASK_CAUSAL, window=0, want_heads=False, **kw):
    B, L = inp["c_kv"].shape[:2]
    rb, ri = np.meshgrid(np.arange(B), np.arange(L), indexing="ij")
    rb, ri = rb.ravel(), ri.ravel()
    res = oracle.prefill_rows(
        c_kv=inp["c_kv"], gamma=inp["gamma"], k_rope=inp["k_rope"], w_ukv=inp["w_ukv"],
        q_rows=inp["q"][rb, ri], lam_rows=inp["lam"][rb, ri], gate_rows=inp["gate"][rb, ri],
        row_b=rb, row_i=ri, g=inp["g"], d_n=inp["d_n"], d_v=inp["d_v"], mask=mask, window=window,
        want_heads=want_heads, **kw)
    if want_heads:
        y, h = res
        return y.reshape(B, L, *y.shape[1:]), h.reshape(B, L, *h.shape[1:])
    return res.reshape(B, L, *res.shape[1:])


# ------------------------------------------------------------------- step 1: RMSNorm
def test_latent_norm_constant_row_closed_form():
    d_c = 16
    gamma = 1 + 0.1 * RNG.standard_normal(d_c)
    for a in (3.0, -0.25):
        c = np.full((1, d_c), a)
        eps = 1e-6
        out = oracle.latent_norm(c, gamma, eps)
        np.testing.assert_allclose(out[0], gamma * a / math.sqrt(a * a + eps), rtol=1e-14)


def test_latent_norm_one_hot_closed_form():
    d_c = 32
    gamma = np.arange(1, d_c + 1, dtype=float)
    c = np.zeros((1, d_c))
    c[0, 5] = 2.0
    out = oracle.latent_norm(c, gamma, 0.0)
    expect = np.zeros(d_c)
    expect[5] = gamma[5] * 2.0 / math.sqrt(4.0 / d_c)
    np.testing.assert_allclose(out[0], expect, rtol=1e-14, atol=0)


def test_latent_norm_scale_invariant():
    c = RNG.standard_normal((7, 24))
    gamma = 1 + 0.1 * RNG.standard_normal(24)
    a = oracle.latent_norm(c, gamma, 0.0)
    b = oracle.latent_norm(17.5 * c, gamma, 0.0)
    np.testing.assert_allclose(a, b, rtol=1e-13)
    # unit RMS after normalisation when gamma = 1
    u = oracle.latent_norm(c, np.ones(24), 0.0)
    np.testing.assert_allclose(np.sqrt((u * u).mean(axis=1)), 1.0, rtol=1e-13)


# ---------------------------------------------------------------- step 2: expansion
def test_expand_head_matches_numpy_matmul():
    T, d_c, n_kv, d_n, d_v = 9, 12, 3, 5, 4
    c = RNG.standard_normal((T, d_c))
    w = RNG.standard_normal((d_c, n_kv * (d_n + d_v)))
    full = c @ w
    for h in range(n_kv):
        k, v = oracle.expand_head(c, w, n_kv, d_n, d_v, h)
        col = h * (d_n + d_v)
        np.testing.assert_allclose(k, full[:, col:col + d_n], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(v, full[:, col + d_n:col + d_n + d_v], rtol=1e-12, atol=1e-12)


# -------------------------------------------------------------------- step 3: RoPE
def test_rope_closed_form_two_dims():
    # d_R = 2: theta_0 = 1, so e_0 rotates to (cos m, sin m) and e_1 to (-sin m, cos m)
    for m in (0, 1, 5, 1000):
        np.testing.assert_allclose(oracle.rope(np.array([1.0, 0.0]), m), [math.cos(m), math.sin(m)], atol=1e-15)
        np.testing.assert_allclose(oracle.rope(np.array([0.0, 1.0]), m), [-math.sin(m), math.cos(m)], atol=1e-15)


def test_rope_closed_form_second_frequency():
    # d_R = 4, base 100: theta_1 = 100^(-2/4) = 0.1; pair (1, 3)
    x = np.array([0.0, 1.0, 0.0, 0.0])
    m = 7
    y = oracle.rope(x, m, base=100.0)
    np.testing.assert_allclose(y, [0.0, math.cos(0.7), 0.0, math.sin(0.7)], atol=1e-15)


def test_rope_matches_complex_form():
    for d_R in (4, 16, 64):
        x = RNG.standard_normal(d_R)
        for m in (0, 3, 4095, 65535):
            # both sides round the angle m*theta in double: error grows like m * ulp
            tol = 1e-13 + 2e-15 * m * np.abs(x).max()
            np.testing.assert_allclose(oracle.rope(x, m), np_rope_complex(x, m), rtol=0, atol=tol)


def test_rope_norm_relative_position_identity():
    d_R = 64
    q = RNG.standard_normal(d_R)
    k = RNG.standard_normal(d_R)
    np.testing.assert_allclose(oracle.rope(q, 0), q, rtol=0, atol=0)
    for m in (1, 100, 32767):
        assert abs(np.linalg.norm(oracle.rope(q, m)) - np.linalg.norm(q)) < 1e-12
    for m, n in ((10, 3), (500, 499), (4000, 17)):
        base_dot = oracle.rope(q, m) @ oracle.rope(k, n)
        for s in (1, 37, 20000):
            assert abs(oracle.rope(q, m + s) @ oracle.rope(k, n + s) - base_dot) < 1e-9


def test_rope_table_consistent_with_rotation():
    d_R, P = 16, 50
    c, s = oracle.rope_table(P, d_R)
    for p in (0, 1, 49):
        for k in range(d_R // 2):
            e = np.zeros(d_R)
            e[k] = 1.0
            y = oracle.rope(e, p)
            assert abs(y[k] - c[p, k]) < 1e-14 and abs(y[k + d_R // 2] - s[p, k]) < 1e-14


# ------------------------------------------------------------ steps 4-6: attention
@pytest.mark.parametrize("mask,window", [(oracle.MASK_CAUSAL, 0), (oracle.MASK_SLIDING, 4), (oracle.MASK_SLIDING, 1)])
def test_attend_row_brute_force_vs_matrix_form(mask, window):
    T, d_n, d_R, d_v = 13, 6, 4, 5
    qn, kn = RNG.standard_normal((T, d_n)), RNG.standard_normal((T, d_n))
    qr, kr = RNG.standard_normal((T, d_R)), RNG.standard_normal((T, d_R))
    v = RNG.standard_normal((T, d_v))
    scale = 0.37
    Hm, Pm = np_attention_matrix(np.hstack([qn, qr]), np.hstack([kn, kr]), v, scale, mask, window)
    for i in range(T):
        h, p = oracle.attend_row(qn[i], qr[i], kn, kr, v, i, mask, window, scale, want_p=True)
        np.testing.assert_allclose(h, Hm[i], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(p, Pm[i, :i + 1], rtol=1e-12, atol=1e-15)
        assert abs(p.sum() - 1.0) < 1e-12


def test_attend_row_zero_query_is_mean_of_visible_values():
    T, d_v = 20, 3
    kn, kr, v = RNG.standard_normal((T, 4)), RNG.standard_normal((T, 2)), RNG.standard_normal((T, d_v))
    for i in (0, 7, 19):
        h = oracle.attend_row(np.zeros(4), np.zeros(2), kn, kr, v, i)
        np.testing.assert_allclose(h, v[:i + 1].mean(axis=0), rtol=1e-13)
        h = oracle.attend_row(np.zeros(4), np.zeros(2), kn, kr, v, i, oracle.MASK_SLIDING, 5)
        np.testing.assert_allclose(h, v[max(0, i - 4):i + 1].mean(axis=0), rtol=1e-13)


def test_attend_row_window_one_returns_own_value():
    T = 9
    kn, kr, v = RNG.standard_normal((T, 4)), RNG.standard_normal((T, 2)), RNG.standard_normal((T, 3))
    for i in range(T):
        h = oracle.attend_row(RNG.standard_normal(4), RNG.standard_normal(2), kn, kr, v, i, oracle.MASK_SLIDING, 1)
        np.testing.assert_array_equal(h, v[i])


def test_attend_row_wide_window_equals_causal_bitwise():
    T = 17
    kn, kr, v = RNG.standard_normal((T, 4)), RNG.standard_normal((T, 2)), RNG.standard_normal((T, 3))
    qn, qr = RNG.standard_normal(4), RNG.standard_normal(2)
    for i in (0, 5, 16):
        a = oracle.attend_row(qn, qr, kn, kr, v, i)
        for W in (i + 1, T, 10 * T):
            np.testing.assert_array_equal(oracle.attend_row(qn, qr, kn, kr, v, i, oracle.MASK_SLIDING, W), a)


def test_attend_row_sliding_is_causal_over_window_subsequence():
    T, W = 30, 6
    kn, kr, v = RNG.standard_normal((T, 4)), RNG.standard_normal((T, 2)), RNG.standard_normal((T, 3))
    qn, qr = RNG.standard_normal(4), RNG.standard_normal(2)
    for i in (W - 1, W, 29):
        lo = i - W + 1
        a = oracle.attend_row(qn, qr, kn, kr, v, i, oracle.MASK_SLIDING, W)
        b = oracle.attend_row(qn, qr, kn[lo:], kr[lo:], v[lo:], i - lo)
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


def test_attend_row_softmax_shift_invariant_and_peaked():
    T = 8
    kn = np.eye(T, 8)
    kr = np.zeros((T, 2))
    v = RNG.standard_normal((T, 3))
    # a query aligned with key 3 and a huge scale puts all weight on token 3
    qn = np.zeros(8)
    qn[3] = 1.0
    h = oracle.attend_row(qn, np.zeros(2), kn, kr, v, 7, scale=1e4)
    np.testing.assert_allclose(h, v[3], rtol=1e-12)


# --------------------------------------------------------- steps 7-8: differential
def test_differential_gate_closed_form_and_head_mapping():
    g, n_N, d_v = 3, 2, 4
    n_S = g * n_N
    h_s = np.zeros((n_S, d_v))
    h_n = np.array([[1.0, 2.0, 3.0, 4.0], [10.0, 20.0, 30.0, 40.0]])
    y = oracle.differential_gate(h_s, h_n, np.zeros(n_S), np.zeros((n_S, d_v)), g)
    # sigmoid(0) = 1/2 for both lambda and the gate: Y_i = -1/4 * H_N[floor(i/g)]
    for i in range(n_S):
        np.testing.assert_allclose(y[i], -0.25 * h_n[i // g], rtol=1e-15)
    h_s = RNG.standard_normal((n_S, d_v))
    lam = RNG.standard_normal(n_S)
    y = oracle.differential_gate(h_s, h_n, lam, np.full((n_S, d_v), 1e4), g)  # gate -> 1
    for i in range(n_S):
        np.testing.assert_allclose(y[i], h_s[i] - h_n[i // g] / (1 + math.exp(-lam[i])), rtol=1e-13)


# ------------------------------------------------------------------ whole prefill
@pytest.mark.parametrize("mask,window", [(oracle.MASK_CAUSAL, 0), (oracle.MASK_SLIDING, 3)])
def test_prefill_matches_numpy_matrix_form(mask, window):
    inp = tiny_inputs()
    y, heads = run_all_rows(inp, mask, window, want_heads=True)
    for b in range(inp["c_kv"].shape[0]):
        ey, eh = np_gdla_prefill(inp["c_kv"][b], inp["gamma"], inp["k_rope"][b], inp["q"][b], inp["w_ukv"],
                                 inp["lam"][b], inp["gate"][b], inp["g"], inp["d_n"], inp["d_v"], mask, window)
        np.testing.assert_allclose(heads[b], eh, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(y[b], ey, rtol=1e-11, atol=1e-12)


def test_prefill_lambda_zero_is_gated_latent_attention():
    inp = tiny_inputs()
    inp["lam"][:] = -1e4  # sigmoid = 0 exactly in double
    y, heads = run_all_rows(inp, want_heads=True)
    n_S = inp["g"] * (inp["w_ukv"].shape[1] // (inp["d_n"] + inp["d_v"]))
    gate = 1 / (1 + np.exp(-inp["gate"]))
    np.testing.assert_allclose(y, gate * heads[:, :, :n_S], rtol=1e-14, atol=0)
    # and the noise queries then have no influence at all
    inp2 = dict(inp)
    inp2["q"] = inp["q"].copy()
    inp2["q"][:, :, n_S:] = RNG.standard_normal(inp2["q"][:, :, n_S:].shape)
    np.testing.assert_array_equal(run_all_rows(inp2), y)


def test_prefill_identical_queries_lambda_one_cancel_exactly():
    inp = tiny_inputs()
    g = inp["g"]
    n_kv = inp["w_ukv"].shape[1] // (inp["d_n"] + inp["d_v"])
    n_S = g * n_kv
    for i in range(n_S):
        inp["q"][:, :, i] = inp["q"][:, :, n_S + i // g]
    inp["lam"][:] = 1e4  # sigmoid = 1 exactly in double
    y = run_all_rows(inp)
    np.testing.assert_array_equal(y, 0.0)


def test_prefill_wide_window_equals_causal_bitwise():
    inp = tiny_inputs()
    L = inp["c_kv"].shape[1]
    a = run_all_rows(inp)
    for W in (L, L + 5):
        np.testing.assert_array_equal(run_all_rows(inp, oracle.MASK_SLIDING, W), a)


def test_prefill_window_one_returns_expanded_value():
    inp = tiny_inputs()
    y, heads = run_all_rows(inp, oracle.MASK_SLIDING, 1, want_heads=True)
    d_n, d_v, g = inp["d_n"], inp["d_v"], inp["g"]
    n_kv = inp["w_ukv"].shape[1] // (d_n + d_v)
    for b in range(inp["c_kv"].shape[0]):
        c = inp["c_kv"][b]
        chat = inp["gamma"] * c / np.sqrt((c * c).mean(axis=1, keepdims=True) + 1e-6)
        kv = (chat @ inp["w_ukv"]).reshape(c.shape[0], n_kv, d_n + d_v)
        for head in range(heads.shape[2]):
            kvh = head // g if head < g * n_kv else head - g * n_kv
            np.testing.assert_allclose(heads[b, :, head], kv[:, kvh, d_n:], rtol=1e-12, atol=1e-13)


def test_prefill_head_permutation_equivariance():
    """Permuting KV heads together with their noise head and their g signal
    heads permutes the output the same way (pins signal head i -> group i//g)."""
    inp = tiny_inputs(n_kv=3, g=2)
    g, d_n, d_v = inp["g"], inp["d_n"], inp["d_v"]
    n_kv = 3
    n_S = g * n_kv
    perm = np.array([2, 0, 1])
    y = run_all_rows(inp)
    p = dict(inp)
    w = inp["w_ukv"].reshape(-1, n_kv, d_n + d_v)[:, perm].reshape(inp["w_ukv"].shape)
    sig = np.concatenate([np.arange(h * g, h * g + g) for h in perm])
    p["w_ukv"] = w
    p["q"] = np.concatenate([inp["q"][:, :, sig], inp["q"][:, :, n_S + perm]], axis=2)
    p["lam"] = inp["lam"][:, :, sig]
    p["gate"] = inp["gate"][:, :, sig]
    np.testing.assert_allclose(run_all_rows(p), y[:, :, sig], rtol=1e-13, atol=1e-14)


def test_prefill_alternative_head_mapping_is_rejected():
    """A mapping i -> i mod n_N would give a different result; the oracle's must
    agree with the repeat-interleave form only."""
    inp = tiny_inputs(n_kv=2, g=2)
    y = run_all_rows(inp)
    ey, _ = np_gdla_prefill(inp["c_kv"][0], inp["gamma"], inp["k_rope"][0], inp["q"][0], inp["w_ukv"],
                            inp["lam"][0], inp["gate"][0], 2, inp["d_n"], inp["d_v"], oracle.MASK_CAUSAL, 0)
    np.testing.assert_allclose(y[0], ey, rtol=1e-11, atol=1e-12)
    # the tiled reading differs on this input
    assert not np.allclose(y[0][:, 1], y[0][:, 2])


def test_prefill_batches_independent_and_scale_invariant():
    inp = tiny_inputs()
    y = run_all_rows(inp, eps=0.0)
    p = dict(inp)
    p["c_kv"] = inp["c_kv"].copy()
    p["c_kv"][0] *= 5.0  # the latent is normalised: with eps = 0 a positive scale is invisible
    p["c_kv"][1] = RNG.standard_normal(p["c_kv"][1].shape)  # batch 1 changed
    y2 = run_all_rows(p, eps=0.0)
    np.testing.assert_allclose(y2[0], y[0], rtol=1e-12, atol=1e-14)
    assert not np.allclose(y2[1], y[1])


def test_prefill_row_subset_equals_full():
    inp = tiny_inputs()
    full = run_all_rows(inp, oracle.MASK_SLIDING, 4)
    rb, ri = np.array([1, 0, 1]), np.array([10, 3, 0])
    sub = oracle.prefill_rows(c_kv=inp["c_kv"], gamma=inp["gamma"], k_rope=inp["k_rope"], w_ukv=inp["w_ukv"],
                              q_rows=inp["q"][rb, ri], lam_rows=inp["lam"][rb, ri], gate_rows=inp["gate"][rb, ri],
                              row_b=rb, row_i=ri, g=inp["g"], d_n=inp["d_n"], d_v=inp["d_v"],
                              mask=oracle.MASK_SLIDING, window=4)
    np.testing.assert_array_equal(sub, full[rb, ri])


# ----------------------------------------------------------------------- decode
def test_decode_equals_last_prefill_row():
    """Decode over the cache (normalised latent, rotated key) a prefill of
    length T leaves equals that prefill's row T-1, causal and sliding."""
    inp = tiny_inputs(B=1, L=12)
    d_n, d_v, g = inp["d_n"], inp["d_v"], inp["g"]
    for mask, window in ((oracle.MASK_CAUSAL, 0), (oracle.MASK_SLIDING, 5)):
        y = run_all_rows(inp, mask, window)
        for T in (1, 6, 12):
            c = inp["c_kv"][0, :T]
            chat = oracle.latent_norm(c, inp["gamma"], oracle.DEFAULT_EPS)
            krr = np.stack([oracle.rope(inp["k_rope"][0, j], j) for j in range(T)])
            yd = oracle.decode_seq(c_hat=chat, k_r_rot=krr, q=inp["q"][0, T - 1], w_ukv=inp["w_ukv"],
                                   lam=inp["lam"][0, T - 1], gate=inp["gate"][0, T - 1], g=g, d_n=d_n, d_v=d_v,
                                   mask=mask, window=window)
            np.testing.assert_allclose(yd, y[0, T - 1], rtol=1e-12, atol=1e-13)


def test_decode_group_selection():
    inp = tiny_inputs(B=1, L=7, n_kv=3, g=2)
    d_n, d_v, g = inp["d_n"], inp["d_v"], inp["g"]
    chat = RNG.standard_normal((7, inp["c_kv"].shape[2]))
    krr = RNG.standard_normal((7, inp["k_rope"].shape[2]))
    kw = dict(c_hat=chat, k_r_rot=krr, q=inp["q"][0, 6], w_ukv=inp["w_ukv"], lam=inp["lam"][0, 6],
              gate=inp["gate"][0, 6], g=g, d_n=d_n, d_v=d_v)
    full = oracle.decode_seq(**kw)
    part = oracle.decode_seq(kv_sel=[1], **kw)
    np.testing.assert_array_equal(part[2:4], full[2:4])
    assert np.isnan(part[:2]).all() and np.isnan(part[4:]).all()


def test_prefill_group_selection_matches_full():
    inp = tiny_inputs(n_kv=3, g=2)
    full = run_all_rows(inp)
    B, L = inp["c_kv"].shape[:2]
    rb, ri = np.meshgrid(np.arange(B), np.arange(L), indexing="ij")
    rb, ri = rb.ravel(), ri.ravel()
    part = oracle.prefill_rows(c_kv=inp["c_kv"], gamma=inp["gamma"], k_rope=inp["k_rope"], w_ukv=inp["w_ukv"],
                               q_rows=inp["q"][rb, ri], lam_rows=inp["lam"][rb, ri], gate_rows=inp["gate"][rb, ri],
                               row_b=rb, row_i=ri, g=2, d_n=inp["d_n"], d_v=inp["d_v"], kv_sel=[1]).reshape(full.shape)
    np.testing.assert_array_equal(part[:, :, 2:4], full[:, :, 2:4])
    assert np.isnan(part[:, :, :2]).all() and np.isnan(part[:, :, 4:]).all()


# ------------------------------------------------------------------ YaRN (context extension)
# "Open-Source Frontier Models: Architecture and Benchmarks of Rnj-1 and Motif-2",
# section 2 (Context Extension via YaRN): per-frequency scale 1 (short wavelengths),
# 1/s (long wavelengths), linear ramp in between; logit temperature from ln s.
def test_yarn_factor_one_is_plain_rope():
    for d_R in (16, 64):
        np.testing.assert_allclose(oracle.yarn_inv_freq(d_R, 1.0, 4096.0), oracle.rope_freqs(d_R), rtol=1e-15, atol=0)


@pytest.mark.parametrize("factor,orig", [(32.0, 4096.0), (64.0, 4096.0), (16.0, 64.0)])
def test_yarn_frequency_regimes(factor, orig):
    d_R = 64
    base = oracle.rope_freqs(d_R)
    ratio = oracle.yarn_inv_freq(d_R, factor, orig) / base
    wavelength = 2 * math.pi / base
    short, long_ = orig / 32.0, orig / 1.0
    hi, lo = wavelength < short, wavelength > long_
    assert lo.any() and (hi.any() or wavelength.min() >= short)        # (short wavelength 2: no kept band)
    np.testing.assert_allclose(ratio[hi], 1.0, rtol=1e-15)            # high frequencies kept
    np.testing.assert_allclose(ratio[lo], 1.0 / factor, rtol=1e-15)   # low frequencies divided by s
    mid = ~hi & ~lo
    assert ((ratio[mid] < 1.0) & (ratio[mid] > 1.0 / factor)).all()
    assert (np.diff(ratio) <= 1e-15).all()                            # monotone in the wavelength
    # the ramp is linear in the wavelength: alpha = (lambda - short) / (long - short)
    alpha = (wavelength[mid] - short) / (long_ - short)
    np.testing.assert_allclose(ratio[mid], (1 - alpha) + alpha / factor, rtol=1e-14)


def test_yarn_interpolated_frequencies_map_positions_back():
    # for a fully interpolated frequency the angle at position s*p equals the native angle at p
    d_R, factor = 64, 32.0
    f = oracle.yarn_inv_freq(d_R, factor, 4096.0)
    base = oracle.rope_freqs(d_R)
    lo = f < base
    k = np.flatnonzero(np.isclose(f, base / factor, rtol=1e-15))
    assert len(k) > 0 and lo.any()
    for p in (1, 7, 4095):
        np.testing.assert_allclose(factor * p * f[k], p * base[k], rtol=1e-14)


def test_yarn_mscale_closed_form():
    assert oracle.yarn_mscale(1.0) == 1.0 and oracle.yarn_mscale(0.5) == 1.0
    assert abs(oracle.yarn_mscale(math.exp(10.0)) - 2.0) < 1e-15
    assert abs(oracle.yarn_mscale(64.0) - (1 + 0.1 * math.log(64.0))) < 1e-15


def test_prefill_explicit_frequencies_match_base_and_matrix_form():
    inp = tiny_inputs(d_R=8)
    plain = run_all_rows(inp)
    np.testing.assert_array_equal(run_all_rows(inp, inv_freq=oracle.rope_freqs(8)), plain)
    theta = oracle.yarn_inv_freq(8, 4.0, 8.0, beta_fast=4.0, beta_slow=1.0)
    scale = oracle.yarn_mscale(4.0) ** 2 / math.sqrt(inp["d_n"] + 8)
    y = run_all_rows(inp, inv_freq=theta, scale=scale)
    assert not np.allclose(y, plain)
    for b in range(inp["c_kv"].shape[0]):
        ey, _ = np_gdla_prefill(inp["c_kv"][b], inp["gamma"], inp["k_rope"][b], inp["q"][b], inp["w_ukv"],
                                inp["lam"][b], inp["gate"][b], inp["g"], inp["d_n"], inp["d_v"], oracle.MASK_CAUSAL, 0,
                                theta=theta, scale=scale)
        np.testing.assert_allclose(y[b], ey, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------------------ gate and lambda logits
# "Motif 3: Technical Report", section "Architecture": lambda_t = sigmoid(x_t W_lambda),
# and the sigmoid gate is computed from the normalised query latent (G = c_hat_Q W_G).
def test_project_exact_on_small_integers():
    # integer entries: every product and sum is exact in fp64, so the oracle must equal
    # the sum of products computed with Python integers
    a = RNG.integers(-9, 10, size=(4, 7))
    w = RNG.integers(-9, 10, size=(7, 5))
    want = [[sum(int(a[t, k]) * int(w[k, n]) for k in range(7)) for n in range(5)] for t in range(4)]
    assert np.array_equal(oracle.project(a.astype(float), w.astype(float)), np.array(want, dtype=float))


def test_project_one_hot_rows_pick_weight_rows():
    w = RNG.standard_normal((6, 3))
    a = np.eye(6)[[4, 0, 5]]
    assert np.array_equal(oracle.project(a, w), w[[4, 0, 5]])


def test_lambda_logits_are_linear_in_x():
    w = RNG.standard_normal((16, 5))
    x1, x2 = RNG.standard_normal((3, 16)), RNG.standard_normal((3, 16))
    lhs = oracle.lambda_logits(2.0 * x1 - 3.0 * x2, w)
    rhs = 2.0 * oracle.lambda_logits(x1, w) - 3.0 * oracle.lambda_logits(x2, w)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_gate_logits_of_a_constant_latent_row():
    # c_Q = a * ones: its RMS is |a|, so (eps = 0) c_hat = sign(a) gamma_q and G = sign(a) gamma_q @ W_G
    d_q, n = 8, 6
    gam = 1.0 + 0.1 * RNG.standard_normal(d_q)
    w = RNG.standard_normal((d_q, n))
    c = np.array([[3.0] * d_q, [-0.25] * d_q])
    got = oracle.gate_logits(c, gam, w, eps=0.0)
    assert np.allclose(got[0], gam @ w, rtol=1e-13, atol=1e-13)
    assert np.allclose(got[1], -(gam @ w), rtol=1e-13, atol=1e-13)


def test_gate_logits_normalise_before_projecting():
    # scale invariance of the normalised latent (eps = 0), and with W_G = I the gate
    # logits are the normalised latent itself, whose mean square is gamma-weighted 1
    d_q = 12
    gam = np.ones(d_q)
    c = RNG.standard_normal((5, d_q))
    g1 = oracle.gate_logits(c, gam, np.eye(d_q), eps=0.0)
    g2 = oracle.gate_logits(7.5 * c, gam, np.eye(d_q), eps=0.0)
    assert np.allclose(g1, g2, rtol=1e-13, atol=1e-13)
    assert np.allclose((g1 ** 2).mean(axis=1), 1.0, rtol=1e-13)
    # the gain multiplies latent column k, i.e. row k of W_G
    gam2 = np.arange(1.0, d_q + 1)
    assert np.allclose(oracle.gate_logits(c, gam2, np.eye(d_q), eps=0.0), g1 * gam2, rtol=1e-13)
