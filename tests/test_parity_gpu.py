"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Small cases are compared element by element over every output; they span
several tiles and a ragged tail. The full-size workloads are compared on a
deterministic sample of query rows (rows 0, 1, 127, 128, W-1, W, W+1, L-1 and
seeded random rows), all heads of every sampled row.
"""
import dataclasses

import numpy as np
import pytest
import torch

import differential_latent_attention_gdla_b200 as gdla
from differential_latent_attention_gdla_b200 import workloads as wl
from gdla_testutil import (assert_parity, f64, max_decode_logit, oracle_decode, oracle_prefill_rows,
                           peaked_elem_bound)

import oracle
from differential_latent_attention_gdla_b200 import _abi

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_prefill(shape, inp, **kw):
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    return gdla.prefill(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, sin,
                        inp["lam_logits"], inp["gate_logits"], g=shape.g, mask=shape.mask, window=shape.window, **kw)


def all_rows(shape):
    return [(b, i) for b in range(shape.B) for i in range(shape.L)]


SMALL = [
    wl.PREFILL["tiny_fp32"],
    wl.PrefillShape("bf16 small causal g=3 ragged", B=2, L=300, n_kv=2, g=3),
    wl.PrefillShape("bf16 small sliding W=100 g=2 ragged", B=1, L=333, n_kv=3, g=2, mask="sliding", window=100),
    wl.PrefillShape("bf16 sliding W=1", B=1, L=130, n_kv=1, g=2, mask="sliding", window=1),
    wl.PrefillShape("bf16 sliding W>=L", B=1, L=200, n_kv=1, g=3, mask="sliding", window=500),
    wl.PrefillShape("bf16 L=1", B=3, L=1, n_kv=2, g=2),
    wl.PrefillShape("bf16 d=64", B=1, L=257, d_c=256, d_R=32, n_kv=2, d_n=64, d_v=64, g=4),
    wl.PrefillShape("fp32 d=128 causal", B=1, L=150, n_kv=1, g=3, dtype="fp32"),
    # the report's attention shape: 16 KV heads, g = 4 (80 query heads), full and 128-token window
    wl.PrefillShape("bf16 80 heads g=4 causal", B=1, L=200, n_kv=16, g=4),
    wl.PrefillShape("bf16 80 heads g=4 sliding W=128", B=1, L=400, n_kv=16, g=4, mask="sliding", window=128),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: s.name)
@pytest.mark.parametrize("act", ["unit", "fan_in"])
def test_prefill_small_every_element(shape, act):
    inp = wl.make_prefill_inputs(shape, seed=11, device=DEV, act=act)
    y = run_prefill(shape, inp)
    torch.cuda.synchronize()
    ref = oracle_prefill_rows(inp, all_rows(shape), g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, mask=shape.mask,
                              window=shape.window)
    got = f64(y).reshape(ref.shape)
    assert_parity(got, ref, wl.torch_dtype(shape.dtype), shape.name)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_latent_expand_against_oracle_expansion(dtype):
    shape = wl.PrefillShape("expand", B=2, L=200, n_kv=3, g=1, dtype=dtype)
    inp = wl.make_prefill_inputs(shape, seed=3, device=DEV)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    kv, krot, chat = gdla.latent_expand(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["w_ukv"], cos, sin,
                                        n_kv=shape.n_kv, d_nope=shape.d_n, d_v=shape.d_v)
    torch.cuda.synchronize()
    w = f64(inp["w_ukv"])
    for b in range(shape.B):
        ch = oracle.latent_norm(f64(inp["c_kv"][b]), f64(inp["gamma"]), oracle.DEFAULT_EPS)
        assert_parity(f64(chat[b]), ch, wl.torch_dtype(dtype), "c_hat")
        for h in range(shape.n_kv):
            k, v = oracle.expand_head(ch, w, shape.n_kv, shape.d_n, shape.d_v, h)
            assert_parity(f64(kv[b, :, h, :shape.d_n]), k, wl.torch_dtype(dtype), f"k_nope head {h}")
            assert_parity(f64(kv[b, :, h, shape.d_n:]), v, wl.torch_dtype(dtype), f"v head {h}")
        kr = np.stack([oracle.rope(f64(inp["k_rope"][b, j]), j) for j in range(shape.L)])
        assert_parity(f64(krot[b]), kr, wl.torch_dtype(dtype), "k_rope_rot")


def _at_byte_offset(t, offset):
    """A contiguous copy of t whose data starts `offset` bytes past a 256-byte boundary."""
    n, es = t.numel(), t.element_size()
    buf = torch.empty(n + 256 // es, dtype=t.dtype, device=t.device)
    v = buf[offset // es: offset // es + n].view(t.shape)
    v.copy_(t)
    assert v.data_ptr() % 256 == offset
    return v


def test_prefill_gate_output_and_rope_tables_only_16_byte_aligned():
    # gate logits and output (then the RoPE tables) 16-byte but not 32-byte aligned: the
    # 16-byte access path, bit-identical to the 32-byte one and within tolerance of the oracle
    shape = wl.PrefillShape("bf16 small causal g=3 ragged", B=2, L=300, n_kv=2, g=3)
    inp = wl.make_prefill_inputs(shape, seed=5, device=DEV)
    y32 = run_prefill(shape, inp)
    inp16 = dict(inp, gate_logits=_at_byte_offset(inp["gate_logits"], 16))
    out16 = _at_byte_offset(torch.zeros_like(y32), 48)
    y16 = run_prefill(shape, inp16, out=out16)
    torch.cuda.synchronize()
    assert y16.data_ptr() == out16.data_ptr()
    assert torch.equal(y16, y32)
    ref = oracle_prefill_rows(inp, all_rows(shape), g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, mask=shape.mask,
                              window=shape.window)
    assert_parity(f64(y16).reshape(ref.shape), ref, torch.bfloat16, "16-byte aligned gate/out")
    # the RoPE tables only 16-byte aligned (gate and output 32-byte aligned)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    cos16, sin16 = _at_byte_offset(cos, 16), _at_byte_offset(sin, 80)
    y_t = gdla.prefill(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos16, sin16,
                       inp["lam_logits"], inp["gate_logits"], g=shape.g, mask=shape.mask, window=shape.window)
    torch.cuda.synchronize()
    assert torch.equal(y_t, y32)


@pytest.mark.parametrize("name", ["b4_l4k_g2", "b1_l32k_g3", "b2_l64k_swa4k"])
def test_prefill_full_size_sampled_rows(name):
    shape = wl.PREFILL[name]
    inp = wl.make_prefill_inputs(shape, seed=0, device=DEV)
    y = run_prefill(shape, inp)
    torch.cuda.synchronize()
    rows = wl.sample_rows(shape, n_random=32)
    ref = oracle_prefill_rows(inp, rows, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, mask=shape.mask,
                              window=shape.window)
    rb = torch.tensor([r[0] for r in rows], device=DEV)
    ri = torch.tensor([r[1] for r in rows], device=DEV)
    got = f64(y[rb, ri])
    assert_parity(got, ref, torch.bfloat16, name)
    assert torch.isfinite(y).all()


def test_prefill_lambda_one_identical_queries_cancel():
    """Signal queries equal to their noise head's query with lambda -> 1 give
    D = 0. On the GPU the noise head's output is held in bf16 for the
    epilogue, so each element may keep a residual of half a bf16 ulp of H:
    |Y(lambda=1)| <= 2^-8 |Y(lambda=0)| element by element (Y(lambda=0) =
    sigmoid(G) H_S with H_S = H_N here)."""
    shape = wl.PrefillShape("cancel", B=1, L=256, n_kv=2, g=3)
    inp = wl.make_prefill_inputs(shape, seed=5, device=DEV)
    for i in range(shape.n_S):
        inp["q"][:, :, i] = inp["q"][:, :, shape.n_S + i // shape.g]
    inp["lam_logits"].fill_(30.0)
    y1 = f64(run_prefill(shape, inp))
    y0 = f64(run_prefill(shape, dict(inp, lam_logits=torch.full_like(inp["lam_logits"], -30.0))))
    rms0 = float(np.sqrt((y0 ** 2).mean()))
    assert float((np.abs(y1) - 2.0 ** -8 * np.abs(y0)).max()) <= 1e-3 * rms0
    assert float(np.sqrt((y1 ** 2).mean())) <= 2e-3 * rms0


def test_prefill_emits_decode_cache_and_decode_matches_last_row():
    shape = wl.PrefillShape("prefill->decode", B=2, L=520, n_kv=2, g=2)
    inp = wl.make_prefill_inputs(shape, seed=9, device=DEV)
    cache_c = torch.empty((shape.B, shape.L, shape.d_c), dtype=torch.bfloat16, device=DEV)
    cache_k = torch.empty((shape.B, shape.L, shape.d_R), dtype=torch.bfloat16, device=DEV)
    y = run_prefill(shape, inp, cache_c_hat=cache_c, cache_k_rope=cache_k)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    for T in (1, 129, 520):
        seqlens = torch.full((shape.B,), T, dtype=torch.int32, device=DEV)
        yd = gdla.decode(cache_c, cache_k, inp["q"][:, T - 1].contiguous(), inp["w_ukv"], cos, sin,
                         inp["lam_logits"][:, T - 1].contiguous(), inp["gate_logits"][:, T - 1].contiguous(), seqlens,
                         g=shape.g)
        torch.cuda.synchronize()
        ref = oracle_prefill_rows(inp, [(b, T - 1) for b in range(shape.B)], g=shape.g, d_nope=shape.d_n,
                                  d_v=shape.d_v)
        assert_parity(f64(yd), ref, torch.bfloat16, f"decode T={T}")
        assert_parity(f64(y[:, T - 1]), ref, torch.bfloat16, f"prefill row {T - 1}")


DECODE_SMALL = [
    (wl.DecodeShape("decode small ragged", B=3, T=300, n_kv=2, g=2), [300, 37, 1], "causal", 0),
    (wl.DecodeShape("decode sliding", B=2, T=700, n_kv=1, g=3), [700, 200], "sliding", 128),
    (wl.DecodeShape("decode d=32 fp32", B=2, T=150, d_c=64, d_R=16, n_kv=4, d_n=32, d_v=32, g=2, dtype="fp32"),
     [150, 77], "causal", 0),
    # 40 sequences: the split heuristic gives splits of three 128-token tiles, so one block
    # walks several tiles (ring reuse, both S^T / P^T buffers, the O^T rescale) and the
    # lengths 1000 .. 103 leave ragged tails and short last splits
    (wl.DecodeShape("decode multi-tile splits", B=40, T=1000, n_kv=16, g=2), [1000 - 23 * i for i in range(40)],
     "causal", 0),
    (wl.DecodeShape("decode multi-tile sliding W=300", B=40, T=1000, n_kv=16, g=2),
     [1000 - 23 * i for i in range(40)], "sliding", 300),
]


@pytest.mark.parametrize("case", DECODE_SMALL, ids=lambda c: c[0].name)
@pytest.mark.parametrize("act", ["unit", "fan_in"])
def test_decode_small_every_element(case, act):
    shape, seqlens, mask, window = case
    inp = wl.make_decode_inputs(shape, seed=4, device=DEV, act=act, seqlens=seqlens)
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                    inp["gate_logits"], inp["seqlens"], g=shape.g, mask=mask, window=window)
    torch.cuda.synchronize()
    ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, mask=mask, window=window)
    assert_parity(f64(y), ref, wl.torch_dtype(shape.dtype), shape.name)


def test_decode_full_size_every_sequence():
    """The bench decode workload (64 sequences x 32768 cached tokens) in the bench's
    launch configuration: every sequence is checked, each on one KV group (its g
    signal heads and the noise head), the group rotating so all 16 are covered."""
    shape = wl.DECODE["b64_t32k"]
    inp = wl.make_decode_inputs(shape, seed=0, device=DEV)
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                    inp["gate_logits"], inp["seqlens"], g=shape.g)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    got, ref = [], []
    for b in range(shape.B):
        h = b % shape.n_kv
        r = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, seqs=[b], kv_sel=[h])[0]
        got.append(f64(y[b, h * shape.g:(h + 1) * shape.g]))
        ref.append(r[h * shape.g:(h + 1) * shape.g])
    assert_parity(np.stack(got), np.stack(ref), torch.bfloat16, "decode b64_t32k, all sequences")


def test_decode_80_heads_g4():
    """The report's head layout in decode: 16 KV heads with g = 4 (64 signal + 16
    noise = 80 query heads), all in one CTA of the wide split kernel."""
    for mask, window in (("causal", 0), ("sliding", 128)):
        shape = wl.DecodeShape("decode 80 heads", B=5, T=700, n_kv=16, g=4)
        inp = wl.make_decode_inputs(shape, seed=51, device=DEV, act="unit", seqlens=[700, 513, 129, 48, 1])
        cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
        y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                        inp["gate_logits"], inp["seqlens"], g=shape.g, mask=mask, window=window)
        torch.cuda.synchronize()
        ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, mask=mask, window=window)
        assert_parity(f64(y), ref, torch.bfloat16, f"decode 80 heads g=4 {mask}")


@pytest.mark.parametrize("n_kv,g", [(16, 3), (12, 4), (10, 6)])
def test_decode_wide_split_every_element(n_kv, g):
    """49 .. 80 query heads take the wide split kernel (one head group of up to 80 heads,
    48-token tiles, K-major P): 64, 60 and 70 heads leave 16, 20 and 10 of its 80 heads as
    padding; lengths that end inside a tile and a one-token sequence; causal and a
    100-token window."""
    for mask, window in (("causal", 0), ("sliding", 100)):
        shape = wl.DecodeShape(f"decode wide n_kv={n_kv} g={g}", B=4, T=500, n_kv=n_kv, g=g)
        inp = wl.make_decode_inputs(shape, seed=60 + g, device=DEV, act="unit", seqlens=[500, 257, 49, 1])
        cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
        y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                        inp["gate_logits"], inp["seqlens"], g=shape.g, mask=mask, window=window)
        torch.cuda.synchronize()
        ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, mask=mask, window=window)
        assert_parity(f64(y), ref, torch.bfloat16, f"{shape.name} {mask}")


def test_decode_80_heads_g4_sequences_over_many_blocks():
    """80 heads over 8 sequences of up to 3000 tokens: ~500 tiles of 48 tokens over 148
    split CTAs, so every sequence is merged from the partials of several CTAs."""
    shape = wl.DecodeShape("decode 80 heads, 8 x 3000", B=8, T=3000, n_kv=16, g=4)
    inp = wl.make_decode_inputs(shape, seed=77, device=DEV, act="unit",
                                seqlens=[3000, 2999, 2400, 1777, 1200, 600, 97, 48])
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                    inp["gate_logits"], inp["seqlens"], g=shape.g)
    torch.cuda.synchronize()
    ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    assert_parity(f64(y), ref, torch.bfloat16, shape.name)


def test_decode_many_sequences_per_split_block():
    """Many short sequences: one split block covers several whole sequences and the
    parts of two more, so it changes sequence (query operand, running maxima and
    value accumulator) between tiles."""
    shape = wl.DecodeShape("decode many short", B=300, T=200, n_kv=2, g=2)
    gen = torch.Generator().manual_seed(5)
    seqlens = torch.randint(1, shape.T + 1, (shape.B,), generator=gen).tolist()
    seqlens[:4] = [1, 1, 48, 49]
    inp = wl.make_decode_inputs(shape, seed=52, device=DEV, act="unit", seqlens=seqlens)
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                    inp["gate_logits"], inp["seqlens"], g=shape.g)
    torch.cuda.synchronize()
    ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    assert_parity(f64(y), ref, torch.bfloat16, "decode 300 short sequences")


def test_decode_out_of_range_seqlens_are_clamped_and_reported():
    """A sequence length outside [1, T_max] (which the host cannot see: seqlens live
    on the device) is clamped into the cache by every decode kernel and reported as
    GDLA_ERR_INVALID_ARG in the workspace status word; the other sequences are
    still computed correctly."""
    for dtype in ("bf16", "fp32"):
        shape = wl.DecodeShape(f"decode bad seqlens {dtype}", B=4, T=160, n_kv=2, g=2, dtype=dtype)
        inp = wl.make_decode_inputs(shape, seed=53, device=DEV, act="unit", seqlens=[160, 0, 77, 100000])
        cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
        ws = torch.empty(gdla.decode_workspace_size(B=shape.B, T_max=shape.T, d_c=shape.d_c, d_rope=shape.d_R,
                                                    n_kv=shape.n_kv, d_nope=shape.d_n, d_v=shape.d_v, g=shape.g,
                                                    dtype=wl.torch_dtype(dtype)), dtype=torch.uint8, device=DEV)
        y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                        inp["gate_logits"], inp["seqlens"], g=shape.g, workspace=ws)
        torch.cuda.synchronize()
        assert gdla.workspace_status(ws) == _abi.GDLA_ERR_INVALID_ARG
        ok = [0, 2]
        ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, seqs=ok)
        assert_parity(f64(y[ok]), ref, wl.torch_dtype(dtype), f"decode with bad seqlens, good rows ({dtype})")
        # the clamped ones equal the decode of their clamped lengths
        inp2 = dict(inp, seqlens=torch.tensor([160, 1, 77, 160], dtype=torch.int32, device=DEV))
        y2 = gdla.decode(inp2["c_cache"], inp2["kr_cache"], inp2["q"], inp2["w_ukv"], cos, sin, inp2["lam_logits"],
                         inp2["gate_logits"], inp2["seqlens"], g=shape.g, workspace=ws)
        torch.cuda.synchronize()
        assert gdla.workspace_status(ws) == 0
        assert torch.equal(y, y2)


def test_binding_raises_on_invalid_arguments():
    shape = wl.PrefillShape("bad", B=1, L=64, n_kv=1, g=2, mask="sliding", window=0)
    inp = wl.make_prefill_inputs(shape, seed=1, device=DEV)
    with pytest.raises(gdla.GdlaError):
        run_prefill(shape, inp)


@pytest.mark.parametrize("scale", [20.0, 30.0])
def test_decode_peaked_softmax_rescale_path(scale):
    """Very peaked attention (q scaled up) makes the running maximum of many
    heads jump across tiles, which exercises the O-rescale path."""
    shape = wl.DecodeShape("decode peaked", B=3, T=2000, n_kv=16, g=2)
    inp = wl.make_decode_inputs(shape, seed=12, device=DEV, act="unit", seqlens=[2000, 1333, 700])
    inp["q"] = (inp["q"].float() * scale).to(torch.bfloat16)
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                    inp["gate_logits"], inp["seqlens"], g=shape.g)
    torch.cuda.synchronize()
    ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    # logits reach |s| ~ 50-150 here: the bf16 absorbed query moves single
    # exponents by ~|s| 2^-9, so the element bound grows with the largest logit
    # (a wrong rescale would be an O(1) error in the RMS bar as well)
    smax = max_decode_logit(inp, g=shape.g, d_nope=shape.d_n, scale=gdla.default_scale(shape.d_n, shape.d_R))
    assert_parity(f64(y), ref, torch.bfloat16, f"decode peaked x{scale} (max logit {smax:.0f})",
                  elem_bound=peaked_elem_bound(smax))


@pytest.mark.parametrize("g", [1, 5, 8])
def test_decode_group_sizes_every_element(g):
    """g + 1 heads per KV group from 2 to 9: the combine blocks hold 8, 6 and 9 query
    rows (one, two or four row groups of its W_UV tile) and the split kernel's padded
    head columns vary."""
    shape = wl.DecodeShape(f"decode g={g}", B=5, T=400, n_kv=2, g=g)
    inp = wl.make_decode_inputs(shape, seed=14 + g, device=DEV, act="fan_in", seqlens=[400, 333, 129, 64, 1])
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                    inp["gate_logits"], inp["seqlens"], g=shape.g)
    torch.cuda.synchronize()
    ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    assert_parity(f64(y), ref, torch.bfloat16, shape.name)


def test_decode_peaked_multi_tile_splits():
    """Peaked attention with several tiles per split block: the running maximum
    jumps between tiles of one block, so O^T is rescaled in TMEM between value
    passes (the path a one-tile split never takes)."""
    shape = wl.DecodeShape("decode peaked multi-tile", B=40, T=1000, n_kv=16, g=2)
    inp = wl.make_decode_inputs(shape, seed=13, device=DEV, act="unit", seqlens=[1000 - 17 * i for i in range(40)])
    inp["q"] = (inp["q"].float() * 20.0).to(torch.bfloat16)
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                    inp["gate_logits"], inp["seqlens"], g=shape.g)
    torch.cuda.synchronize()
    ref = oracle_decode(inp, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    smax = max_decode_logit(inp, g=shape.g, d_nope=shape.d_n, scale=gdla.default_scale(shape.d_n, shape.d_R))
    assert_parity(f64(y), ref, torch.bfloat16, f"decode peaked multi-tile (max logit {smax:.0f})",
                  elem_bound=peaked_elem_bound(smax))


# ------------------------------------------------------------------ YaRN context extension
# Rescaled RoPE tables and the YaRN logit temperature are inputs of the same kernels
# ("Open-Source Frontier Models: Architecture and Benchmarks of Rnj-1 and Motif-2",
# section 2); positions far beyond the native length exercise the interpolated band.
YARN = dict(factor=16.0, orig=64)


def yarn_scale(d_qk):
    return gdla.yarn_mscale(YARN["factor"]) ** 2 / float(np.sqrt(d_qk))


def test_prefill_yarn_every_element():
    shape = wl.PrefillShape("bf16 YaRN x16 from 64 tokens, g=3", B=1, L=300, n_kv=2, g=3)
    inp = wl.make_prefill_inputs(shape, seed=31, device=DEV, act="unit")
    cos, sin = gdla.yarn_rope_tables(shape.L, shape.d_R, YARN["factor"], YARN["orig"], device=DEV)
    scale = yarn_scale(shape.d_n + shape.d_R)
    y = gdla.prefill(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                     inp["gate_logits"], g=shape.g, softmax_scale=scale)
    torch.cuda.synchronize()
    rows = all_rows(shape)
    rb = torch.tensor([r[0] for r in rows], device=DEV)
    ri = torch.tensor([r[1] for r in rows], device=DEV)
    ref = oracle.prefill_rows(
        c_kv=f64(inp["c_kv"]), gamma=f64(inp["gamma"]), k_rope=f64(inp["k_rope"]), w_ukv=f64(inp["w_ukv"]),
        q_rows=f64(inp["q"][rb, ri]), lam_rows=f64(inp["lam_logits"][rb, ri]), gate_rows=f64(inp["gate_logits"][rb, ri]),
        row_b=rb.cpu().numpy(), row_i=ri.cpu().numpy(), g=shape.g, d_n=shape.d_n, d_v=shape.d_v, scale=scale,
        inv_freq=oracle.yarn_inv_freq(shape.d_R, YARN["factor"], YARN["orig"]))
    assert_parity(f64(y).reshape(ref.shape), ref, torch.bfloat16, shape.name)
    # the rescaled tables change the result (the check above is not vacuous)
    plain = oracle.prefill_rows(
        c_kv=f64(inp["c_kv"]), gamma=f64(inp["gamma"]), k_rope=f64(inp["k_rope"]), w_ukv=f64(inp["w_ukv"]),
        q_rows=f64(inp["q"][rb, ri]), lam_rows=f64(inp["lam_logits"][rb, ri]), gate_rows=f64(inp["gate_logits"][rb, ri]),
        row_b=rb.cpu().numpy(), row_i=ri.cpu().numpy(), g=shape.g, d_n=shape.d_n, d_v=shape.d_v)
    assert np.sqrt(np.mean((plain - ref) ** 2)) > 0.1 * np.sqrt(np.mean(ref ** 2))


def test_decode_yarn_every_element():
    shape = wl.DecodeShape("bf16 YaRN decode B=3 T=300", B=3, T=300, n_kv=2, g=2)
    inp = wl.make_decode_inputs(shape, seed=33, device=DEV, act="unit", seqlens=[300, 190, 64])
    cos, sin = gdla.yarn_rope_tables(shape.T, shape.d_R, YARN["factor"], YARN["orig"], device=DEV)
    scale = yarn_scale(shape.d_n + shape.d_R)
    y = gdla.decode(inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                    inp["gate_logits"], inp["seqlens"], g=shape.g, softmax_scale=scale)
    torch.cuda.synchronize()
    theta = oracle.yarn_inv_freq(shape.d_R, YARN["factor"], YARN["orig"])
    ref = np.stack([oracle.decode_seq(
        c_hat=f64(inp["c_cache"][b, :T]), k_r_rot=f64(inp["kr_cache"][b, :T]), q=f64(inp["q"][b]),
        w_ukv=f64(inp["w_ukv"]), lam=f64(inp["lam_logits"][b]), gate=f64(inp["gate_logits"][b]), g=shape.g,
        d_n=shape.d_n, d_v=shape.d_v, scale=scale, inv_freq=theta)
        for b, T in enumerate(int(t) for t in inp["seqlens"])])
    assert_parity(f64(y), ref, torch.bfloat16, shape.name)
