"""GPU: attention over a block of query rows, and the host-buffer prefill that
streams its inputs through such blocks.

A query block (positions q_start .. q_start+q_len-1 against keys 0 .. L-1) is
the whole-sequence attention restricted to those rows, so a block that starts
on a 64-row boundary must reproduce the whole call's rows bit for bit; any
other block is held to the oracle like every prefill. gdla_prefill_host runs
the same kernels chunk by chunk, so with chunks of a multiple of 64 tokens it
must equal gdla_prefill bit for bit, with page-locked or pageable host memory.
"""
import numpy as np
import pytest
import torch

import differential_latent_attention_gdla_b200 as gdla
from differential_latent_attention_gdla_b200 import workloads as wl
from gdla_testutil import assert_parity, f64, oracle_prefill_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def expand(shape, inp, cos, sin):
    kv, krot, _ = gdla.latent_expand(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["w_ukv"], cos, sin,
                                     n_kv=shape.n_kv, d_nope=shape.d_n, d_v=shape.d_v)
    return kv, krot


def attend_block(shape, inp, kv, krot, cos, sin, q_start, q_len):
    # fresh allocations: a contiguous row slice of a tensor can start off a 16-byte boundary
    sl = slice(q_start, q_start + q_len)
    rows = {k: inp[k][:, sl].clone(memory_format=torch.contiguous_format) for k in ("q", "lam_logits", "gate_logits")}
    return gdla.attend(rows["q"], kv, krot, cos, sin, rows["lam_logits"], rows["gate_logits"], g=shape.g,
                       mask=shape.mask, window=shape.window, q_start=q_start)


BLOCK_SHAPES = [
    wl.PrefillShape("bf16 causal g=3", B=2, L=700, n_kv=2, g=3),
    wl.PrefillShape("bf16 sliding W=100 g=2", B=1, L=600, n_kv=2, g=2, mask="sliding", window=100),
    wl.PrefillShape("fp32 causal g=2", B=1, L=300, n_kv=1, g=2, dtype="fp32"),
]


@pytest.mark.parametrize("shape", BLOCK_SHAPES, ids=lambda s: s.name)
def test_attend_query_blocks_bit_identical_to_whole(shape):
    inp = wl.make_prefill_inputs(shape, seed=21, device=DEV)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    kv, krot = expand(shape, inp, cos, sin)
    whole = gdla.attend(inp["q"], kv, krot, cos, sin, inp["lam_logits"], inp["gate_logits"], g=shape.g,
                        mask=shape.mask, window=shape.window)
    starts = list(range(0, shape.L, 256)) + [shape.L]
    for q0, q1 in zip(starts[:-1], starts[1:]):
        blk = attend_block(shape, inp, kv, krot, cos, sin, q0, q1 - q0)
        torch.cuda.synchronize()
        assert torch.equal(blk, whole[:, q0:q1]), (shape.name, q0, q1)
    # one row, the last one
    blk = attend_block(shape, inp, kv, krot, cos, sin, shape.L - 1, 1)
    assert torch.equal(blk, whole[:, shape.L - 1:])


@pytest.mark.parametrize("shape", BLOCK_SHAPES[:2], ids=lambda s: s.name)
def test_attend_ragged_query_block_against_oracle(shape):
    # a block that starts inside a 64-row tile and ends inside one
    inp = wl.make_prefill_inputs(shape, seed=22, device=DEV)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    kv, krot = expand(shape, inp, cos, sin)
    q_start, q_len = 100, 250
    blk = attend_block(shape, inp, kv, krot, cos, sin, q_start, q_len)
    torch.cuda.synchronize()
    rows = [(b, i) for b in range(shape.B) for i in range(q_start, q_start + q_len)]
    ref = oracle_prefill_rows(inp, rows, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v, mask=shape.mask,
                              window=shape.window)
    assert_parity(f64(blk).reshape(ref.shape), ref, wl.torch_dtype(shape.dtype), shape.name)


def host_copy(inp, pinned):
    keys = ("c_kv", "k_rope", "q", "lam_logits", "gate_logits")
    return {k: (inp[k].cpu().pin_memory() if pinned else inp[k].cpu()) for k in keys}


def run_host(shape, inp, host, cos, sin, chunk, **kw):
    out = gdla.prefill_host(host["c_kv"], inp["gamma"], host["k_rope"], host["q"], inp["w_ukv"], cos, sin,
                            host["lam_logits"], host["gate_logits"], g=shape.g, mask=shape.mask,
                            window=shape.window, chunk_tokens=chunk, **kw)
    torch.cuda.synchronize()
    return out


HOST_SHAPES = [
    wl.PrefillShape("bf16 causal B=2 L=1000", B=2, L=1000, n_kv=2, g=3),
    wl.PrefillShape("bf16 sliding W=100", B=1, L=777, n_kv=2, g=2, mask="sliding", window=100),
    wl.PrefillShape("fp32 causal", B=2, L=300, n_kv=1, g=2, dtype="fp32"),
]


@pytest.mark.parametrize("shape", HOST_SHAPES, ids=lambda s: s.name)
@pytest.mark.parametrize("chunk", [64, 256, 0])
def test_prefill_host_equals_device_prefill(shape, chunk):
    inp = wl.make_prefill_inputs(shape, seed=31, device=DEV)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    ref = gdla.prefill(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, sin,
                       inp["lam_logits"], inp["gate_logits"], g=shape.g, mask=shape.mask, window=shape.window)
    host = host_copy(inp, pinned=True)
    out = run_host(shape, inp, host, cos, sin, chunk)
    assert not out.is_cuda and out.is_pinned()
    assert torch.equal(out, ref.cpu()), (shape.name, chunk)


def test_prefill_host_pageable_memory_and_cache_outputs():
    shape = HOST_SHAPES[0]
    inp = wl.make_prefill_inputs(shape, seed=32, device=DEV)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    cc = torch.empty((shape.B, shape.L, shape.d_c), dtype=torch.bfloat16, device=DEV)
    ck = torch.empty((shape.B, shape.L, shape.d_R), dtype=torch.bfloat16, device=DEV)
    ref = gdla.prefill(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, sin,
                       inp["lam_logits"], inp["gate_logits"], g=shape.g, cache_c_hat=cc, cache_k_rope=ck)
    cc2, ck2 = torch.empty_like(cc), torch.empty_like(ck)
    host = host_copy(inp, pinned=False)
    out = torch.empty(ref.shape, dtype=ref.dtype)  # pageable output too
    run_host(shape, inp, host, cos, sin, 320, out=out, cache_c_hat=cc2, cache_k_rope=ck2)
    assert torch.equal(out, ref.cpu())
    assert torch.equal(cc2, cc) and torch.equal(ck2, ck)


def test_prefill_host_ragged_chunks_against_oracle():
    # chunks of 100 tokens start inside 64-row tiles: held to the oracle on every element
    shape = wl.PrefillShape("bf16 host chunks of 100", B=1, L=450, n_kv=2, g=3)
    inp = wl.make_prefill_inputs(shape, seed=33, device=DEV, act="fan_in")
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    out = run_host(shape, inp, host_copy(inp, pinned=True), cos, sin, 100)
    rows = [(0, i) for i in range(shape.L)]
    ref = oracle_prefill_rows(inp, rows, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    assert_parity(f64(out).reshape(ref.shape), ref, torch.bfloat16, shape.name)


def test_prefill_host_status_word_is_clear_after_call():
    shape = HOST_SHAPES[0]
    inp = wl.make_prefill_inputs(shape, seed=34, device=DEV)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    ws = torch.empty(gdla.prefill_host_workspace_size(B=shape.B, L=shape.L, d_c=shape.d_c, d_rope=shape.d_R,
                                                      n_kv=shape.n_kv, d_nope=shape.d_n, d_v=shape.d_v, g=shape.g,
                                                      chunk_tokens=128), dtype=torch.uint8, device=DEV)
    ws.fill_(0xFF)  # a stale status word must be cleared by the call
    out = run_host(shape, inp, host_copy(inp, pinned=True), cos, sin, 128, workspace=ws)
    assert gdla.workspace_status(ws) == 0
    assert np.isfinite(f64(out)).all()
