"""GPU parity of gdla_gates, the gate and lambda logits computed from the layer's
activations ("Motif 3: Technical Report", section "Architecture": lambda_t =
sigmoid(x_t W_lambda); the output gate comes from the normalised query latent),
against the fp64 oracle on the same seeded inputs. bf16 products whose widths are
multiples of 8 run on the tensor cores (the gate with bf16 output, lambda with fp32
output); other widths and fp32 take the CUDA cores."""
import math

import numpy as np
import pytest
import torch

import differential_latent_attention_gdla_b200 as gdla
from differential_latent_attention_gdla_b200 import workloads as wl
from gdla_testutil import assert_parity, f64, oracle_prefill_rows

import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def make(B, L, d_q, d_x, n_S, d_v, dtype, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)

    def rn(*shape, scale=1.0):
        return (torch.randn(*shape, generator=g) * scale).to(dtype).to(DEV)

    return dict(c_q=rn(B, L, d_q), gamma_q=(1.0 + 0.1 * torch.randn(d_q, generator=g)).to(dtype).to(DEV),
                w_g=rn(d_q, n_S * d_v, scale=1.0 / math.sqrt(d_q)), x=rn(B, L, d_x),
                w_lambda=rn(d_x, n_S, scale=1.0 / math.sqrt(d_x)))


def check(inp, n_S, d_v, dtype, what):
    gate, lam = gdla.gates(inp["c_q"], inp["gamma_q"], inp["w_g"], inp["x"], inp["w_lambda"], n_signal=n_S, d_v=d_v)
    torch.cuda.synchronize()
    B, L, d_q = inp["c_q"].shape
    ref_g = oracle.gate_logits(f64(inp["c_q"]).reshape(B * L, d_q), f64(inp["gamma_q"]), f64(inp["w_g"]))
    ref_l = oracle.lambda_logits(f64(inp["x"]).reshape(B * L, -1), f64(inp["w_lambda"]))
    assert gate.shape == (B, L, n_S, d_v) and gate.dtype == dtype
    assert lam.shape == (B, L, n_S) and lam.dtype == torch.float32
    assert_parity(f64(gate).reshape(ref_g.shape), ref_g, dtype, what + " gate")
    # lambda: exact products of the stored inputs, fp32 sums over d_x terms
    err = np.abs(f64(lam).reshape(ref_l.shape) - ref_l)
    assert err.max() <= 1e-4 * max(1.0, float(np.abs(ref_l).max())), (what, err.max())


@pytest.mark.parametrize("n_S", [32, 48])
def test_gates_report_shapes_tensor_cores(n_S):
    # d_q = 1536, n_S * d_v = 4096 / 6144: the tcgen05 product
    inp = make(2, 300, 1536, 2048, n_S, 128, torch.bfloat16, seed=n_S)
    check(inp, n_S, 128, torch.bfloat16, f"bf16 n_S={n_S}")


def test_gates_odd_widths():
    # gate: n_S * d_v = 384 is not a multiple of the 256-column tile and d_q = 200 not one of
    # the 64-deep K block (tensor cores, zero-filled tails); lambda: n_S = 6 (CUDA cores)
    inp = make(3, 77, 200, 96, 6, 64, torch.bfloat16, seed=5)
    check(inp, 6, 64, torch.bfloat16, "bf16 odd widths")


def test_gates_gate_width_not_a_multiple_of_64():
    # gate: n_S * d_v = 200 columns = three full 64-column store boxes and one of 8 columns,
    # 90 tokens = a ragged 128-row tile (rows 90 .. 127 are not written); d_q = 136 is a
    # K tail of the 64-deep block
    inp = make(2, 45, 136, 72, 5, 40, torch.bfloat16, seed=9)
    check(inp, 5, 40, torch.bfloat16, "bf16 gate width 200")


def test_gates_many_tiles_per_block():
    # 1024 tokens x 6144 gate columns = 192 output tiles of 128 x 256 on 148 blocks, and
    # 40000 tokens of lambda = 313 tiles of 128 x 64 (fp32): both walk several tiles per
    # block through the double-buffered accumulator, with a ragged last row tile
    inp = make(1, 1024, 1536, 2048, 48, 128, torch.bfloat16, seed=11)
    check(inp, 48, 128, torch.bfloat16, "bf16 1024 tokens, 48 signal heads")
    g = torch.Generator(device="cpu").manual_seed(12)
    x = torch.randn(40000, 2048, generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn(2048, 40, generator=g) / math.sqrt(2048)).to(torch.bfloat16).to(DEV)
    _, lam = gdla.gates(x=x, w_lambda=w, n_signal=40)
    torch.cuda.synchronize()
    ref = oracle.lambda_logits(f64(x), f64(w))
    err = np.abs(f64(lam) - ref)
    assert err.max() <= 1e-4 * max(1.0, float(np.abs(ref).max())), err.max()


def test_gates_fp32_tiny_config():
    # the tiny fp32 configuration: d_q = 64, 8 signal heads of d_v = 32
    inp = make(1, 128, 64, 64, 8, 32, torch.float32, seed=6)
    check(inp, 8, 32, torch.float32, "fp32 tiny")


def test_gates_one_token_per_sequence_and_either_half():
    # decode form: c_q [B, d_q]; and each half alone
    inp = make(5, 1, 1536, 512, 32, 128, torch.bfloat16, seed=7)
    c2, x2 = inp["c_q"][:, 0].contiguous(), inp["x"][:, 0].contiguous()
    gate, lam = gdla.gates(c2, inp["gamma_q"], inp["w_g"], x2, inp["w_lambda"], n_signal=32, d_v=128)
    assert gate.shape == (5, 32, 128) and lam.shape == (5, 32)
    g_only, none = gdla.gates(c2, inp["gamma_q"], inp["w_g"], n_signal=32, d_v=128)
    none2, l_only = gdla.gates(x=x2, w_lambda=inp["w_lambda"], n_signal=32)
    torch.cuda.synchronize()
    assert none is None and none2 is None
    assert torch.equal(g_only, gate) and torch.equal(l_only, lam)


def test_prefill_with_computed_gates_against_oracle():
    # the whole chain: gates from (c_q, x), then the prefill, against the oracle's chain
    shape = wl.PrefillShape("chain", B=1, L=260, n_kv=2, g=3)
    inp = wl.make_prefill_inputs(shape, seed=8, device=DEV, act="fan_in")
    act = make(shape.B, shape.L, 1536, 1024, shape.n_S, shape.d_v, torch.bfloat16, seed=9)
    gate, lam = gdla.gates(act["c_q"], act["gamma_q"], act["w_g"], act["x"], act["w_lambda"], n_signal=shape.n_S,
                           d_v=shape.d_v)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    y = gdla.prefill(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, sin, lam, gate,
                     g=shape.g)
    torch.cuda.synchronize()
    T = shape.B * shape.L
    ref_g = oracle.gate_logits(f64(act["c_q"]).reshape(T, -1), f64(act["gamma_q"]), f64(act["w_g"]))
    ref_l = oracle.lambda_logits(f64(act["x"]).reshape(T, -1), f64(act["w_lambda"]))
    chain = dict(inp, gate_logits=torch.from_numpy(ref_g.reshape(gate.shape)).to(DEV),
                 lam_logits=torch.from_numpy(ref_l.reshape(lam.shape)).to(DEV))
    rows = [(0, i) for i in range(shape.L)]
    ref = oracle_prefill_rows(chain, rows, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    assert_parity(f64(y).reshape(ref.shape), ref, torch.bfloat16, "gates -> prefill")
