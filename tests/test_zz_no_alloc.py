"""gdla_decode_noalloc: the decode entry point for callers that cannot allocate
device memory while they run (a latency-bound serving loop, where an allocation
can block or fail mid-step; a plugin that only receives its inputs and outputs).
It runs the same kernels as gdla_decode, which takes a caller-allocated
workspace, so it must return the same bytes, call after call, even though every
call reuses the library's one fixed scratch array.

Kept in its own file so that pytest collects it last."""
import ctypes

import pytest
import torch

import differential_latent_attention_gdla_b200 as gdla
from differential_latent_attention_gdla_b200 import _abi
from differential_latent_attention_gdla_b200 import workloads as wl
from gdla_testutil import assert_parity, f64, oracle_decode

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    (wl.DecodeShape("noalloc B=16 T=4096 g=2", B=16, T=4096, g=2), None),
    (wl.DecodeShape("noalloc ragged B=3 T=300 n_kv=2", B=3, T=300, n_kv=2, g=2), [300, 37, 1]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_noalloc_decode_matches_workspace_decode_on_two_calls(case):
    shape, seqlens = case
    inp = wl.make_decode_inputs(shape, seed=21, device=DEV, act="unit", seqlens=seqlens)
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    args = (inp["c_cache"], inp["kr_cache"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
            inp["gate_logits"], inp["seqlens"])
    need = gdla.decode_workspace_size(B=shape.B, T_max=shape.T, d_c=shape.d_c, d_rope=shape.d_R, n_kv=shape.n_kv,
                                      d_nope=shape.d_n, d_v=shape.d_v, g=shape.g)
    assert need <= _abi.GDLA_DECODE_NOALLOC_SCRATCH_BYTES
    ref = gdla.decode(*args, g=shape.g)
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.full_like(ref, float("nan"))
        gdla.decode_noalloc(*args, g=shape.g, out=y)
        torch.cuda.synchronize()
        # the same kernels on the same inputs: identical bytes (decode is bit-reproducible)
        assert torch.equal(y, ref), f"noalloc call {call}: max diff {(y.float() - ref.float()).abs().max()}"
        assert_parity(f64(y), f64(ref), torch.bfloat16, f"noalloc call {call}")


def test_noalloc_decode_replays_from_a_cuda_graph():
    # the serving-loop use: one eager call (the scratch address is looked up and the
    # kernels' attributes set), then the call captured in a CUDA graph and replayed
    # twice, with new query values copied into the captured input between replays
    shape = wl.DecodeShape("noalloc graph B=8 T=2048 g=2", B=8, T=2048, g=2)
    inp = wl.make_decode_inputs(shape, seed=23, device=DEV, act="unit", seqlens=[2048, 1500, 1, 129, 700, 2048, 64, 1024])
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    q_in = inp["q"].clone()
    q_next = wl.make_decode_inputs(shape, seed=24, device=DEV, act="unit")["q"]

    def args(q):
        return (inp["c_cache"], inp["kr_cache"], q, inp["w_ukv"], cos, sin, inp["lam_logits"], inp["gate_logits"],
                inp["seqlens"])

    ref1 = gdla.decode(*args(inp["q"]), g=shape.g)
    ref2 = gdla.decode(*args(q_next), g=shape.g)
    y = torch.empty_like(ref1)
    gdla.decode_noalloc(*args(q_in), g=shape.g, out=y)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gdla.decode_noalloc(*args(q_in), g=shape.g, out=y)
    for q_new, ref in ((inp["q"], ref1), (q_next, ref2)):
        q_in.copy_(q_new)
        y.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, ref)
    # the second replay against the oracle
    inp2 = dict(inp, q=q_next)
    ref_o = oracle_decode(inp2, g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    assert_parity(f64(y), ref_o, torch.bfloat16, "noalloc graph replay")
    del graph


def test_noalloc_rejects_a_batch_beyond_its_scratch():
    # 1024 sequences need 54 KB of query image each (57 MB) plus their partials;
    # the call must be refused before anything runs (the tensors stay unread)
    shape = wl.DecodeShape("noalloc too large", B=1024, T=64, g=2)
    e = lambda *s, dt=torch.bfloat16: torch.empty(s, dtype=dt, device=DEV)  # noqa: E731
    cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=DEV)
    with pytest.raises(gdla.GdlaError) as err:
        gdla.decode_noalloc(e(shape.B, shape.T, shape.d_c), e(shape.B, shape.T, shape.d_R),
                            e(shape.B, shape.H_q, shape.d_qk), e(shape.d_c, shape.n_kv * (shape.d_n + shape.d_v)),
                            cos, sin, e(shape.B, shape.n_S, dt=torch.float32), e(shape.B, shape.n_S, shape.d_v),
                            torch.full((shape.B,), shape.T, dtype=torch.int32, device=DEV), g=shape.g)
    assert err.value.code == _abi.GDLA_ERR_SCRATCH_LIMIT
    assert b"SCRATCH_LIMIT" in _abi.load().gdla_status_string(_abi.GDLA_ERR_SCRATCH_LIMIT)
    assert ctypes.sizeof(_abi.DecodeArgs) > 0
