"""The Python binding's argument checks on CPU (no GPU): tensors that the C ABI
would read as device memory must be CUDA tensors, the host-buffer prefill takes
its activations as CPU tensors, and every tensor must be contiguous. These checks
raise before the library is called."""
import pytest
import torch

import differential_latent_attention_gdla_b200 as gdla
from differential_latent_attention_gdla_b200 import workloads as wl

SHAPE = wl.PrefillShape("binding", B=1, L=64, n_kv=2, g=2)


def _inputs():
    inp = wl.make_prefill_inputs(SHAPE, seed=2)
    cos = torch.zeros((SHAPE.L, SHAPE.d_R // 2))
    return inp, cos


def test_device_entry_points_reject_cpu_tensors():
    inp, cos = _inputs()
    with pytest.raises(ValueError, match="CUDA device tensors"):
        gdla.prefill(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, cos,
                     inp["lam_logits"], inp["gate_logits"], g=SHAPE.g)
    kv = torch.zeros((1, SHAPE.L, SHAPE.n_kv, SHAPE.d_n + SHAPE.d_v), dtype=torch.bfloat16)
    kr = torch.zeros((1, SHAPE.L, SHAPE.d_R), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device tensors"):
        gdla.attend(inp["q"], kv, kr, cos, cos, inp["lam_logits"], inp["gate_logits"], g=SHAPE.g)


def test_host_prefill_wants_parameters_on_the_device():
    # activations on the host are accepted; gamma (a parameter) on the host is not
    inp, cos = _inputs()
    with pytest.raises(ValueError, match="CUDA device tensors"):
        gdla.prefill_host(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, cos,
                          inp["lam_logits"], inp["gate_logits"], g=SHAPE.g, out=torch.empty(1))


def test_host_prefill_rejects_non_contiguous_activations():
    # (c_kv is the first pointer taken, so its check runs before the device-side ones)
    inp, cos = _inputs()
    c_nc = inp["c_kv"].transpose(1, 2).contiguous().transpose(1, 2)  # same shape, column-major
    assert not c_nc.is_contiguous()
    with pytest.raises(ValueError, match="contiguous"):
        gdla.prefill_host(c_nc, inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, cos,
                          inp["lam_logits"], inp["gate_logits"], g=SHAPE.g, out=torch.empty(1))


def test_unsupported_dtype_is_rejected():
    inp, cos = _inputs()
    with pytest.raises(ValueError, match="dtype"):
        gdla.prefill(inp["c_kv"].half(), inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, cos,
                     inp["lam_logits"], inp["gate_logits"], g=SHAPE.g)


def test_gates_binding_checks():
    # neither half requested, and CPU tensors where the library reads device memory
    with pytest.raises(ValueError, match="c_q"):
        gdla.gates(n_signal=4)
    c_q = torch.zeros((2, 8, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device tensors"):
        gdla.gates(c_q, torch.ones(64, dtype=torch.bfloat16), torch.zeros((64, 128), dtype=torch.bfloat16),
                   n_signal=4, d_v=32)
