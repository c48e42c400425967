"""Failure detection on the GPU without a fault: every device-side wait in the
kernels is bounded (about a second), and one that runs out records
GDLA_ERR_TIMEOUT in the caller's status word instead of hanging. The diagnostic
entry point runs such a wait on an mbarrier that nothing ever arrives on; the
host must read the timeout, and the context must stay usable afterwards."""
import time

import pytest
import torch

import differential_latent_attention_gdla_b200 as gdla
from differential_latent_attention_gdla_b200 import _abi
from differential_latent_attention_gdla_b200 import workloads as wl
from gdla_testutil import assert_parity, f64, oracle_prefill_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_stalled_wait_ends_reports_timeout_and_context_survives():
    status = torch.full((256,), 0x55, dtype=torch.uint8, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    gdla.diag_wait_timeout(status)
    code = gdla.workspace_status(status)  # synchronises the stream
    dt = time.perf_counter() - t0
    assert code == _abi.GDLA_ERR_TIMEOUT
    words = status.view(torch.int32).cpu()
    assert int(words[1]) == 901            # the tag of the wait that gave up
    assert 0.5 < dt < 10.0, dt             # it waited for its limit, then ended
    # the CUDA context is intact: a prefill afterwards runs and is correct
    shape = wl.PrefillShape("after timeout", B=1, L=130, n_kv=2, g=3)
    inp = wl.make_prefill_inputs(shape, seed=41, device=DEV)
    cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=DEV)
    y = gdla.prefill(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["q"], inp["w_ukv"], cos, sin, inp["lam_logits"],
                     inp["gate_logits"], g=shape.g)
    torch.cuda.synchronize()
    ref = oracle_prefill_rows(inp, [(0, i) for i in range(shape.L)], g=shape.g, d_nope=shape.d_n, d_v=shape.d_v)
    assert_parity(f64(y).reshape(ref.shape), ref, torch.bfloat16, shape.name)


def test_diag_rejects_misaligned_status_word():
    buf = torch.zeros(512, dtype=torch.uint8, device=DEV)
    with pytest.raises(gdla.GdlaError) as err:
        gdla.diag_wait_timeout(buf[16:])
    assert err.value.code == _abi.GDLA_ERR_INVALID_ARG
