"""The binding's RoPE table set-up against the oracle's own tables (CPU only).

The kernels take cos/sin tables and the softmax scale as inputs, so a rescaled
RoPE such as YaRN ("Open-Source Frontier Models: Architecture and Benchmarks of
Rnj-1 and Motif-2", section 2) is only a different set of tables plus a
different scale. The binding builds them in its own code; here they must agree
with the oracle's (which are pinned in test_oracle_pins.py) to fp32 rounding."""
import numpy as np
import pytest

import differential_latent_attention_gdla_b200 as gdla
import oracle


def test_plain_tables_match_oracle():
    c, s = gdla.rope_tables(5000, 64, device="cpu")
    co, so = oracle.rope_table(5000, 64)
    assert np.abs(c.double().numpy() - co).max() < 1e-6
    assert np.abs(s.double().numpy() - so).max() < 1e-6


@pytest.mark.parametrize("factor,orig,beta_fast,beta_slow", [(16.0, 4096, 32.0, 1.0), (64.0, 4096, 32.0, 1.0),
                                                             (8.0, 64, 16.0, 2.0)])
def test_yarn_tables_match_oracle(factor, orig, beta_fast, beta_slow):
    c, s = gdla.yarn_rope_tables(6000, 64, factor, orig, beta_fast=beta_fast, beta_slow=beta_slow, device="cpu")
    co, so = oracle.rope_table_freq(6000, oracle.yarn_inv_freq(64, factor, orig, beta_fast=beta_fast,
                                                              beta_slow=beta_slow))
    assert np.abs(c.double().numpy() - co).max() < 1e-6
    assert np.abs(s.double().numpy() - so).max() < 1e-6


def test_yarn_factor_one_tables_equal_plain():
    c1, s1 = gdla.yarn_rope_tables(3000, 64, 1.0, 4096, device="cpu")
    c0, s0 = gdla.rope_tables(3000, 64, device="cpu")
    assert np.abs((c1 - c0).numpy()).max() < 1e-7 and np.abs((s1 - s0).numpy()).max() < 1e-7


def test_yarn_mscale_matches_oracle():
    for f in (0.5, 1.0, 4.0, 64.0):
        assert gdla.yarn_mscale(f) == pytest.approx(oracle.yarn_mscale(f), rel=1e-15)
