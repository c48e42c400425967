"""The oracle against its stored regression fixture (tests/golden/tiny_prefill.json,
written by tests/golden/make_golden.py from the oracle alone)."""
import json
import os

import numpy as np

import oracle

FIX = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_prefill.json")


def test_oracle_matches_stored_fixture():
    doc = json.load(open(FIX))
    d = doc["dims"]
    inp = {k: np.array(v) for k, v in doc["inputs"].items()}
    L = d["L"]
    rb = np.zeros(L, dtype=np.int64)
    ri = np.arange(L)
    for name, mask, window in (("causal", oracle.MASK_CAUSAL, 0), ("sliding3", oracle.MASK_SLIDING, 3)):
        y = oracle.prefill_rows(c_kv=inp["c_kv"], gamma=inp["gamma"], k_rope=inp["k_rope"], w_ukv=inp["w_ukv"],
                                q_rows=inp["q"][rb, ri], lam_rows=inp["lam"][rb, ri], gate_rows=inp["gate"][rb, ri],
                                row_b=rb, row_i=ri, g=d["g"], d_n=d["d_n"], d_v=d["d_v"], mask=mask, window=window)
        np.testing.assert_allclose(y, np.array(doc["outputs"][name]), rtol=1e-12, atol=1e-14)
    chat = oracle.latent_norm(inp["c_kv"][0], inp["gamma"], d["eps"])
    krr = np.stack([oracle.rope(inp["k_rope"][0, j], j) for j in range(L)])
    yd = oracle.decode_seq(c_hat=chat, k_r_rot=krr, q=inp["q"][0, L - 1], w_ukv=inp["w_ukv"], lam=inp["lam"][0, L - 1],
                           gate=inp["gate"][0, L - 1], g=d["g"], d_n=d["d_n"], d_v=d["d_v"])
    np.testing.assert_allclose(yd, np.array(doc["outputs"]["decode_last"]), rtol=1e-12, atol=1e-14)
    # the sliding row 5 with W=3 sees tokens 3..5 only; rows 0..2 equal the causal ones
    np.testing.assert_array_equal(np.array(doc["outputs"]["sliding3"])[:3], np.array(doc["outputs"]["causal"])[:3])
