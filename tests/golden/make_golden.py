"""Writes tests/golden/tiny_prefill.json: a small GDLA prefill case (causal and
sliding window W=3) and a decode case, inputs drawn from a seeded numpy
generator, outputs computed by the fp64 oracle only. It guards the oracle's
arithmetic against silent drift; any intended change to that arithmetic must
regenerate this file and say, in its commit message, which passage of the
layer's statement justifies it.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import math
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
import oracle  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_prefill.json")


def make():
    rng = np.random.default_rng(20260812)
    B, L, d_c, d_R, n_kv, d_n, d_v, g = 1, 6, 4, 4, 2, 3, 2, 2
    n_S = g * n_kv
    inp = dict(
        c_kv=rng.standard_normal((B, L, d_c)).round(4),
        gamma=(1 + 0.1 * rng.standard_normal(d_c)).round(4),
        k_rope=rng.standard_normal((B, L, d_R)).round(4),
        w_ukv=(rng.standard_normal((d_c, n_kv * (d_n + d_v))) / math.sqrt(d_c)).round(4),
        q=rng.standard_normal((B, L, n_S + n_kv, d_n + d_R)).round(4),
        lam=rng.standard_normal((B, L, n_S)).round(4),
        gate=rng.standard_normal((B, L, n_S, d_v)).round(4),
    )
    rb = np.zeros(L, dtype=np.int64)
    ri = np.arange(L)
    outs = {}
    for name, mask, window in (("causal", oracle.MASK_CAUSAL, 0), ("sliding3", oracle.MASK_SLIDING, 3)):
        y = oracle.prefill_rows(c_kv=inp["c_kv"], gamma=inp["gamma"], k_rope=inp["k_rope"], w_ukv=inp["w_ukv"],
                                q_rows=inp["q"][rb, ri], lam_rows=inp["lam"][rb, ri], gate_rows=inp["gate"][rb, ri],
                                row_b=rb, row_i=ri, g=g, d_n=d_n, d_v=d_v, mask=mask, window=window)
        outs[name] = y.tolist()
    chat = oracle.latent_norm(inp["c_kv"][0], inp["gamma"], oracle.DEFAULT_EPS)
    krr = np.stack([oracle.rope(inp["k_rope"][0, j], j) for j in range(L)])
    outs["decode_last"] = oracle.decode_seq(c_hat=chat, k_r_rot=krr, q=inp["q"][0, L - 1], w_ukv=inp["w_ukv"],
                                            lam=inp["lam"][0, L - 1], gate=inp["gate"][0, L - 1], g=g, d_n=d_n,
                                            d_v=d_v).tolist()
    doc = {
        "about": "GDLA forward (Motif 3: Technical Report, Architecture), oracle-written regression fixture",
        "dims": dict(B=B, L=L, d_c=d_c, d_R=d_R, n_kv=n_kv, d_n=d_n, d_v=d_v, g=g, eps=oracle.DEFAULT_EPS,
                     rope_base=oracle.DEFAULT_ROPE_BASE),
        "inputs": {k: v.tolist() for k, v in inp.items()},
        "outputs": outs,
    }
    return doc


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump(make(), f, indent=1)
    print("wrote", OUT)
