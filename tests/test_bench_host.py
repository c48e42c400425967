"""The benchmark's host logic on CPU (no GPU): the DRAM-traffic table is used only
on the sources it was captured on, the oracle sample counts the FLOPs of what it
computes, and the reference arm prints one well-formed JSON line."""
import contextlib
import hashlib
import io
import json
import os
import types

import numpy as np
import pytest

import bench
from differential_latent_attention_gdla_b200 import workloads as wl


def test_traffic_entries_name_existing_sources():
    for (kernel, workload), (nbytes, files, digest) in bench.MEASURED_TRAFFIC.items():
        assert nbytes > 1e8 and len(digest) == 16
        for f in files:
            assert os.path.exists(os.path.join(bench.CSRC, f)), f


def test_traffic_is_dropped_once_the_kernel_source_changes(monkeypatch):
    files = ("attn_tc.cu", "sm100.cuh")
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(bench.CSRC, f), "rb").read())
    good = h.hexdigest()[:16]
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {("k", "w"): (3.0e9, files, good),
                                                    ("k", "stale"): (3.0e9, files, "0" * 16)})
    assert bench.measured_traffic("k", "w") == 3.0e9
    assert bench.measured_traffic("k", "stale") is None
    assert bench.measured_traffic("k", "absent") is None


def test_oracle_sample_counts_the_flops_it_computes():
    shape = wl.PREFILL["tiny_fp32"]
    inp = wl.make_prefill_inputs(shape, seed=1)
    dt, flops, desc, thr = bench.oracle_sample(shape, inp, n_rows=8, kv_groups=[0, 2])
    rows = [int(i) for i in np.linspace(shape.L // 8, shape.L - 1, 8)]
    T = max(rows) + 1
    want = 2.0 * T * shape.d_c * 2 * (shape.d_n + shape.d_v)  # expansion of two KV groups
    for i in rows:  # causal: row i sees i + 1 keys, in g + 1 heads of each group
        want += 2.0 * (shape.d_qk + shape.d_v) * (i + 1) * 2 * (shape.g + 1)
    assert flops == pytest.approx(want)
    assert dt > 0 and thr >= 1
    assert f"L={shape.L}" in desc and "2 of 4 KV groups" in desc


def test_reference_arm_prints_one_json_line(monkeypatch):
    monkeypatch.setattr(bench, "PREFILL_NAME", "tiny_fp32")
    monkeypatch.delenv("RANK", raising=False)
    args = types.SimpleNamespace(seed=0, warmup=1, steps=2, gpus=1)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(args) == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(types.SimpleNamespace(seed=0, warmup=1, steps=1, gpus=2)) == 0
    assert buf.getvalue() == ""
