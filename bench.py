#!/usr/bin/env python
"""GDLA forward throughput on B200: prefill TFLOP/s and decode GB/s.

One step is one pass of the whole hot path on synthetic inputs already resident
in HBM:
  * prefill of B=1, L=32768, g=3 (48 signal + 16 noise heads, 16 KV heads,
    d_c=512, d_qk=192, d_v=128), full causal mask, through gdla_latent_expand
    then gdla_attend (the two halves of gdla_prefill);
  * decode of B=64 sequences over a 32768-token latent cache, g=2, through
    gdla_decode.
`value` is the prefill's algorithmic TFLOP/s (expansion GEMM plus QK and PV
over the visible pairs, all ranks' work over the slowest rank's time);
`decode` carries the decode's algorithmic GB/s (the cache read once). Inputs are
larger than L2 (q alone is 805 MB), so no flush is needed between steps.
`e2e` is the same prefill through gdla_prefill_host: the activations start in
page-locked host memory and Y ends there, and the call overlaps the chunked
copies with the kernels.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With --impl reference the fp64 CPU oracle is timed on a bounded sample of the
same prefill workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDLA prefill TFLOP/s & decode GB/s at 1 B200, % of bf16/HBM roofline"
PREFILL_NAME = "b1_l32k_g3"
DECODE_NAME = "b64_t32k"
CSRC = os.path.join(ROOT, "differential_latent_attention_gdla_b200", "csrc")

# DRAM bytes (read + write) per launch from one ncu capture of the full-size workload
# (dram__bytes_read.sum + dram__bytes_write.sum), with a hash of the kernel sources they
# were taken on: once a kernel changes, its figure no longer applies and the bench
# reports null.
MEASURED_TRAFFIC = {
    ("attn_tc_kernel", "b1_l32k_g3"): (2.165e9, ("attn_tc.cu", "sm100.cuh"), "79c179dd071b6bbd"),
    ("decode_tc_kernel", "b64_t32k"): (2.474e9, ("decode_tc.cu", "sm100.cuh"), "5de5419009465d0a"),
}


def measured_traffic(kernel: str, workload: str):
    """The captured DRAM bytes of one launch, or None if absent or taken on other sources."""
    import hashlib

    entry = MEASURED_TRAFFIC.get((kernel, workload))
    if entry is None:
        return None
    nbytes, files, digest = entry
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return nbytes if h.hexdigest()[:16] == digest else None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-chunk", type=int, default=0, help="tokens per host-copy chunk (0: library default)")
    ap.add_argument("--prefill", default=PREFILL_NAME, help="prefill workload name (profiling uses smaller ones)")
    ap.add_argument("--decode", default=DECODE_NAME, help="decode workload name")
    return ap.parse_args()


def max_over_ranks(values, world: int, device="cpu"):
    """Element-wise max of per-rank timings (every rank calls this once)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def weak_scaling_value(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / seconds


def rank_seed(seed: int, rank: int, which: str) -> int:
    """Each rank draws an independent problem of the same shape."""
    return seed + rank + (1000 if which == "decode" else 0)


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "fallback": True}


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(shape, inp_cpu, n_rows: int, kv_groups):
    """Time the fp64 oracle on `n_rows` query rows (evenly spread over the
    sequence) of the KV groups `kv_groups`; returns (seconds, algorithmic flops
    of the sample, description, threads)."""
    import numpy as np

    import oracle

    L = shape.L
    rows = [(0, int(i)) for i in np.linspace(L // n_rows, L - 1, n_rows)]
    T = max(i for _, i in rows) + 1
    rb = np.array([r[0] for r in rows])
    ri = np.array([r[1] for r in rows])
    f = lambda t: t.double().numpy()  # noqa: E731
    args = dict(c_kv=f(inp_cpu["c_kv"][:, :T]), gamma=f(inp_cpu["gamma"]), k_rope=f(inp_cpu["k_rope"][:, :T]),
                w_ukv=f(inp_cpu["w_ukv"]), q_rows=f(inp_cpu["q"][rb, ri]), lam_rows=f(inp_cpu["lam_logits"][rb, ri]),
                gate_rows=f(inp_cpu["gate_logits"][rb, ri]), row_b=rb, row_i=ri, g=shape.g, d_n=shape.d_n,
                d_v=shape.d_v, kv_sel=list(kv_groups))
    t0 = time.perf_counter()
    oracle.prefill_rows(**args)
    dt = time.perf_counter() - t0
    G = len(kv_groups)
    flops = 2.0 * T * shape.d_c * G * (shape.d_n + shape.d_v)
    flops += sum(2.0 * (shape.d_qk + shape.d_v) * (i + 1) * G * (shape.g + 1) for _, i in rows)
    desc = (f"{n_rows} query rows evenly spread over [0, {L}) of the B={shape.B} L={L} g={shape.g} {shape.mask} "
            f"prefill, {G} of {shape.n_kv} KV groups ({G * (shape.g + 1)} heads), expansion of the {T} visible tokens")
    return dt, flops, desc, oracle.num_threads()


def run_reference(a):
    """The fp64 oracle on host cores, one bounded sample per step."""
    import torch

    from differential_latent_attention_gdla_b200 import workloads as wl

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    shape = wl.PREFILL[PREFILL_NAME]
    inp = wl.make_prefill_inputs(shape, seed=a.seed, device="cpu")
    times, flops, desc, thr = [], 0.0, "", 1
    for k in range(a.warmup + a.steps):
        dt, fl, desc, thr = oracle_sample(shape, inp, n_rows=8, kv_groups=[(4 * k + u) % shape.n_kv for u in range(4)])
        if k >= a.warmup:
            times.append(dt)
            flops = fl
    mean = sum(times) / len(times)
    value = flops / mean / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": mean * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"prefill {PREFILL_NAME}: bounded oracle sample per step", "sample": desc},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    del torch
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index: int):
        self.proc = None
        # raw samples go to $GDLA_CLOCKS_DIR/clocks_rank<i>.csv when set (to keep them), else to /tmp
        out_dir = os.environ.get("GDLA_CLOCKS_DIR")
        self.path = (os.path.join(out_dir, f"clocks_rank{index}.csv") if out_dir
                     else f"/tmp/gdla_clocks_{os.getpid()}_{index}.csv")
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        load = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------- our path
def run_ours(a):
    import torch
    import torch.distributed as dist

    import differential_latent_attention_gdla_b200 as gdla
    from differential_latent_attention_gdla_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    P = wl.PREFILL[a.prefill]
    D = wl.DECODE[a.decode]
    # every rank runs its own independent problem (weak scaling, no collective on the data path)
    pin = wl.make_prefill_inputs(P, seed=rank_seed(a.seed, rank, "prefill"), device=dev)
    din = wl.make_decode_inputs(D, seed=rank_seed(a.seed, rank, "decode"), device=dev)
    cos, sin = gdla.rope_tables(max(P.L, D.T), P.d_R, device=dev)
    kv = torch.empty((P.B, P.L, P.n_kv, P.d_n + P.d_v), dtype=torch.bfloat16, device=dev)
    krot = torch.empty((P.B, P.L, P.d_R), dtype=torch.bfloat16, device=dev)
    chat = torch.empty((P.B, P.L, P.d_c), dtype=torch.bfloat16, device=dev)
    y = torch.empty((P.B, P.L, P.n_S, P.d_v), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(256, dtype=torch.uint8, device=dev)
    yd = torch.empty((D.B, D.n_S, D.d_v), dtype=torch.bfloat16, device=dev)
    dws = torch.empty(gdla.decode_workspace_size(B=D.B, T_max=D.T, d_c=D.d_c, d_rope=D.d_R, n_kv=D.n_kv,
                                                 d_nope=D.d_n, d_v=D.d_v, g=D.g), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def expand():
        gdla.latent_expand(pin["c_kv"], pin["gamma"], pin["k_rope"], pin["w_ukv"], cos, sin, n_kv=P.n_kv,
                           d_nope=P.d_n, d_v=P.d_v, kv_out=kv, k_rope_out=krot, c_hat_out=chat, stream=stream)

    def attend():
        gdla.attend(pin["q"], kv, krot, cos, sin, pin["lam_logits"], pin["gate_logits"], g=P.g, mask=P.mask,
                    window=P.window, out=y, status=status, stream=stream)

    def decode():
        gdla.decode(din["c_cache"], din["kr_cache"], din["q"], din["w_ukv"], cos, sin, din["lam_logits"],
                    din["gate_logits"], din["seqlens"], g=D.g, out=yd, workspace=dws, stream=stream)

    launches_per_step = 2 + 1 + 3  # norm+rope, expansion GEMM | attention | absorb, split-KV, combine
    for _ in range(a.warmup):
        expand()
        attend()
        decode()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(a.steps)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for k in range(a.steps):
        ev[k][0].record(stream)
        expand()
        ev[k][1].record(stream)
        attend()
        ev[k][2].record(stream)
        decode()
        ev[k][3].record(stream)
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - t0
    clk = clocks.stop()
    if int(gdla.workspace_status(status)) != 0 or int(gdla.workspace_status(dws)) != 0:
        raise RuntimeError("device status word reports a failed wait")

    t_exp = sum(e[0].elapsed_time(e[1]) for e in ev) / a.steps
    t_att = sum(e[1].elapsed_time(e[2]) for e in ev) / a.steps
    t_dec = sum(e[2].elapsed_time(e[3]) for e in ev) / a.steps
    t_step = ev[0][0].elapsed_time(ev[-1][3]) / a.steps
    t_exp, t_att, t_dec, t_step = max_over_ranks([t_exp, t_att, t_dec, t_step], world, dev)

    pf = P.algorithmic_flops()
    f_exp = 2.0 * P.B * P.L * P.d_c * P.n_kv * (P.d_n + P.d_v)
    f_att = pf - f_exp
    db = D.algorithmic_bytes()
    pk = peaks()
    value = weak_scaling_value(pf, world, (t_exp + t_att) * 1e-3) / 1e12
    att_tflops = f_att / (t_att * 1e-3) / 1e12
    dec_gbs = weak_scaling_value(db, world, t_dec * 1e-3) / 1e9

    # end to end through the public host-buffer call (gdla_prefill_host): the activations
    # start in page-locked host memory and Y ends there; every copy is inside the timed region
    e2e = None
    if a.e2e_steps > 0:
        keys = ["c_kv", "k_rope", "q", "lam_logits", "gate_logits"]
        host = {k: pin[k].cpu().pin_memory() for k in keys}
        yh = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
        ws = torch.empty(gdla.prefill_host_workspace_size(B=P.B, L=P.L, d_c=P.d_c, d_rope=P.d_R, n_kv=P.n_kv,
                                                          d_nope=P.d_n, d_v=P.d_v, g=P.g,
                                                          chunk_tokens=a.e2e_chunk),
                         dtype=torch.uint8, device=dev)

        def e2e_step():
            gdla.prefill_host(host["c_kv"], pin["gamma"], host["k_rope"], host["q"], pin["w_ukv"], cos, sin,
                              host["lam_logits"], host["gate_logits"], g=P.g, mask=P.mask, window=P.window,
                              chunk_tokens=a.e2e_chunk, out=yh, workspace=ws, stream=stream)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(a.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        (t,) = max_over_ranks([e0.elapsed_time(e1) / a.e2e_steps], world, dev)
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        e2e = {"value": weak_scaling_value(pf, world, t * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": yh.numel() * yh.element_size(), "ms_per_step": t}
        if int(gdla.workspace_status(ws)) != 0:
            raise RuntimeError("device status word reports a failed wait (host-buffer prefill)")
        e2e["chunk_tokens"] = a.e2e_chunk if a.e2e_chunk > 0 else "library default"
        del ws, host

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        inp_cpu = {k: v.cpu() for k, v in pin.items()}
        dt, fl, desc, thr = oracle_sample(P, inp_cpu, n_rows=24, kv_groups=list(range(P.n_kv)))
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": desc,
               "seconds": dt}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": t_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) recipe)",
            "config": {"workload": f"prefill {P.name} (value, TFLOP/s) + decode {D.name} "
                                   f"(decode.value, GB/s)", "prefill": a.prefill, "decode": a.decode,
                       "l2": "inputs larger than L2 (q 805 MB, cache 2.4 GB); no flush",
                       "parallelism": f"{world} independent replicas (weak scaling)"},
            "prefill": {"ms": t_exp + t_att, "expand_ms": t_exp, "attend_ms": t_att,
                        "algorithmic_tflop": pf / 1e12},
            "decode": {"value": dec_gbs, "unit": "GB/s", "ms": t_dec, "algorithmic_gb": db / 1e9,
                       "roofline": {"bound": "hbm", "achieved": dec_gbs / world, "peak": pk["hbm_gbs"],
                                    "unit": "GB/s", "frac": dec_gbs / world / pk["hbm_gbs"],
                                    "peak_kind": "measured copy", "kernel": "whole gdla_decode call",
                                    "traffic": measured_traffic("decode_tc_kernel", a.decode),
                                    "traffic_kernel": "decode_tc_kernel (split-KV pass)"}},
            "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": pk["bf16_tflops_sustained"],
                         "unit": "TFLOP/s", "frac": att_tflops / pk["bf16_tflops_sustained"],
                         "traffic": measured_traffic("attn_tc_kernel", a.prefill),
                         "kernel": "gdla_attend (attention + differential epilogue)",
                         "peak_kind": "measured sustained bf16 (burst %.1f: frac %.3f)" % (
                             pk["bf16_tflops"], att_tflops / pk["bf16_tflops"])},
            "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": launches_per_step * a.steps, "clocks": clk,
            "wall_s": wall,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    a = parse()
    if a.impl == "reference":
        return run_reference(a)
    return run_ours(a)


if __name__ == "__main__":
    sys.exit(main())
