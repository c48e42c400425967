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
over the visible pairs, all ranks' work over the slowest rank's time). Inputs
are larger than L2 (q alone is 805 MB, the decode cache 2.4 GB), so no flush is
needed between steps.

Beside the timed steps (outside their timed region):
  * `decode`: the decode call timed in its own loop after its own warm-up, before the
    prefill steps (the `roofline` of the decode, with the SM clocks sampled over that
    loop), and its time inside the steps (`in_step_ms`), where it follows the
    power-capped prefill;
  * `prefill_cfg2` (B=4 L=4096 g=2 causal), `prefill_cfg4` (B=2 L=65536 g=2,
    4096-token window) and the report's own layout, g=4 (80 heads):
    `prefill_g4_swa128` (128-token window), `decode_g4`, and `gates` (gate and lambda
    logits for the bench prefill's tokens);
  * `e2e`: the same prefill through gdla_prefill_host (activations start in
    page-locked host memory, Y ends there; the chunked copies overlap the
    kernels), and `e2e.decode`: q, lambda and gate copied in from page-locked
    host memory, gdla_decode, Y copied back, every step.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
With --impl reference the fp64 CPU oracle is timed on a bounded sample of the
same prefill workload (the sample of the `cpu_baseline` leg), on this host's cores.
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
    ("attn_tc_kernel", "b1_l32k_g3"): (2.247e9, ("attn_tc.cu", "sm100.cuh"), "72d70f98881b0bb9"),
    ("decode_tc_kernel", "b64_t32k"): (2.433e9, ("decode_tc.cu", "sm100.cuh"), "45965a23734dcc7d"),
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
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="skip the other configurations (profiling runs of one workload)")
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


NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16 (NVIDIA's figure without 2:4 sparsity)
NOMINAL_HBM_GBS = 8000.0      # the "~8 TB/s" HBM3e figure


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "fallback": True}


def tensor_roofline(tflops: float, pk: dict) -> dict:
    """A tensor-bound kernel timed alone (milliseconds, not a seconds-long loop):
    the fraction of the measured burst bf16 peak; the sustained and nominal
    fractions beside it."""
    return {"bound": "tensor", "achieved": tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": tflops / pk["bf16_tflops"],
            "peak_kind": "measured burst bf16" + (" (fallback)" if pk.get("fallback") else ""),
            "frac_of_sustained": tflops / pk["bf16_tflops_sustained"],
            "frac_of_nominal": tflops / NOMINAL_BF16_TFLOPS}


def hbm_roofline(gbs: float, pk: dict) -> dict:
    return {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
            "peak_kind": "measured copy" + (" (fallback)" if pk.get("fallback") else ""),
            "frac_of_nominal": gbs / NOMINAL_HBM_GBS}


GATE_D_X = 2048  # width of the layer input x of the lambda projection (the caller's choice)
DECODE_WARMUP, DECODE_STEPS = 100, 600  # the decode's own loop (a call is ~0.5 ms)

# The cpu_baseline leg and the reference arm time the oracle on the same sample.
ORACLE_ROWS = 24


def oracle_kv_groups(shape):
    return list(range(shape.n_kv))


def bench_config(prefill_key: str, decode_key: str, world: int) -> dict:
    """The workload description both arms print (workload keys of workloads.py)."""
    from differential_latent_attention_gdla_b200 import workloads as wl

    P, D = wl.PREFILL[prefill_key], wl.DECODE[decode_key]
    return {"workload": f"prefill {P.name} (value, TFLOP/s) + decode {D.name} (decode.value, GB/s)",
            "prefill": prefill_key, "decode": decode_key,
            "l2": "inputs larger than L2 (q 805 MB, cache 2.4 GB); no flush",
            "parallelism": f"{world} independent replicas (weak scaling)"}


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
    """The fp64 oracle on host cores, one bounded sample per step: the sample of
    the cpu_baseline leg (ORACLE_ROWS rows of every KV group)."""
    import torch

    from differential_latent_attention_gdla_b200 import workloads as wl

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    shape = wl.PREFILL[PREFILL_NAME]
    inp = wl.make_prefill_inputs(shape, seed=a.seed, device="cpu")
    times, flops, desc, thr = [], 0.0, "", 1
    for k in range(a.warmup + a.steps):
        dt, fl, desc, thr = oracle_sample(shape, inp, n_rows=ORACLE_ROWS, kv_groups=oracle_kv_groups(shape))
        if k >= a.warmup:
            times.append(dt)
            flops = fl
    mean = sum(times) / len(times)
    value = flops / mean / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": mean * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) recipe)",
            "config": bench_config(PREFILL_NAME, DECODE_NAME, 1),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    del torch
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index: int, tag: str = ""):
        self.proc = None
        # raw samples go to $GDLA_CLOCKS_DIR/clocks_<tag>rank<i>.csv when set (to keep them), else to /tmp
        out_dir = os.environ.get("GDLA_CLOCKS_DIR")
        pre = f"{tag}_" if tag else ""
        self.path = (os.path.join(out_dir, f"clocks_{pre}rank{index}.csv") if out_dir
                     else f"/tmp/gdla_clocks_{pre}{os.getpid()}_{index}.csv")
        q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "20", "-i", str(index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, window=None):
        """Summary of the samples; with window = (t0, t1) (host time.time()), only the
        samples taken inside it."""
        import datetime

        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(p[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if window is not None and not (window[0] <= ts <= window[1]):
                    continue
                sm.append(float(p[2]))
                mx.append(float(p[3]))
            except ValueError:
                continue
            for n, v in zip(names, p[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        load = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------- our path
def time_loop(fn, steps: int, warmup: int, stream):
    """Mean milliseconds of fn() over `steps` calls after `warmup` untimed ones
    (CUDA events on `stream`, synchronised on both sides)."""
    import torch

    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


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
    pk = peaks()
    stream = torch.cuda.current_stream()

    def prefill_case(shape, seed):
        """Inputs and the two calls (expansion, attention) of one prefill workload."""
        inp = wl.make_prefill_inputs(shape, seed=seed, device=dev)
        cos, sin = gdla.rope_tables(shape.L, shape.d_R, device=dev)
        kv = torch.empty((shape.B, shape.L, shape.n_kv, shape.d_n + shape.d_v), dtype=torch.bfloat16, device=dev)
        krot = torch.empty((shape.B, shape.L, shape.d_R), dtype=torch.bfloat16, device=dev)
        chat = torch.empty((shape.B, shape.L, shape.d_c), dtype=torch.bfloat16, device=dev)
        y = torch.empty((shape.B, shape.L, shape.n_S, shape.d_v), dtype=torch.bfloat16, device=dev)
        status = torch.zeros(256, dtype=torch.uint8, device=dev)

        def expand():
            gdla.latent_expand(inp["c_kv"], inp["gamma"], inp["k_rope"], inp["w_ukv"], cos, sin, n_kv=shape.n_kv,
                               d_nope=shape.d_n, d_v=shape.d_v, kv_out=kv, k_rope_out=krot, c_hat_out=chat,
                               stream=stream)

        def attend():
            gdla.attend(inp["q"], kv, krot, cos, sin, inp["lam_logits"], inp["gate_logits"], g=shape.g,
                        mask=shape.mask, window=shape.window, out=y, status=status, stream=stream)

        return inp, (cos, sin), expand, attend, status

    def decode_case(shape, seed):
        din = wl.make_decode_inputs(shape, seed=seed, device=dev)
        cos, sin = gdla.rope_tables(shape.T, shape.d_R, device=dev)
        yd = torch.empty((shape.B, shape.n_S, shape.d_v), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(gdla.decode_workspace_size(B=shape.B, T_max=shape.T, d_c=shape.d_c, d_rope=shape.d_R,
                                                    n_kv=shape.n_kv, d_nope=shape.d_n, d_v=shape.d_v, g=shape.g),
                         dtype=torch.uint8, device=dev)

        def decode():
            gdla.decode(din["c_cache"], din["kr_cache"], din["q"], din["w_ukv"], cos, sin, din["lam_logits"],
                        din["gate_logits"], din["seqlens"], g=shape.g, mask=shape.mask, window=shape.window,
                        out=yd, workspace=ws, stream=stream)

        return din, (cos, sin), yd, ws, decode

    # every rank runs its own independent problem (weak scaling, no collective on the data path)
    pin, pcs, expand, attend, status = prefill_case(P, rank_seed(a.seed, rank, "prefill"))
    din, dcs, yd, dws, decode = decode_case(D, rank_seed(a.seed, rank, "decode"))

    launches_per_step = 2 + 1 + 3  # norm+rope, expansion GEMM | attention | absorb, split-KV, combine

    # ---- the decode call in its own loop, at its own steady state (its own warm-up,
    # not right after the power-capped prefill, whose decode time is `in_step_ms`)
    # (SM clocks sampled over it too: nvidia-smi gets half a second to start sampling)
    dclocks = ClockSampler(local, "decode")
    time.sleep(0.5)
    w0 = time.time()
    t_dec_alone = time_loop(decode, max(a.steps, DECODE_STEPS), max(a.warmup, DECODE_WARMUP), stream)
    dclk = dclocks.stop((w0, time.time()))
    if int(gdla.workspace_status(dws)) != 0:
        raise RuntimeError("device status word reports a failed wait (decode)")

    for _ in range(a.warmup):
        expand()
        attend()
        decode()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(a.steps)]
    clocks = ClockSampler(local)
    time.sleep(0.5)  # nvidia-smi's first samples land before the timed steps
    barrier()
    torch.cuda.synchronize()
    w0 = time.time()
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
    clk = clocks.stop((w0, time.time()))
    if int(gdla.workspace_status(status)) != 0 or int(gdla.workspace_status(dws)) != 0:
        raise RuntimeError("device status word reports a failed wait")

    t_exp = sum(e[0].elapsed_time(e[1]) for e in ev) / a.steps
    t_att = sum(e[1].elapsed_time(e[2]) for e in ev) / a.steps
    t_dec = sum(e[2].elapsed_time(e[3]) for e in ev) / a.steps
    t_step = ev[0][0].elapsed_time(ev[-1][3]) / a.steps

    # ---- measured after the timed steps, outside their region
    # end to end through host buffers: the prefill through gdla_prefill_host, and the
    # decode with its per-token inputs copied in and Y copied back every step
    e2e, t_e2e, t_e2e_dec, e2e_extra = None, 0.0, 0.0, {}
    if a.e2e_steps > 0:
        keys = ["c_kv", "k_rope", "q", "lam_logits", "gate_logits"]
        host = {k: pin[k].cpu().pin_memory() for k in keys}
        yh = torch.empty((P.B, P.L, P.n_S, P.d_v), dtype=torch.bfloat16, pin_memory=True)
        ws = torch.empty(gdla.prefill_host_workspace_size(B=P.B, L=P.L, d_c=P.d_c, d_rope=P.d_R, n_kv=P.n_kv,
                                                          d_nope=P.d_n, d_v=P.d_v, g=P.g,
                                                          chunk_tokens=a.e2e_chunk),
                         dtype=torch.uint8, device=dev)

        def e2e_step():
            gdla.prefill_host(host["c_kv"], pin["gamma"], host["k_rope"], host["q"], pin["w_ukv"], pcs[0], pcs[1],
                              host["lam_logits"], host["gate_logits"], g=P.g, mask=P.mask, window=P.window,
                              chunk_tokens=a.e2e_chunk, out=yh, workspace=ws, stream=stream)

        t_e2e = time_loop(e2e_step, a.e2e_steps, 1, stream)
        if int(gdla.workspace_status(ws)) != 0:
            raise RuntimeError("device status word reports a failed wait (host-buffer prefill)")
        h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
        e2e_extra["prefill"] = {"h2d_bytes_per_step": h2d, "d2h_bytes_per_step": yh.numel() * yh.element_size(),
                                "chunk_tokens": a.e2e_chunk if a.e2e_chunk > 0 else "library default"}
        del ws, host

        dkeys = ["q", "lam_logits", "gate_logits"]
        dhost = {k: din[k].cpu().pin_memory() for k in dkeys}
        ddev = {k: torch.empty_like(din[k]) for k in dkeys}
        ydh = torch.empty(yd.shape, dtype=yd.dtype, pin_memory=True)

        def e2e_decode():
            for k in dkeys:
                ddev[k].copy_(dhost[k], non_blocking=True)
            gdla.decode(din["c_cache"], din["kr_cache"], ddev["q"], din["w_ukv"], dcs[0], dcs[1],
                        ddev["lam_logits"], ddev["gate_logits"], din["seqlens"], g=D.g, out=yd, workspace=dws,
                        stream=stream)
            ydh.copy_(yd, non_blocking=True)

        t_e2e_dec = time_loop(e2e_decode, a.steps, a.warmup, stream)
        e2e_extra["decode"] = {"h2d_bytes_per_step": sum(dhost[k].numel() * dhost[k].element_size() for k in dkeys),
                               "d2h_bytes_per_step": ydh.numel() * ydh.element_size()}

    # the other prefill configurations and the report's own head layout (g = 4)
    extra_ms = {}
    if a.extras:
        for key, name in (("prefill_cfg2", "b4_l4k_g2"), ("prefill_cfg4", "b2_l64k_swa4k"),
                          ("prefill_g4_swa128", "b1_l32k_g4_swa128")):
            S = wl.PREFILL[name]
            _, _, ex, at, st = prefill_case(S, rank_seed(a.seed, rank, "prefill"))
            # the short workloads (about 1 ms a call) get more calls, so that a clock
            # excursion of a few ms does not decide their number
            n_t, n_w = (3, 2) if S.B * S.L >= 131072 else (20, 5)
            t_e = time_loop(ex, n_t, n_w, stream)
            t_a = time_loop(at, n_t, n_w, stream)
            if int(gdla.workspace_status(st)) != 0:
                raise RuntimeError(f"device status word reports a failed wait ({name})")
            extra_ms[key] = (name, S, t_e, t_a)
            torch.cuda.empty_cache()
        S = wl.DECODE["b64_t32k_g4"]
        _, _, _, ws4, dec4 = decode_case(S, rank_seed(a.seed, rank, "decode"))
        t4 = time_loop(dec4, DECODE_STEPS, DECODE_WARMUP, stream)
        if int(gdla.workspace_status(ws4)) != 0:
            raise RuntimeError("device status word reports a failed wait (decode g=4)")
        extra_ms["decode_g4"] = ("b64_t32k_g4", S, t4, None)
        # the gate logits (tensor cores) and lambda logits (HBM-bound) for the bench
        # prefill's tokens, with a 2048-wide layer input
        gi = wl.make_gate_inputs(P, d_x=GATE_D_X, seed=rank_seed(a.seed, rank, "prefill") + 7, device=dev)
        g_out = torch.empty((P.B, P.L, P.n_S, P.d_v), dtype=torch.bfloat16, device=dev)
        l_out = torch.empty((P.B, P.L, P.n_S), dtype=torch.float32, device=dev)

        def gate_call():
            gdla.gates(gi["c_q"], gi["gamma_q"], gi["w_g"], n_signal=P.n_S, d_v=P.d_v, gate_out=g_out)

        def lam_call():
            gdla.gates(x=gi["x"], w_lambda=gi["w_lambda"], n_signal=P.n_S, lam_out=l_out)
        extra_ms["gates"] = ("gates", None, time_loop(gate_call, 5, 3, stream), time_loop(lam_call, 10, 3, stream))
        del gi, g_out, l_out
        torch.cuda.empty_cache()

    vals = [t_exp, t_att, t_dec, t_step, t_dec_alone, t_e2e, t_e2e_dec]
    for key in sorted(extra_ms):
        vals += [extra_ms[key][2], extra_ms[key][3] or 0.0]
    vals = max_over_ranks(vals, world, dev)
    t_exp, t_att, t_dec, t_step, t_dec_alone, t_e2e, t_e2e_dec = vals[:7]

    pf = P.algorithmic_flops()
    f_exp = 2.0 * P.B * P.L * P.d_c * P.n_kv * (P.d_n + P.d_v)
    f_att = pf - f_exp
    db = D.algorithmic_bytes()
    value = weak_scaling_value(pf, world, (t_exp + t_att) * 1e-3) / 1e12
    att_tflops = f_att / (t_att * 1e-3) / 1e12
    dec_gbs = weak_scaling_value(db, world, t_dec_alone * 1e-3) / 1e9

    if a.e2e_steps > 0:
        e2e = {"value": weak_scaling_value(pf, world, t_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
               **e2e_extra["prefill"], "ms_per_step": t_e2e,
               "decode": {"value": weak_scaling_value(db, world, t_e2e_dec * 1e-3) / 1e9, "unit": "GB/s",
                          "ms_per_step": t_e2e_dec, **e2e_extra["decode"]}}

    extras = {}
    i = 7
    for key in sorted(extra_ms):
        name, S, t_first, t_second = extra_ms[key]
        te, ta = vals[i], vals[i + 1]
        i += 2
        if key == "gates":
            f_g = 2.0 * P.B * P.L * P.d_q * P.n_S * P.d_v
            b_l = P.B * P.L * (GATE_D_X * 2 + P.n_S * 4) + GATE_D_X * P.n_S * 2
            extras[key] = {"workload": f"gate and lambda logits, B={P.B} L={P.L}, d_q={P.d_q}, n_S={P.n_S}, "
                                       f"d_v={P.d_v}, d_x={GATE_D_X}",
                           "gate_ms": te, "gate_tflops": weak_scaling_value(f_g, world, te * 1e-3) / 1e12,
                           "gate_roofline": tensor_roofline(f_g / (te * 1e-3) / 1e12, pk),
                           "lambda_ms": ta, "lambda_gbs": weak_scaling_value(b_l, world, ta * 1e-3) / 1e9,
                           "lambda_roofline": hbm_roofline(b_l / (ta * 1e-3) / 1e9, pk)}
        elif t_second is None:  # a decode workload
            gbs = weak_scaling_value(S.algorithmic_bytes(), world, te * 1e-3) / 1e9
            extras[key] = {"workload": S.name, "value": gbs, "unit": "GB/s", "ms": te,
                           "roofline": hbm_roofline(gbs / world, pk)}
        else:
            fl = S.algorithmic_flops()
            fe = 2.0 * S.B * S.L * S.d_c * S.n_kv * (S.d_n + S.d_v)
            tf = weak_scaling_value(fl, world, (te + ta) * 1e-3) / 1e12
            extras[key] = {"workload": S.name, "value": tf, "unit": "TFLOP/s", "ms": te + ta, "expand_ms": te,
                           "attend_ms": ta, "algorithmic_tflop": fl / 1e12,
                           "roofline": dict(tensor_roofline((fl - fe) / (ta * 1e-3) / 1e12, pk),
                                            kernel="gdla_attend")}

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        inp_cpu = {k: v.cpu() for k, v in pin.items()}
        dt, fl, desc, thr = oracle_sample(P, inp_cpu, n_rows=ORACLE_ROWS, kv_groups=oracle_kv_groups(P))
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": thr, "kind": "oracle", "sample": desc,
               "seconds": dt}

    if rank == 0:
        roof = tensor_roofline(att_tflops, pk)
        roof.update({"traffic": measured_traffic("attn_tc_kernel", a.prefill),
                     "kernel": "gdla_attend (attention + differential epilogue)"})
        droof = hbm_roofline(dec_gbs / world, pk)
        droof.update({"kernel": "whole gdla_decode call (absorb, split-KV, combine)",
                      "traffic": measured_traffic("decode_tc_kernel", a.decode),
                      "traffic_kernel": "decode_tc_kernel (split-KV pass)"})
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": t_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) recipe)",
            "config": bench_config(a.prefill, a.decode, world),
            "prefill": {"ms": t_exp + t_att, "expand_ms": t_exp, "attend_ms": t_att,
                        "algorithmic_tflop": pf / 1e12},
            "decode": {"value": dec_gbs, "unit": "GB/s", "ms": t_dec_alone, "algorithmic_gb": db / 1e9,
                       "timing": "own loop after its own warm-up, before the prefill steps", "in_step_ms": t_dec,
                       "in_step_value": weak_scaling_value(db, world, t_dec * 1e-3) / 1e9, "roofline": droof,
                       "clocks": dclk},
            "roofline": roof, **extras,
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
