"""The benchmark's multi-rank logic on CPU with two gloo ranks: the timing
reduction is a max over ranks, the whole-job value counts every rank's units
over the slowest rank's time, and every rank draws its own problem."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from differential_latent_attention_gdla_b200 import workloads as wl

        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], world, "cpu")
        shape = wl.PrefillShape("mr", B=1, L=8, n_kv=1, g=1)
        inp = wl.make_prefill_inputs(shape, seed=bench.rank_seed(0, rank, "prefill"))
        s = float(inp["q"].float().sum())
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, torch.tensor([s], dtype=torch.float64))
        q.put((rank, got, [float(x) for x in sums]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_timing_reduction_and_independent_problems():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, sums in res:
        assert got == [2.0, 10.0, 3.0]
        assert sums[0] != sums[1]  # each rank has its own seeded problem


def test_weak_scaling_value():
    import bench

    assert bench.weak_scaling_value(10.0, 4, 2.0) == pytest.approx(20.0)
    assert bench.rank_seed(5, 3, "decode") != bench.rank_seed(5, 3, "prefill")
