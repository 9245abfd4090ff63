"""Host logic of the multi-GPU bench path, run as two gloo ranks on the CPU.

Attention over different (batch, head) slices is independent, so with N GPUs
every rank runs its own batch and the only cross-rank traffic is the timing
reduction (max over ranks).  These tests check that part without a GPU.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    import bench
    from exact_attention_117_b200.workloads import WORKLOADS, make_inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(WORKLOADS["c1"], rank)
        x = make_inputs(w, "cpu", with_do=False)
        # each rank reports a different step time; every rank must see the max
        mx = bench.max_over_ranks([10.0 + rank, 3.0 * (1 - rank)], world)
        out[rank] = (w.seed_base, float(x["q"].float().sum()), mx)
    finally:
        dist.destroy_process_group()


def test_two_ranks_independent_batches_and_max_time():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    (s0, q0, mx0), (s1, q1, mx1) = res[0], res[1]
    assert s0 != s1 and q0 != q1          # distinct problems per rank
    assert mx0 == mx1 == [11.0, 3.0]     # max over ranks, same on every rank


def test_job_throughput_counts_every_rank():
    import bench
    one = bench.job_tflops(1e12, 1, 1.0)
    assert one == pytest.approx(1000.0)
    assert bench.job_tflops(1e12, 8, 1.0) == pytest.approx(8 * one)
    fwd, bwd = bench.attention_flops(2, 16, 4096, 128, True)
    assert fwd == 4 * 2 * 16 * 4096 * 4096 * 128 / 2 and bwd == 2.5 * fwd
