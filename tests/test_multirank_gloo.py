"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on the CPU: every rank
draws its own batch, the slowest rank's time is what both report, and the whole-job throughput
counts the work of every rank.  The reference arm exits at once on ranks other than 0."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = 10.0 * (rank + 1)  # fake per-rank timed-loop durations (ms)
        worst = bench.max_over_ranks(elapsed, True, device="cpu")
        value = bench.whole_job_value(1e12, 5, worst, world, 1e12)
        dist.barrier()
        out.put((rank, worst, value, bench.rank_seed(2, rank)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_rank_and_the_whole_job():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]  # both ranks see the max
    # 2 ranks x 1 TFLOP x 5 steps in 20 ms = 500 TFLOP/s
    assert res[0][2] == pytest.approx(500.0) and res[1][2] == pytest.approx(500.0)
    seeds = [r[3] for r in res]
    assert seeds[0] != seeds[1]
    a = synth.normal_f32(seeds[0], synth.K_ID, (64,))
    b = synth.normal_f32(seeds[1], synth.K_ID, (64,))
    assert not np.array_equal(a, b)  # independent batches per rank


def test_reference_arm_does_nothing_on_other_ranks():
    class Args:
        workload, warmup, steps, gpus = None, 3, 5, 2
    assert bench.run_reference(Args(), rank=1, world=2) == 0


def test_kernel_hash_ignores_comments_and_layout():
    import bench

    code = "int f(int a) {\n  return a + 1;  // one more\n}\n/* note */"
    assert bench.code_tokens(code) == bench.code_tokens("int f(int a) { return a + 1; }")
    assert bench.code_tokens(code) != bench.code_tokens("int f(int a) { return a + 2; }")
    for fam in bench.FAMILY_SOURCES:
        assert len(bench.kernel_sources_hash(fam)) == 16
