"""The benchmark's multi-rank host logic on CPU (gloo, world size 2).

Windows, heads and images are independent, so N GPUs run N independent
batches (weak scaling) and the data path has no collective.  What the ranks
share is host logic: each rank seeds its own batch, the timed region is
bracketed by barriers, timings are reduced as the maximum over ranks, and the
job's throughput counts every rank's tokens.  A rank that never reaches the
barrier must end the others' wait with an error (short process-group
timeout), not hang them.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=30):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _timing_worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench
    from windowed_attention_vision_b200 import inputs as I
    _init(rank, world, port)
    try:
        dist.barrier()
        # per-rank timings: the reduced value is the slowest rank's
        elapsed, kernel = bench.max_over_ranks([10.0 + 5.0 * rank, 1.0 + rank], "cpu")
        # every rank draws its own batch: seeds differ by rank
        w = I.Workload("mr", 1, 8, 8, 4, (0,), 2, 32, "bf16", "standard")
        (qkv,), _, _ = I.make_inputs(w, "cpu", base=rank)
        mine = qkv[0].float()
        gathered = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)
        distinct = not torch.equal(gathered[0], gathered[1])
        value = bench.job_tokens_per_s(w, 1, 4, world, elapsed)
        results[rank] = (elapsed, kernel, distinct, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_timing_worker, args=(world, port, results), nprocs=world, start_method="spawn")
        res = dict(results)
    assert set(res) == {0, 1}
    for rank in range(world):
        elapsed, kernel, distinct, value = res[rank]
        assert elapsed == 15.0 and kernel == 2.0, "timings are the maximum over ranks"
        assert distinct, "each rank draws its own batch"
        # 2 ranks x 4 steps x 64 tokens in 15 ms
        assert value == pytest.approx(2 * 4 * 64 / 0.015)


def _dropout_worker(rank, world, port, results):
    _init(rank, world, port, timeout_s=3)
    try:
        dist.barrier()
        if rank == 1:
            # leaves between steps: none of its work is in flight
            results[rank] = "left"
            os._exit(0)
        try:
            dist.barrier()
            results[rank] = "no error"
        except Exception as e:  # the survivor learns of it from the timeout
            results[rank] = "error: " + type(e).__name__
    finally:
        if rank == 0:
            try:
                dist.destroy_process_group()
            except Exception:
                pass


def test_rank_that_leaves_ends_the_others_wait():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        procs = [ctx.Process(target=_dropout_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=60)
        alive = [p for p in procs if p.is_alive()]
        for p in alive:
            p.kill()
        res = dict(results)
    assert not alive, "a surviving rank hung instead of timing out"
    assert res.get(1) == "left"
    assert str(res.get(0, "")).startswith("error"), res
