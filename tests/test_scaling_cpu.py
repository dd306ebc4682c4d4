"""The N > 1 benchmark path on CPU: two gloo ranks, independent batches, the
max-over-ranks timing and the whole-job throughput (no GPU needed)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tiled_attention_18_b200.scaling import job_throughput, max_over_ranks, rank_seed
from tiled_attention_18_b200.workloads import WORKLOADS, make_inputs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank draws its own batch of the same shape
        q, _, _ = make_inputs(1, 2, 64, 64, "bf16", seed=rank_seed(0, rank))
        digest = float(q.float().sum())
        # a per-rank elapsed time; the job's time is the slowest rank's
        elapsed_ms = 10.0 + 5.0 * rank
        dist.barrier()
        m = max_over_ranks(elapsed_ms)
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        out.put((rank, m, digests))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    # every rank sees the slowest rank's time
    assert [r[1] for r in results] == [15.0, 15.0]
    # the ranks' batches are independent (different seeds give different data)
    digests = results[0][2]
    assert digests[0] != digests[1]


def test_job_throughput_counts_all_ranks():
    w = WORKLOADS["c5a"]
    one = job_throughput(w.flops, steps=10, world=1, max_ms=50.0)
    two = job_throughput(w.flops, steps=10, world=2, max_ms=50.0)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(w.flops * 10 / 0.05 / 1e12)
    with pytest.raises(ValueError):
        job_throughput(w.flops, 1, 1, 0.0)


def test_max_over_ranks_without_group():
    assert not dist.is_initialized()
    assert max_over_ranks(3.5) == 3.5
    assert rank_seed(0, 0) == 0 and rank_seed(0, 3) == 3
    assert torch.equal(make_inputs(1, 1, 8, 64, "fp16", seed=rank_seed(5, 0))[0],
                       make_inputs(1, 1, 8, 64, "fp16", seed=5)[0])
