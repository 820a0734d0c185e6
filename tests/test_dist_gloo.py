"""Multi-rank plumbing of the benchmark on CPU: two gloo ranks exercise the
max-over-ranks timing, the sum of per-rank counts, the barrier and the unit
sharding that bench.py uses under torchrun (no GPU, no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from bit_hadamard_rotated_b200 import dist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        assert dist.env_world() == (rank, rank, world)
        assert dist.init("gloo", timeout_s=60)
        dist.barrier()
        t_max = dist.max_over_ranks(1.5 + rank)          # slowest rank's time
        total = dist.sum_over_ranks(10 * (rank + 1))      # whole-job units
        parts = [list(dist.shard(10, r, world)) for r in range(world)]
        dist.barrier()
        dist.finish()
        q.put((rank, t_max, total, parts))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, repr(e), None, None))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    out = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
    assert out[0][1] == 2.5 and out[1][1] == 2.5, out
    assert out[0][2] == 30 and out[1][2] == 30, out
    assert out[0][3] == [[0, 1, 2, 3, 4], [5, 6, 7, 8, 9]]


def test_single_rank_defaults():
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert dist.env_world() == (0, 0, 1)
    assert dist.init("gloo") is False
    assert dist.max_over_ranks(3.0) == 3.0
    assert list(dist.shard(7, 0, 1)) == list(range(7))
