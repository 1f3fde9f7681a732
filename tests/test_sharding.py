"""Host logic of the query-sharded prefill (block_sparse_long_kbar_b200.sharding), on the CPU:
the zig-zag partition covers every query row once and gives every rank the same causal work,
and the all-gather over two gloo ranks rebuilds the sequence in token order from the ranks'
chunks."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from block_sparse_long_kbar_b200.sharding import chunk_owner, zigzag_ranges  # noqa: E402


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_zigzag_covers_every_row_once_with_equal_causal_work(world):
    T, B = 131072, 8
    seen = np.zeros(T, dtype=np.int64)
    work = []
    for r in range(world):
        rs = zigzag_ranges(T, world, r)
        assert len(rs) == 2 and all(t1 - t0 == T // (2 * world) for t0, t1 in rs)
        w = 0
        for t0, t1 in rs:
            seen[t0:t1] += 1
            w += sum(t // B for t in range(t0, t1))  # scored candidates, proportional to t
        work.append(w)
    assert (seen == 1).all()
    assert max(work) - min(work) <= T // (2 * world)  # equal up to rounding of t / B
    for c in range(2 * world):
        r, s = chunk_owner(c, world)
        assert zigzag_ranges(T, world, r)[s] == (c * T // (2 * world), (c + 1) * T // (2 * world))


def test_zigzag_rejects_uneven_splits():
    with pytest.raises(ValueError):
        zigzag_ranges(1000, 3, 0)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    from block_sparse_long_kbar_b200.sharding import gather_sequence, zigzag_ranges
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T = 64
        # batch 2, rows of 3 (float32: gloo gathers no 16-bit types; NCCL moves the bf16 tensors)
        full = torch.arange(2 * T * 3, dtype=torch.float32).reshape(2, T, 3)
        local = [full[:, t0:t1].contiguous() for t0, t1 in zigzag_ranges(T, world, rank)]
        got = gather_sequence(local, world)
        q.put((rank, bool(torch.equal(got, full))))
    finally:
        dist.destroy_process_group()


def test_gather_rebuilds_the_sequence_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert res == [(0, True), (1, True)]
