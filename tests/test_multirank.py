"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, as torchrun would start them.

The recurrence shards over independent (batch, head) sequences, so the ranks share no
data; the only collectives are the timing reduction (max over ranks) and barriers.
These tests check that reduction, the per-rank input draw and the whole-job rate."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from synthetic_inputs import make_inputs
        ms = bench.max_over_ranks(10.0 + 5.0 * rank)  # rank 1 is the slow one
        x = make_inputs(1, 64, 2, 64, 64, dtype="bf16", seed=bench.rank_seed(rank))
        # every rank's first query row, gathered so that rank 0 can compare them
        row = x["q"][0, 0, 0].float().contiguous()
        rows = [torch.empty_like(row) for _ in range(world)]
        dist.all_gather(rows, row)
        q.put((rank, ms, [r.tolist() for r in rows]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_time_max_and_distinct_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=100) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    by_rank = {r: (ms, rows) for r, ms, rows in out}
    # both ranks report the slowest rank's time
    assert by_rank[0][0] == by_rank[1][0] == 15.0
    # the ranks drew different batches
    rows = by_rank[0][1]
    assert rows[0] != rows[1]


def test_job_rate_is_the_sum_over_ranks():
    sys.path.insert(0, ROOT)
    import bench
    # 32768 tokens per rank in 0.5 ms on each of 4 ranks
    assert bench.job_rate(32768, 4, 0.5) == pytest.approx(4 * 32768 / 0.5e-3)
    assert bench.max_over_ranks(3.0) == 3.0  # no process group: unchanged
    assert bench.rank_seed(0) != bench.rank_seed(1)
