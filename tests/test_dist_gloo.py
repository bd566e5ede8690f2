"""Multi-rank host logic on CPU with two gloo ranks: rank discovery, the
max-over-ranks timing reduction, sharding of batch-head units and the
whole-job throughput aggregation the benchmark reports."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from flash_fwd_b200 import dist as fdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, w, l = fdist.init("gloo", timeout_s=60)
    assert (r, w, l) == (rank, world, rank)
    fdist.barrier()
    m = fdist.max_over_ranks(10.0 + 5.0 * rank)
    lo, hi = fdist.shard_range(7, w, r)
    out.put((rank, m, lo, hi))
    fdist.shutdown()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [m for _, m, _, _ in res] == [15.0, 15.0]
    spans = [(lo, hi) for _, _, lo, hi in res]
    assert spans == [(0, 4), (4, 7)]


@pytest.mark.parametrize("n,world", [(64, 8), (7, 3), (3, 4), (1, 1)])
def test_shard_range_partitions(n, world):
    spans = [fdist.shard_range(n, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (a, b), (c, _) in zip(spans, spans[1:]):
        assert b == c and b >= a
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_aggregate_throughput():
    # two ranks, 10 TFLOP each, slowest 2 s -> 10 TFLOP/s
    assert fdist.aggregate_throughput([10e12, 10e12], 2000.0) == 10e12
