"""Host-side multi-process logic on CPU with the gloo backend, world size 2.

The layer runs data-parallel (each rank owns full copies of its layers and its
own tokens); what ranks share is the timing protocol: a barrier around the
timed region, the maximum of the per-rank device times, and the sum of the
tokens processed.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

from bit_quantized_moe_softmax_b200 import dist as D


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(world))
    try:
        r, local, w = D.init("gloo", timeout_s=30)
        D.barrier()
        mx = D.max_over_ranks(1.5 + r)          # per-rank "elapsed"
        tot = D.sum_over_ranks(100 * (r + 1))   # per-rank tokens
        lo, hi = D.shard_range(10, r, w)
        q.put((r, w, mx, tot, lo, hi))
        D.finish()
    except Exception as e:  # report instead of hanging the parent
        q.put(("error", repr(e)))


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    assert all(g[0] != "error" for g in got), got
    got.sort()
    assert [g[2] for g in got] == [2.5, 2.5]          # max over ranks
    assert [g[3] for g in got] == [300.0, 300.0]      # sum over ranks
    assert [(g[4], g[5]) for g in got] == [(0, 5), (5, 10)]


@pytest.mark.parametrize("total,world", [(10, 3), (0, 2), (7, 8), (11709, 8)])
def test_shard_range_covers_exactly(total, world):
    spans = [D.shard_range(total, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == total
    assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_single_process_identity():
    assert D.max_over_ranks(3.0) == 3.0
    assert D.sum_over_ranks(4.0) == 4.0
