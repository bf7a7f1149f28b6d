"""Sharding plans on CPU: every query row (prefill) or sequence (decode) of a workload lands on
exactly one rank, the ranks' causal indexer work is balanced, and the plans that two gloo
ranks compute independently agree when gathered."""
import os
import socket
import sys
from datetime import timedelta

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from indexed_sparse_attention_fp8_b200 import shard
from indexed_sparse_attention_fp8_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rows_of(wl, world):
    cover = {}
    for r in range(world):
        for b0, b1, t0, t1 in shard.plan(wl, world, r):
            for b in range(b0, b1):
                for t in range(t0, t1):
                    cover[(b, t)] = cover.get((b, t), 0) + 1
    return cover


@pytest.mark.parametrize("name", ["tiny", "prefill32k", "decode256k", "chunk1m"])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_every_row_on_exactly_one_rank(name, world):
    wl = W.WORKLOADS[name]
    if wl.T > 20000:
        wl = wl.replace(T=wl.T // 16, ctx=wl.ctx // 16)    # same structure, fewer rows to count
    cover = _rows_of(wl, world)
    assert len(cover) == wl.B * wl.T and set(cover.values()) == {1}


@pytest.mark.parametrize("world", [2, 4, 8])
def test_zigzag_balances_the_causal_indexer_work(world):
    # prefill 128K: per-rank visible (query, key) pairs within 0.1% of each other, whereas plain
    # contiguous blocks would differ by a factor of about 2*world - 1
    T = S = 131072
    work = [sum(shard.visible_pairs(S, T, t0, t1, S) for t0, t1 in shard.zigzag_chunks(T, world, r))
            for r in range(world)]
    assert sum(work) == shard.visible_pairs(S, T, 0, T, S)
    assert max(work) / min(work) < 1.001
    rows = [sum(t1 - t0 for t0, t1 in shard.zigzag_chunks(T, world, r)) for r in range(world)]
    assert max(rows) - min(rows) <= 2                      # the attention's work: k keys per row
    blocks = [shard.visible_pairs(S, T, r * T // world, (r + 1) * T // world, S) for r in range(world)]
    assert max(blocks) / min(blocks) > 2 * world - 2


def test_decode_batch_slices_and_bad_ranks():
    assert [shard.batch_slice(32, 8, r) for r in range(8)] == [(4 * r, 4 * r + 4) for r in range(8)]
    assert [shard.batch_slice(5, 2, r) for r in range(2)] == [(0, 3), (3, 5)]
    assert shard.plan(W.WORKLOADS["decode256k"].replace(B=3), 4, 3) == []     # more ranks than sequences
    with pytest.raises(ValueError):
        shard.zigzag_chunks(100, 2, 2)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    from indexed_sparse_attention_fp8_b200 import shard as sh
    from indexed_sparse_attention_fp8_b200 import workloads as wls
    wl = wls.WORKLOADS["prefill128k"]
    mine = sh.plan(wl, world, rank)
    work = sum(sh.visible_pairs(wl.ctx, wl.T, t0, t1, wl.S) for _, _, t0, t1 in mine)
    plans = [None] * world
    dist.all_gather_object(plans, (mine, work))
    q.put((rank, plans))
    dist.destroy_process_group()


def test_two_gloo_ranks_plan_the_prefill_consistently():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0][1] == got[1][1]                          # both ranks see the same plans
    plans = got[0][1]
    rows = sorted(t for boxes, _ in plans for _, _, t0, t1 in boxes for t in (t0, t1))
    T = W.WORKLOADS["prefill128k"].T
    assert rows[0] == 0 and rows[-1] == T
    ranges = sorted((t0, t1) for boxes, _ in plans for _, _, t0, t1 in boxes)
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))   # contiguous, no gap or overlap
    works = [w for _, w in plans]
    assert max(works) / min(works) < 1.001
