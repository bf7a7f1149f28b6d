"""bench.py's work counts and roofline arithmetic on CPU: the causal-pair and selected-key
counts against their closed forms, and the roofline entries computed from a given per-kernel
breakdown (no GPU involved)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from indexed_sparse_attention_fp8_b200 import workloads as W  # noqa: E402

PK = {"hbm_gbs": 6535.7, "bf16": 1672.2, "bf16_sus": 1382.4, "src": "measured"}


def test_work_counts_closed_forms():
    wl = W.WORKLOADS["prefill128k"]
    L, k = wl.T, wl.topk
    assert bench.causal_pairs(wl) == L * (L + 1) // 2                 # query t sees t + 1 keys
    assert bench.selected_pairs(wl) == k * (k + 1) // 2 + (L - k) * k  # min(k, t + 1) summed
    d = W.WORKLOADS["decode256k"]
    assert bench.causal_pairs(d) == d.B * d.S                          # one query at the end of each cache
    p = W.WORKLOADS["chunk1m_pool"]
    first = p.ctx - p.T                                                # position of the first new query
    assert bench.causal_pairs(p) == sum(pos // 4 + 1 for pos in range(first, p.ctx))


def test_roofline_prefill_entries():
    wl = W.WORKLOADS["prefill128k"]
    brk = {"indexer": 89.3, "topk": 30.7, "attn": 451.4, "fused_select": 70.0,
           "per_launch": {"indexer_chunk": 11.2, "topk_chunk": 3.8, "attn_layer": 112.85}}
    r = bench.roofline(wl, brk, PK, 16384)
    assert r["kernel"] == "attn" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    flops = 128 * 2 * (576 + 512) * bench.selected_pairs(wl)
    assert r["achieved"] == pytest.approx(4 * flops / 451.4e-3 / 1e12)
    assert r["peak"] == 1382.4 and r["frac"] == pytest.approx(r["achieved"] / 1382.4)
    unit, per_q = bench.TRAFFIC_PER_UNIT.get(("prefill128k", "attn"), (None, None))
    assert r["traffic"] == (None if per_q is None else pytest.approx(per_q * wl.B * wl.T))
    ix, tk, fs = r["others"]["indexer"], r["others"]["topk"], r["others"]["fused_select"]
    # indexer and top-k traffic: per visible pair, times the pairs of an average 16384-query chunk
    for name, ent in (("indexer", ix), ("topk", tk)):
        unit, per_p = bench.TRAFFIC_PER_UNIT.get(("prefill128k", name), (None, None))
        assert ent["traffic"] == (None if per_p is None else pytest.approx(per_p * bench.causal_pairs(wl) / 8))
        assert unit in (None, "pair")
    assert ix["achieved"] == pytest.approx(2 * 64 * 128 * bench.causal_pairs(wl) / 89.3e-3 / 1e12)
    assert ix["peak"] == pytest.approx(2 * 1382.4)
    assert fs["achieved"] == pytest.approx(2 * 64 * 128 * bench.causal_pairs(wl) / 70.0e-3 / 1e12)
    assert tk["bound"] == "hbm"
    assert tk["achieved"] == pytest.approx((4 * bench.causal_pairs(wl) + 4 * wl.T * 2048) / 30.7e-3 / 1e9)
    assert tk["frac"] == pytest.approx(tk["achieved"] / 6535.7)


def test_roofline_decode_is_hbm_bound():
    wl = W.WORKLOADS["decode256k"]
    brk = {"indexer": 0.21, "topk": 0.084, "attn": 0.218,
           "per_launch": {"indexer_chunk": 0.21, "topk_chunk": 0.084, "attn_layer": 0.0545}}
    r = bench.roofline(wl, brk, PK, 1)
    assert r["kernel"] == "attn" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(4 * bench.attn_bytes(wl) / 0.218e-3 / 1e9)
    ix = r["others"]["indexer"]
    assert ix["bound"] == "hbm"
    assert ix["achieved"] == pytest.approx((32 * 262144 * 128 + 32 * 64 * 132) / 0.21e-3 / 1e9)
    assert r["traffic"] is None and ix["traffic"] is None          # no capture at this context


def test_roofline_sums_the_work_of_shards():
    """A rank's shards (zig-zag chunks) add up: two halves give the whole workload's figures."""
    wl = W.WORKLOADS["prefill32k"]
    boxes = [(0, 1, 0, wl.T // 2), (0, 1, wl.T // 2, wl.T)]
    halves = [bench.box_workload(wl, b) for b in boxes]
    assert sum(bench.causal_pairs(h) for h in halves) == bench.causal_pairs(wl)
    assert sum(bench.selected_pairs(h) for h in halves) == bench.selected_pairs(wl)
    brk = {"indexer": 8.0, "topk": 2.0, "attn": 40.0,
           "per_launch": {"indexer_chunk": 4.0, "topk_chunk": 1.0, "attn_layer": 5.0}}
    assert bench.roofline(halves, brk, PK, 16384)["achieved"] == pytest.approx(
        bench.roofline(wl, brk, PK, 16384)["achieved"])
