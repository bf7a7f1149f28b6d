"""Benchmark of the DSA layer group on B200: query tokens/s per 4-layer IndexShare group.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill128k] [--impl ours|reference]

A step is one IndexShare group over the whole workload: the FP8 indexer and the top-k over
every query (in workspace-sized query chunks), then sparse attention for each of the 4
layers, all inside one dsa_group_forward call (the C ABI).  Inputs are synthetic and seeded
(indexed_sparse_attention_fp8_b200.workloads), already resident in HBM for `value`; `e2e`
repeats the step from pinned host buffers with the host<->device copies inside the timed
region.  Inputs are larger than L2, so no flush is needed between steps.

Multi-GPU (torchrun, one process per GPU, --gpus N must equal the world size): the one
workload is sharded with no exchange step -- prefill query rows in zig-zag contiguous chunks,
decode sequences in batch slices (indexed_sparse_attention_fp8_b200.shard) -- with the key
caches replicated; value = the workload's queries / max-over-ranks time, scaling "strong"
(the total work is fixed).

The JSON line also carries: the decode line (32 x 256K), the per-layer-indexer comparator
at 128K with the IndexShare speedup, chunked prefill at a 1M-token cache without and with
IndexPool (and that speedup), a per-kernel breakdown from CUDA events, the roofline
of the dominant kernel, SM clocks sampled during the timed region, and the CPU oracle's
throughput on a bounded sample (cpu_baseline).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from indexed_sparse_attention_fp8_b200 import shard  # noqa: E402
from indexed_sparse_attention_fp8_b200 import workloads as W  # noqa: E402

METRIC = "query tok/s per 4-layer IndexShare group (prefill 128K, decode 256K); % roofline"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sus": d["bf16_tflops_sustained"],
                "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "src": "fallback"}


# ------------------------------------------------------------------------------ work counts

def causal_pairs(wl: W.Workload) -> int:
    """Visible (query, key-row) pairs of the indexer (pooled rows when pool > 1)."""
    tot = 0
    for t in range(wl.T):
        pos = wl.ctx - wl.T + t
        tot += min(wl.S // wl.pool, pos // wl.pool + 1)
    return tot * wl.B


def selected_pairs(wl: W.Workload) -> int:
    """Sum over queries of the number of selected tokens (k_eff, expanded for IndexPool)."""
    tot = 0
    for t in range(wl.T):
        pos = wl.ctx - wl.T + t
        if wl.pool == 1:
            tot += min(wl.topk, pos + 1)
        else:
            nb = min(wl.topk, pos // wl.pool + 1)
            tot += min(nb * wl.pool, pos + 1)
    return tot * wl.B


def indexer_flops(wl):
    return 2 * wl.H_I * wl.d_I * causal_pairs(wl)


def attn_flops(wl):
    return wl.Hq * 2 * (wl.d_qk + wl.d_v) * selected_pairs(wl)


def attn_bytes(wl):
    """Gathered KV rows (bf16) + q + out + idx per layer."""
    row = wl.d_qk * 2 if wl.kv_latent else (wl.d_qk + wl.d_v) * 2
    return selected_pairs(wl) * row + wl.B * wl.T * wl.Hq * (wl.d_qk + wl.d_v) * 2 + wl.B * wl.T * wl.topk * wl.pool * 4


# ------------------------------------------------------------------------------ clocks

def gpu_id(dev) -> str:
    """nvidia-smi identifier of a torch device (UUID, so CUDA_VISIBLE_DEVICES cannot mislead it)."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:  # pragma: no cover
        return str(torch.cuda.current_device())


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ our arm

def make_group(wl, dev, dsa, layers=None, indexer_layer=0, share_q=False):
    ind = W.make_indexer_inputs(wl, device=dev, layer=indexer_layer)
    n = wl.group if layers is None else layers
    lays = []
    for l in range(n):
        a = W.make_attn_inputs(wl, l, device=dev) if (l == 0 or not share_q) else \
            {"q": lays[0]["q"], "kv": W.make_attn_inputs(wl, l, device=dev)["kv"], "v": None}
        lays.append({"q": a["q"], "kv": a["kv"], "v": a["v"]})
    return ind, lays


def rank_boxes(wl, world, rank):
    """This rank's (b0, b1, t0, t1) boxes of the workload: all of it on one GPU, else its
    share of the sharding plan (zig-zag query-row chunks for prefill, batch slices for decode)."""
    return [(0, wl.B, 0, wl.T)] if world == 1 else shard.plan(wl, world, rank)


def box_workload(wl, box):
    """The workload restricted to one box: its rows keep their positions (ctx moves to the
    chunk's end), so the work counts below apply to it unchanged."""
    b0, b1, t0, t1 = box
    return wl.replace(B=b1 - b0, T=t1 - t0, ctx=wl.ctx - (wl.T - t1))


class Part:
    """One box of the rank's share: its sub-workload, its input tensors and its group call.
    With IndexPool the pooled key cache is state kept beside the key cache, as a serving loop
    keeps it: pooled once here, and each step refreshes only the blocks that hold the step's
    T new rows (dsa_index_pool_tail) before the group call reads it."""

    def __init__(self, wl, box, ind, lays, dsa):
        self.wl, self.box, self.ind, self.lays = box_workload(wl, box), box, ind, lays
        self.dsa = dsa
        self.k_pool = dsa.dsa_index_pool(ind["k_idx"], pool=wl.pool) if wl.pool > 1 else None
        self.g = dsa.Group(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], wl.topk, lays, wl.sm_scale,
                           wl.d_v, pool=wl.pool, k_pooled=self.k_pool)

    def refresh_pool(self, stream):
        if self.k_pool is not None:
            self.dsa.dsa_index_pool_tail(self.ind["k_idx"], self.ind["ctx_len"], self.wl.T, self.k_pool,
                                         pool=self.wl.pool, stream=stream)

    def step(self, ws, stream):
        self.refresh_pool(stream)
        self.g.forward(ws, stream)


def make_parts(wl, dev, dsa, boxes):
    """Inputs of every box of this rank.  The whole workload keeps its tensors as made; a
    shard copies its query rows out of the full (identically seeded) tensors, one layer at a
    time, and views the replicated key caches."""
    whole = boxes == [(0, wl.B, 0, wl.T)]
    ind_full = W.make_indexer_inputs(wl, device=dev)

    def rows(x, box):
        b0, b1, t0, t1 = box
        return x if whole else x[b0:b1, t0:t1].contiguous()

    inds = [{"q_idx": rows(ind_full["q_idx"], bx), "w": rows(ind_full["w"], bx),
             "k_idx": ind_full["k_idx"][bx[0]:bx[1]],
             "ctx_len": ind_full["ctx_len"][bx[0]:bx[1]] - (wl.T - bx[3])} for bx in boxes]
    lays = [[] for _ in boxes]
    for l in range(wl.group):
        a = W.make_attn_inputs(wl, l, device=dev)
        for i, bx in enumerate(boxes):
            lays[i].append({"q": rows(a["q"], bx), "kv": a["kv"][bx[0]:bx[1]],
                            "v": None if a["v"] is None else a["v"][bx[0]:bx[1]]})
        del a
    del ind_full
    return [Part(wl, bx, ind, lay, dsa) for bx, ind, lay in zip(boxes, inds, lays)]


def score_t_chunk(args, wl):
    return args.t_chunk or max(1, min(wl.T, (args.score_ws_gb << 30) // (wl.B * ((wl.S // wl.pool + 3) // 4 * 4) * 4)))


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (every rank takes part; world 1 returns x)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def job_throughput(units_per_rank_step: int, world: int, ms_per_step: float) -> float:
    """Whole-job units/s when every rank processes its own units each step (replicas, weak
    scaling) and the step takes as long as the slowest rank."""
    return units_per_rank_step * world / (ms_per_step / 1e3)


def l2_note(wl) -> str:
    """How the timed steps relate to the 126 MB L2: the key caches and the per-layer inputs of a
    step either exceed it (no flush is needed between steps) or not (small profiling cases,
    which are timed without a flush and say so)."""
    step_bytes = (wl.B * wl.S // wl.pool * wl.d_I + wl.B * wl.T * wl.H_I * (wl.d_I + 4)
                  + wl.group * wl.B * (wl.T * wl.Hq * wl.d_qk + wl.S * (wl.d_qk + (0 if wl.kv_latent else wl.d_v))) * 2)
    if step_bytes > 126e6:
        return "inputs larger than L2 (126 MB); no flush"
    return f"inputs of {step_bytes / 1e6:.1f} MB fit in L2 (126 MB): a small profiling case, not flushed"


def time_region(fn, steps, stream):
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(steps):
        fn()
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e)


def run_ours(args, rank, world, dev):
    import indexed_sparse_attention_fp8_b200 as dsa
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    pk = peaks()
    wl = W.WORKLOADS[args.workload]
    if args.T:
        wl = wl.replace(T=args.T)
    boxes = rank_boxes(wl, world, rank)
    parts = make_parts(wl, dev, dsa, boxes)
    t_chunk = score_t_chunk(args, wl)
    ws = torch.empty(max([1] + [p.g.workspace_size(t_chunk) for p in parts]), dtype=torch.uint8, device=dev)

    def step():
        for p in parts:
            p.step(ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    l0 = dsa.launch_count()
    with ClockSampler(gpu_id(dev)) as clk:
        ms = time_region(step, args.steps, stream)
    launches = dsa.launch_count() - l0
    ms = max_over_ranks(ms, world, dev)
    ms_step = ms / args.steps
    # every query row of the workload is processed once per step, spread over the ranks
    value = wl.B * wl.T / (ms_step / 1e3)

    # ---- per-kernel breakdown: the same step as separate C-ABI calls with events between them
    brk = breakdown(parts, ws, t_chunk, stream, dsa, args.steps if args.steps <= 3 else 3)

    res = {
        "metric": METRIC, "value": value, "unit": "query tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak" if world == 1 else "strong",
        "vs_baseline": None, "dtype": "fp8-e4m3 indexer / bf16 attention (fp32 accumulate)", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "ctx": wl.ctx, "H_I": wl.H_I, "d_I": wl.d_I,
                   "topk": wl.topk, "pool": wl.pool, "Hq": wl.Hq, "d_qk": wl.d_qk, "d_v": wl.d_v,
                   "group": wl.group, "t_chunk": t_chunk,
                   "parallelism": "1 GPU" if world == 1 else
                   (f"query rows sharded zig-zag over {world} ranks" if wl.T > 1 else f"batch sharded over {world} ranks"),
                   "l2": l2_note(wl)},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "breakdown_ms": brk,
    }
    if world > 1:
        res["config"]["rank0_rows"] = sum(p.wl.B * p.wl.T for p in parts)
    res["roofline"] = roofline([p.wl for p in parts], brk, pk, t_chunk)
    del ws
    torch.cuda.empty_cache()
    return res, wl, parts


def breakdown(parts, ws, t_chunk, stream, dsa, reps, fused=True):
    """Average device time of each step of the group per step over `reps` steps, CUDA events on
    `stream` (the launches queued ahead of the GPU), summed over this rank's parts: the refresh
    of the pooled key cache (IndexPool), the selection as the group call runs it (the indexer
    writing full score rows, then the row top-k, per query chunk), and each attention layer;
    with `fused`, also the fused selection (dsa_index_select) over the same chunks, for
    comparison."""
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    tot = {"pool": 0.0, "indexer": 0.0, "topk": 0.0, "attn": 0.0, "fused_select": 0.0}
    n = {k: 0 for k in tot}
    dev = ws.device
    for p in parts:
        wl, ind, g = p.wl, p.ind, p.g
        S_eff = ind["k_idx"].shape[1] // wl.pool
        ld = (S_eff + 3) // 4 * 4
        tc_max = min(t_chunk, wl.T)
        sc_buf = torch.empty(wl.B * tc_max * ld, dtype=torch.float32, device=dev)
        attn_ws = torch.empty(max(1, dsa.dsa_sparse_attn_workspace_size(wl.B, wl.T, wl.Hq, wl.d_v, wl.topk * wl.pool)),
                              dtype=torch.uint8, device=dev)
        sel_ws = None
        if fused:
            sel_ws = torch.empty(dsa.dsa_index_select_workspace_size(wl.B, tc_max, S_eff, wl.pool), dtype=torch.uint8,
                                 device=dev)
        for rep in range(reps):
            marks = []
            # hold the stream for a few ms, so every launch below is queued before the GPU reaches
            # it: the marks then time the kernels back to back, not the host's calls (which, for
            # the short decode kernels, take longer than the kernels)
            torch.cuda._sleep(5_000_000)
            keys = ind["k_idx"]
            if wl.pool > 1:
                a, b = ev(), ev()
                a.record(stream)
                p.refresh_pool(stream)
                b.record(stream)
                marks.append(("pool", a, b))
                keys = p.k_pool
            for t0 in range(0, wl.T, t_chunk):
                tc = min(t_chunk, wl.T - t0)
                sc = sc_buf[: wl.B * tc * ld].view(wl.B, tc, ld)   # [B, tc, ld], batch stride tc * ld
                a, b, c = ev(), ev(), ev()
                a.record(stream)
                dsa.dsa_index_scores(ind["q_idx"], ind["w"], keys, ind["ctx_len"], pool=wl.pool, t_begin=t0,
                                     t_count=tc, scores=sc, stream=stream)
                b.record(stream)
                dsa.dsa_topk(sc, ind["ctx_len"], wl.T, S_eff, wl.topk, pool=wl.pool, t_begin=t0, idx=g.idx,
                             stream=stream)
                c.record(stream)
                marks += [("indexer", a, b), ("topk", b, c)]
            for L in g.layers:
                a, b = ev(), ev()
                a.record(stream)
                dsa.dsa_sparse_attn(L["q"], L["kv"], g.idx, wl.sm_scale, wl.d_v, v=L["v"], out=L["out"], ws=attn_ws,
                                    stream=stream)
                b.record(stream)
                marks.append(("attn", a, b))
            if fused and rep == 0:
                for t0 in range(0, wl.T, t_chunk):
                    tc = min(t_chunk, wl.T - t0)
                    a, b = ev(), ev()
                    a.record(stream)
                    dsa.dsa_index_select(ind["q_idx"], ind["w"], keys, ind["ctx_len"], wl.topk, pool=wl.pool,
                                         t_begin=t0, t_count=tc, idx=g.idx, ws=sel_ws, stream=stream)
                    b.record(stream)
                    marks.append(("fused_select", a, b))
            torch.cuda.synchronize()
            for name, a, b in marks:
                tot[name] += a.elapsed_time(b) / (1 if name == "fused_select" else reps)
                n[name] += 1
        del sc_buf, attn_ws, sel_ws
    out = {k: tot[k] for k in ("pool", "indexer", "topk", "attn", "fused_select") if n[k]}
    out["per_launch"] = {"indexer_chunk": tot["indexer"] / max(1, n["indexer"] / reps),
                         "topk_chunk": tot["topk"] / max(1, n["topk"] / reps),
                         "attn_layer": tot["attn"] / max(1, n["attn"] / reps)}
    return out


# DRAM bytes (read + write) per unit of work, from one ncu capture with the bench's 131072-row
# context and its last 2048 queries (dram__bytes_read.sum + dram__bytes_write.sum per launch):
# per query for the attention (each query reads its q, writes its output and gathers its own
# 2048 key rows), per visible (query, key) pair for the indexer and the top-k (their bytes are
# the score rows, 4 B per pair written and read back).  A launch's traffic is the figure times
# the units it processes.  Only kernels unchanged since that capture are listed (others report
# None), and other contexts were not measured.
TRAFFIC_PER_UNIT = {("prefill128k", "attn"): ("query", 603.7e3), ("prefill128k", "indexer"): ("pair", 3.922),
                    ("prefill128k", "topk"): ("pair", 4.285)}


def roofline(wls, brk, pk, t_chunk):
    """Roofline of the kernel with the largest share of the time (indexer, top-k or attention,
    as the group call runs them); `wls` are the (sub-)workloads this rank ran, whose work adds
    up.  The fused selection, when timed, is listed too (against the indexer's roofline, its
    sampling pass, threshold and top-k counting as overhead)."""
    wls = wls if isinstance(wls, (list, tuple)) else [wls]
    wl = wls[0]
    fp8_peak = 2.0 * pk["bf16_sus"]   # nominal fp8:bf16 ratio 2 on the measured bf16 figure
    n_layers = wl.group
    rows = sum(w.B * w.T for w in wls)
    decode = rows <= 64
    ifl = sum(indexer_flops(w) for w in wls)
    ibytes = sum(w.B * (w.S // w.pool) * w.d_I + w.B * w.T * w.H_I * (w.d_I + 4) for w in wls)
    topk_bytes = sum(4 * causal_pairs(w) + 4 * w.B * w.T * w.topk * w.pool for w in wls)

    def idx_entry(ms, what):
        if decode:
            return {"bound": "hbm", "achieved": ibytes / (ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "traffic": None, "peak_src": f"{pk['src']} copy",
                    "work": f"indexer key, query and weight bytes; time of {what}"}
        return {"bound": "tensor", "achieved": ifl / (ms * 1e-3) / 1e12, "peak": fp8_peak, "unit": "TFLOP/s",
                "dtype": "fp8", "traffic": None, "peak_src": f"2 x {pk['src']} bf16 sustained",
                "work": f"indexer flops (2*H_I*d_I per visible pair); time of {what}"}
    ent = {
        "indexer": idx_entry(brk["indexer"], "the indexer"),
        "topk": {"bound": "hbm", "achieved": topk_bytes / (brk["topk"] * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                 "unit": "GB/s", "traffic": None, "peak_src": f"{pk['src']} copy",
                 "work": "score rows read + selected ids written"},
    }
    if decode:   # HBM-bound: the selected rows' bytes
        ent["attn"] = {"bound": "hbm", "achieved": sum(attn_bytes(w) for w in wls) * n_layers / (brk["attn"] * 1e-3) / 1e9,
                       "peak": pk["hbm_gbs"], "unit": "GB/s", "traffic": None, "peak_src": f"{pk['src']} copy"}
    else:
        ent["attn"] = {"bound": "tensor",
                       "achieved": sum(attn_flops(w) for w in wls) * n_layers / (brk["attn"] * 1e-3) / 1e12,
                       "peak": pk["bf16_sus"], "unit": "TFLOP/s", "dtype": "bf16", "traffic": None,
                       "peak_src": f"{pk['src']} bf16 sustained"}
    if "fused_select" in brk:
        ent["fused_select"] = idx_entry(brk["fused_select"], "the fused indexer + top-k")
    n_chunks = -(-rows // max(1, min(t_chunk, rows)))   # query chunks of the indexer and top-k
    units = {"query": {"attn": rows / len(wls)},
             "pair": {k: sum(causal_pairs(w) for w in wls) / n_chunks for k in ("indexer", "topk")}}
    for k in ("attn", "indexer", "topk"):
        unit, per = TRAFFIC_PER_UNIT.get((wl.name, k), (None, None))
        ent[k]["traffic"] = None if per is None else per * units[unit][k]   # bytes per (average) launch
    top = max(("indexer", "topk", "attn"), key=lambda k: brk[k])
    r = dict(ent[top])
    r["kernel"] = top
    r["frac"] = r["achieved"] / r["peak"]
    r["others"] = {k: {kk: vv for kk, vv in v.items()} | {"frac": v["achieved"] / v["peak"]}
                   for k, v in ent.items() if k != top}
    return r


def run_e2e(args, wl, parts, dev, stream, world):
    """Same step from pinned host memory, through the library's public calls (per query chunk the
    indexer and the top-k, then each attention layer): every input goes host -> device and every
    output device -> host inside the timed region.  The copies run on one stream per direction
    and overlap the compute and each other: the selection waits only for the indexer inputs, a
    layer's attention only for its own q and kv, and a layer's output leaves as soon as it is
    written.  A copy into a buffer waits for the previous step's last reader of that buffer, and
    a kernel writing an output buffer for the previous step's copy out of it."""
    import indexed_sparse_attention_fp8_b200 as dsa
    t_chunk = score_t_chunk(args, wl)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    h2d, d2h, plans = 0, 0, []
    for p in parts:
        host = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in p.ind.items()}
        for k in host:
            host[k].copy_(p.ind[k])
        hq = torch.empty_like(p.lays[0]["q"], device="cpu").pin_memory()
        hkv = torch.empty_like(p.lays[0]["kv"], device="cpu").pin_memory()
        hq.copy_(p.lays[0]["q"])
        hkv.copy_(p.lays[0]["kv"])
        hout = torch.empty_like(p.g.layers[0]["out"], device="cpu").pin_memory()
        hidx = torch.empty_like(p.g.idx, device="cpu").pin_memory()
        h2d += sum(v.numel() * v.element_size() for v in host.values()) + len(p.lays) * (
            hq.numel() * hq.element_size() + hkv.numel() * hkv.element_size())
        d2h += len(p.lays) * hout.numel() * hout.element_size() + p.g.idx.numel() * 4
        S_eff = p.ind["k_idx"].shape[1] // p.wl.pool
        ld = (S_eff + 3) // 4 * 4
        tc_max = min(t_chunk, p.wl.T)
        nl = len(p.g.layers)
        plans.append(dict(p=p, host=host, hq=hq, hkv=hkv, hout=hout, hidx=hidx, S_eff=S_eff, ld=ld,
                          sc=torch.empty(p.wl.B * tc_max * ld, dtype=torch.float32, device=dev),
                          aws=torch.empty(max(1, dsa.dsa_sparse_attn_workspace_size(
                              p.wl.B, p.wl.T, p.wl.Hq, p.wl.d_v, p.wl.topk * p.wl.pool)), dtype=torch.uint8, device=dev),
                          ind_in=ev(), sel_done=ev(), idx_out=ev(), lay_in=[ev() for _ in range(nl)],
                          attn_done=[ev() for _ in range(nl)], out_out=[ev() for _ in range(nl)]))

    def step():
        for P in plans:
            p, w_ = P["p"], P["p"].wl
            with torch.cuda.stream(s_in):          # inputs in, each after its last reader
                s_in.wait_event(P["sel_done"])
                for k in P["host"]:
                    p.ind[k].copy_(P["host"][k], non_blocking=True)
                P["ind_in"].record(s_in)
                for l, L in enumerate(p.g.layers):
                    s_in.wait_event(P["attn_done"][l])
                    L["q"].copy_(P["hq"], non_blocking=True)
                    L["kv"].copy_(P["hkv"], non_blocking=True)
                    P["lay_in"][l].record(s_in)
            stream.wait_event(P["ind_in"])         # the selection, per query chunk
            stream.wait_event(P["idx_out"])
            keys = p.ind["k_idx"]
            if w_.pool > 1:
                keys = dsa.dsa_index_pool(p.ind["k_idx"], pool=w_.pool, stream=stream)
            for t0 in range(0, w_.T, t_chunk):
                tc = min(t_chunk, w_.T - t0)
                sc = P["sc"][: w_.B * tc * P["ld"]].view(w_.B, tc, P["ld"])
                dsa.dsa_index_scores(p.ind["q_idx"], p.ind["w"], keys, p.ind["ctx_len"], pool=w_.pool,
                                     t_begin=t0, t_count=tc, scores=sc, stream=stream)
                dsa.dsa_topk(sc, p.ind["ctx_len"], w_.T, P["S_eff"], w_.topk, pool=w_.pool, t_begin=t0, idx=p.g.idx,
                             stream=stream)
            P["sel_done"].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(P["sel_done"])
                P["hidx"].copy_(p.g.idx, non_blocking=True)
                P["idx_out"].record(s_out)
            for l, L in enumerate(p.g.layers):     # the layers, each output out as soon as written
                stream.wait_event(P["lay_in"][l])
                stream.wait_event(P["out_out"][l])
                dsa.dsa_sparse_attn(L["q"], L["kv"], p.g.idx, w_.sm_scale, w_.d_v, v=L["v"], out=L["out"],
                                    ws=P["aws"], stream=stream)
                P["attn_done"][l].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(P["attn_done"][l])
                    P["hout"].copy_(L["out"], non_blocking=True)
                    P["out_out"][l].record(s_out)

    def run(steps):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for _ in range(steps):
            step()
        for P in plans:                             # the end mark follows every copy out
            stream.wait_event(P["idx_out"])
            for e in P["out_out"]:
                stream.wait_event(e)
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    run(1)
    steps = max(1, min(args.steps, args.e2e_steps))
    ms = run(steps) / steps
    del plans
    return {"value": wl.B * wl.T / (ms / 1e3), "unit": "query tok/s", "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "copies": "one stream per direction, overlapping the compute and each other (per layer)"}


def run_secondary(args, name, dev, steps=3, per_layer=False):
    """Another workload (decode) or the per-layer-indexer comparator, timed the same way."""
    import indexed_sparse_attention_fp8_b200 as dsa
    stream = torch.cuda.current_stream()
    wl = W.WORKLOADS[name]
    if not per_layer:
        parts = make_parts(wl, dev, dsa, rank_boxes(wl, 1, 0))
        g = parts[0].g
        t_chunk = max(1, min(wl.T, (args.score_ws_gb << 30) // (wl.B * ((wl.S // wl.pool + 3) // 4 * 4) * 4)))
        ws = torch.empty(g.workspace_size(t_chunk), dtype=torch.uint8, device=dev)
        fn = lambda: parts[0].step(ws, stream)  # noqa: E731
        for _ in range(max(3, args.warmup)):
            fn()
        graph = None
        if wl.T == 1:
            # a decode step is a short chain of launches: it runs as one CUDA graph, as a serving
            # loop would run it, so the host's launch path does not set its pace
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                parts[0].step(ws, torch.cuda.current_stream())
            fn = graph.replay
            for _ in range(3):
                fn()
        ms = time_region(fn, steps, stream) / steps
        brk = breakdown(parts, ws, t_chunk, stream, dsa, 3)
        r = {"workload": name, "value": wl.B * wl.T / (ms / 1e3), "unit": "query tok/s", "ms_per_step": ms,
             "steps": steps, "cuda_graph": graph is not None, "breakdown_ms": brk,
             "roofline": roofline([parts[0].wl], brk, peaks(), t_chunk)}
        del graph
        del g, ws, parts
        torch.cuda.empty_cache()
        return r
    # per-layer indexer: each layer runs its own indexer + top-k (group_size 1, own indexer inputs)
    inds = [W.make_indexer_inputs(wl, device=dev, layer=l) for l in range(wl.group)]
    q0 = W.make_attn_inputs(wl, 0, device=dev)["q"]   # q shared across layers to fit memory (same work)
    lays = [{"q": q0, "kv": W.make_attn_inputs(wl, l, device=dev)["kv"], "v": None} for l in range(wl.group)]
    outbuf = torch.empty((wl.B, wl.T, wl.Hq, wl.d_v), dtype=torch.bfloat16, device=dev)
    gs = [dsa.Group(inds[l]["q_idx"], inds[l]["w"], inds[l]["k_idx"], inds[l]["ctx_len"], wl.topk,
                    [dict(lays[l], out=outbuf)], wl.sm_scale, wl.d_v) for l in range(wl.group)]
    t_chunk = max(1, min(wl.T, (args.score_ws_gb << 30) // (wl.B * ((wl.S + 3) // 4 * 4) * 4)))
    ws = torch.empty(gs[0].workspace_size(t_chunk), dtype=torch.uint8, device=dev)
    fn = lambda: [g.forward(ws, stream) for g in gs]  # noqa: E731
    fn()
    ms = time_region(fn, steps, stream) / steps
    r = {"workload": name + " per-layer indexer", "value": wl.B * wl.T / (ms / 1e3), "unit": "query tok/s",
         "ms_per_step": ms, "steps": steps}
    del gs, ws, inds, lays, outbuf
    torch.cuda.empty_cache()
    return r


# ------------------------------------------------------------------------------ oracle arm

_ORACLE_CACHE = {}


def _oracle_inputs(wl):
    """CPU inputs for timing the oracle: one sequence's full key caches (decoded once, input
    conversion outside the timed region) and 64 query rows, from the same seeded generators."""
    import oracle as O
    if wl.name in _ORACLE_CACHE:
        return _ORACLE_CACHE[wl.name]
    small = wl.replace(B=1, T=min(wl.T, 64))
    ind = W.make_indexer_inputs(small, device="cpu")
    kdec = O.e4m3_to_f64(ind["k_idx"][0].numpy())
    kp = O.e4m3_to_f64(O.index_pool(ind["k_idx"][0].numpy())) if wl.pool > 1 else None
    layers = []
    for l in range(wl.group):
        a = W.make_attn_inputs(small.replace(T=1), l, device="cpu")
        K = O.bf16_to_f64(a["kv"][0].view(torch.int16).numpy().view(np.uint16))
        V = K[:, : wl.d_v] if wl.kv_latent else O.bf16_to_f64(a["v"][0].view(torch.int16).numpy().view(np.uint16))
        q = O.bf16_to_f64(a["q"][0, 0].view(torch.int16).numpy().view(np.uint16))
        layers.append({"q": q, "K": K, "V": V})
    qrows = [O.e4m3_to_f64(ind["q_idx"][0, i].numpy()) for i in range(small.T)]
    wrows = [ind["w"][0, i].numpy() for i in range(small.T)]
    _ORACLE_CACHE[wl.name] = (kdec, kp, layers, qrows, wrows)
    return _ORACLE_CACHE[wl.name]


def oracle_threads() -> int:
    """Threads the oracle's numpy runs on: its BLAS thread pool (all host cores by default)."""
    try:
        from threadpoolctl import threadpool_info
        n = max((i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"), default=0)
    except Exception:
        n = 0
    return n or os.cpu_count() or 1


def oracle_sample(wl, seconds: float, seed: int = 0):
    """Time the CPU oracle, as it stands, on query rows drawn uniformly from the workload's
    positions: per row the indexer over every visible key, the top-k, and the attention of
    every layer of the group.  Returns (rows/s, rows, threads, seconds spent)."""
    import oracle as O
    kdec, kp, layers, qrows, wrows = _oracle_inputs(wl)
    rng = np.random.default_rng(seed)
    rows, spent = 0, 0.0
    while spent < seconds:
        t = int(rng.integers(0, wl.T))
        pos = wl.ctx - wl.T + t
        s0 = time.perf_counter()
        O.group_forward_row(qrows[t % len(qrows)], wrows[t % len(wrows)], kdec, pos, wl.topk, layers, wl.sm_scale,
                            wl.pool, kp)
        spent += time.perf_counter() - s0
        rows += 1
    return rows / spent, rows, oracle_threads(), spent


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wl = W.WORKLOADS[args.workload]
    per_step = max(1.0, args.ref_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(wl, per_step * 0.2)
    vals, rows_tot, spent_tot = [], 0, 0.0
    for s in range(args.steps):
        v, rows, cores, spent = oracle_sample(wl, per_step, seed=s)
        vals.append(v)
        rows_tot += rows
        spent_tot += spent
    value = rows_tot / spent_tot
    note = (f"{rows_tot} query rows sampled uniformly from {wl.name}; each row = indexer over all visible keys, "
            f"top-{wl.topk}, sparse attention for {wl.group} layers, fp64 numpy; key caches decoded once outside timing; "
            f"ms_per_step extrapolates the sampled rate to all {wl.B * wl.T} query rows of one step")
    return {"metric": METRIC, "value": value, "unit": "query tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": wl.B * wl.T * 1e3 / value, "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "ctx": wl.ctx, "topk": wl.topk, "group": wl.group},
            "cpu_baseline": {"value": value, "unit": "query tok/s", "cores": cores, "kind": "oracle",
                             "sample": note},
            "e2e": {"value": value, "unit": "query tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill128k", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--t-chunk", type=int, default=0)
    ap.add_argument("--T", type=int, default=0, help="override the number of new queries (small profiling cases)")
    ap.add_argument("--score-ws-gb", type=int, default=8, help="GiB of workspace for indexer score chunks")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--ref-seconds", type=float, default=60.0)
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        # one process per GPU: N GPUs need N ranks (torch.distributed.run --nproc-per-node N)
        sys.stderr.write(f"bench.py --gpus {args.gpus} needs {args.gpus} ranks, found WORLD_SIZE={world}: run it "
                         f"under python -m torch.distributed.run --nproc-per-node {args.gpus}\n")
        sys.exit(2)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                             timeout=datetime.timedelta(seconds=600))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    res, wl, parts = run_ours(args, rank, world, dev)
    if not args.no_e2e:
        try:
            e2e = run_e2e(args, wl, parts, dev, torch.cuda.current_stream(), world)
        except (RuntimeError, torch.cuda.OutOfMemoryError) as e:  # pinned host memory can run out
            e2e = {"error": str(e)[:300]}
        # every rank joins the reduction, a failed one with an infinite time
        ms = max_over_ranks(e2e.get("ms_per_step", math.inf), world, dev)
        h2d = sum_over_ranks(e2e.get("h2d_bytes_per_step", 0), world, dev)
        d2h = sum_over_ranks(e2e.get("d2h_bytes_per_step", 0), world, dev)
        if "error" not in e2e:
            if math.isfinite(ms):
                # every query row crosses once per step, spread over the ranks; bytes of all ranks
                e2e.update(value=wl.B * wl.T / (ms / 1e3), ms_per_step=ms, h2d_bytes_per_step=int(h2d),
                           d2h_bytes_per_step=int(d2h))
            else:
                e2e = {"error": "the end-to-end step failed on another rank"}
        res["e2e"] = e2e
    del parts
    torch.cuda.empty_cache()
    if world > 1:
        torch.distributed.barrier()
    if world == 1 and not args.no_secondary and args.workload == "prefill128k":
        try:
            pl = run_secondary(args, "prefill128k", dev, steps=2, per_layer=True)
            pl["indexshare_speedup"] = pl["ms_per_step"] / res["ms_per_step"]
            res["per_layer_indexer"] = pl
        except torch.cuda.OutOfMemoryError as e:  # pragma: no cover
            res["per_layer_indexer"] = {"error": str(e)[:200]}
        res["decode256k"] = run_secondary(args, "decode256k", dev, steps=10)
        # IndexPool at decode: 4 keys pooled into one, top-512 blocks
        res["decode256k_pool"] = run_secondary(args, "decode256k_pool", dev, steps=10)
        # IndexPool at a 1M-token cache: 8192 new queries, without and with pooling of 4 keys
        for name in ("chunk1m", "chunk1m_pool"):
            try:
                res[name] = run_secondary(args, name, dev, steps=2)
            except torch.cuda.OutOfMemoryError as e:  # pragma: no cover
                res[name] = {"error": str(e)[:200]}
        if "ms_per_step" in res["chunk1m"] and "ms_per_step" in res["chunk1m_pool"]:
            res["indexpool_speedup_1m"] = res["chunk1m"]["ms_per_step"] / res["chunk1m_pool"]["ms_per_step"]
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        v, rows, cores, spent = oracle_sample(W.WORKLOADS[args.workload], args.cpu_seconds)
        res["cpu_baseline"] = {"value": v, "unit": "query tok/s", "cores": cores, "kind": "oracle",
                               "sample": f"{rows} query rows of {args.workload} in {spent:.1f}s (indexer row + "
                                         f"top-k + {W.WORKLOADS[args.workload].group} attention layers, fp64)"}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
