"""Context parallelism (key shards over ranks): the plan and the exchange on CPU (gloo, two
processes), and on the GPU the whole path for 2, 3 and 4 ranks run in one process, the ranks'
tensors joined in place of the all-gather: the merged selection equals the single-GPU selection
id for id, and each layer's merged attention matches the single-GPU output and the oracle."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from indexed_sparse_attention_fp8_b200 import context_parallel as cp


@pytest.mark.parametrize("S,world", [(20000, 2), (262144, 8), (300, 4), (128, 1), (1000, 3)])
def test_key_shards_cover_the_cache_in_aligned_contiguous_ranges(S, world):
    sh = cp.key_shards(S, world)
    assert len(sh) == world
    assert sh[0][0] == 0 and sum(n for _, n in sh) == S
    for (s0, n), (s1, _) in zip(sh, sh[1:]):
        assert s1 == s0 + n                       # contiguous, in rank order
    full = [n for _, n in sh if n > 0]
    assert all(n % 128 == 0 for n in full[:-1])   # whole key tiles except the last
    tiles = [-(-n // 128) for _, n in sh]
    assert max(tiles) - min(t for t in tiles) <= 1 or sh[-1][1] == 0 or S < 128 * world


def _gather_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = cp.nccl_all_gather()
        t = torch.arange(6, dtype=torch.float32).view(2, 3) + 100 * rank
        out = g(t)
        q.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


def test_exchange_stacks_the_ranks_in_rank_order():
    """The all-gather that group_forward uses, over a real process group (gloo, two ranks)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    ps = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    got = dict(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = np.stack([np.arange(6, dtype=np.float32).reshape(2, 3) + 100 * r for r in range(2)])
    for r in range(2):
        assert np.array_equal(got[r], want)


# ---------------------------------------------------------------- GPU

def _emulate(dsa, wl, ind, lays, world, t_chunk):
    """Every rank's steps in one process; the ranks' tensors stacked in place of the all-gather."""
    S = ind["k_idx"].shape[1]
    shards = cp.key_shards(S, world)
    ranks = [cp.Rank(sh, ind["q_idx"], ind["w"], ind["k_idx"][:, sh[0]:sh[0] + sh[1]].contiguous(), ind["ctx_len"],
                     [L["kv"][:, sh[0]:sh[0] + sh[1]].contiguous() for L in lays], S) for sh in shards]
    B, T = ind["q_idx"].shape[:2]
    idx = torch.full((B, T, wl.topk), -1, dtype=torch.int32, device="cuda")
    idx_locals = [torch.full((B, T, wl.topk), -1, dtype=torch.int32, device="cuda") for _ in ranks]
    for t0 in range(0, T, t_chunk):
        tc = min(t_chunk, T - t0)
        parts = [cp.select_candidates(dsa, rk, wl.topk, t0, tc, il) for rk, il in zip(ranks, idx_locals)]
        cp.merge_selection(dsa, torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]),
                           ind["ctx_len"], T, S, wl.topk, t0, idx)
    outs = []
    for layer, L in enumerate(lays):
        parts = [cp.attend_local(dsa, rk, layer, L["q"], idx, wl.sm_scale, wl.d_v) for rk in ranks]
        outs.append(cp.combine(dsa, torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts])))
    return idx, outs


@pytest.mark.gpu
@pytest.mark.parametrize("name,over,ctx,world,t_chunk", [
    # ragged contexts: one wholly inside rank 0, one of a single key, one ending mid-shard
    ("decode256k", dict(B=4, T=1, ctx=20000), [20000, 9000, 1, 12001], 2, 1),
    ("decode256k", dict(B=3, T=1, ctx=33000), [33000, 22100, 2048], 3, 1),
    ("prefill32k", dict(B=2, T=384, ctx=5000), [5000, 3000], 4, 160),
])
def test_context_parallel_equals_one_gpu(name, over, ctx, world, t_chunk):
    import indexed_sparse_attention_fp8_b200 as dsa
    from indexed_sparse_attention_fp8_b200 import workloads as W
    from tests import parity as P
    wl = W.WORKLOADS[name].replace(**over)
    ind = W.make_indexer_inputs(wl, device="cuda")
    ind["ctx_len"] = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    lays = [W.make_attn_inputs(wl, l, device="cuda") for l in range(2)]
    ref_idx, ref_outs = dsa.dsa_group_forward(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], wl.topk,
                                              [dict(L) for L in lays], wl.sm_scale, wl.d_v)
    idx, outs = _emulate(dsa, wl, ind, lays, world, t_chunk)
    assert torch.equal(idx, ref_idx)                        # the selection, id for id
    assert dsa.dsa_device_status() == 0
    idx_h = P.to_np(idx)
    for li, (L, (o, lse)) in enumerate(zip(lays, outs)):
        ref = ref_outs[li][0] if isinstance(ref_outs[li], tuple) else ref_outs[li]
        d = (o.float() - ref.float()).abs()
        assert float(d.max()) <= 2e-2 and float(d.mean()) <= 1e-3, (float(d.max()), float(d.mean()))
        for b, t in [(0, 0), (wl.B - 1, wl.T - 1), (0, wl.T // 2)]:
            Kb = P.bf16_np(L["kv"][b])
            msg = P.check_attn_row(P.bf16_np(o[b, t]), P.bf16_np(L["q"][b, t]), Kb, Kb[:, : wl.d_v], idx_h[b, t],
                                   wl.sm_scale, P.to_np(lse[b, t]).astype(np.float64))
            assert msg is None, f"layer {li} row {(b, t)}: {msg}"


@pytest.mark.gpu
def test_context_parallel_guards_skip_and_flag_bad_ids():
    """Ids that the exchange steps may not read are skipped and reported, not read: a selected id
    past the score row in the candidate gather; in the merge, a candidate id past the row's
    visible keys, and a row left with fewer than k candidates (written as all -1)."""
    import indexed_sparse_attention_fp8_b200 as dsa
    dev = "cuda"
    B, T, k, ld = 1, 2, 4, 64
    scores = torch.arange(B * T * ld, dtype=torch.float32, device=dev).view(B, T, ld)
    idx = torch.tensor([[[0, 5, 63, 64], [1, -1, 2, 10 ** 6]]], dtype=torch.int32, device=dev)
    assert dsa.dsa_device_status() == 0
    cs, ci = dsa.dsa_gather_selected(scores, idx, 0, 100)
    assert dsa.dsa_device_status() == 7
    assert ci.tolist() == [[[100, 105, 163, -1], [101, -1, 102, -1]]]
    assert cs[0, 0, :3].tolist() == [0.0, 5.0, 63.0] and cs[0, 1, 0].item() == 65.0
    assert torch.isinf(cs[0, 0, 3]) and torch.isinf(cs[0, 1, 3])
    # merge: two parts of k candidates for one row at position 99 of a 100-key context
    ctx = torch.tensor([100], dtype=torch.int32, device=dev)
    sc = torch.tensor([[[[9.0, 8.0, 7.0, 6.0]]], [[[5.0, 4.0, 3.0, 2.0]]]], device=dev)
    good = torch.tensor([[[[10, 20, 30, 40]]], [[[50, 60, 70, 80]]]], dtype=torch.int32, device=dev)
    out = dsa.dsa_topk_merge(sc, good, ctx, 1, 100, k)
    assert dsa.dsa_device_status() == 0
    assert out.tolist() == [[[10, 20, 30, 40]]]
    bad = good.clone()
    bad[0, 0, 0, 1] = 100          # not a visible key (positions 0..99): skipped
    out = dsa.dsa_topk_merge(sc, bad, ctx, 1, 100, k)
    assert dsa.dsa_device_status() == 7
    assert out.tolist() == [[[10, 30, 40, 50]]]
    few = torch.full_like(good, -1)
    few[0, 0, 0, :3] = torch.tensor([1, 2, 3], dtype=torch.int32)   # 3 < k candidates in all
    out = dsa.dsa_topk_merge(sc, few, ctx, 1, 100, k)
    assert dsa.dsa_device_status() == 7
    assert out.tolist() == [[[-1, -1, -1, -1]]]
