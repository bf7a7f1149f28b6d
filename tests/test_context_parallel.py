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


# ---------------------------------------------------------------- the whole key-sharded group
# over a real process group (gloo, three CPU ranks), with a stand-in for the library whose steps
# are the oracle's definitions: this checks group_forward's plan, its query chunks, its two
# exchanges and its merge order, not the kernels (those are the GPU tests above).

class _OracleSteps:
    """The library's step calls, computed on the CPU from the oracle's definitions (test only)."""

    def __init__(self):
        import oracle as O
        self.O = O

    def dsa_index_scores(self, q_idx, w, k_idx, ctx_len, t_begin=0, t_count=None, stream=None):
        O = self.O
        B, T = q_idx.shape[:2]
        S = k_idx.shape[1]
        ld = (S + 3) // 4 * 4
        out = torch.full((B, t_count, ld), float("-inf"))
        for b in range(B):
            kd = O.e4m3_to_f64(k_idx[b].numpy())
            for r in range(t_count):
                t = t_begin + r
                pos = int(ctx_len[b]) - T + t
                out[b, r, :S] = torch.from_numpy(O.index_scores_row(O.e4m3_to_f64(q_idx[b, t].numpy()),
                                                                    w[b, t].numpy(), kd, pos))
        return out

    def dsa_topk(self, sc, ctx_len, T, S, k, t_begin=0, idx=None, stream=None):
        B, tc = sc.shape[:2]
        for b in range(B):
            for r in range(tc):
                pos = int(ctx_len[b]) - T + t_begin + r
                n_valid = 0 if pos < 0 else min(S, pos + 1)
                sel = self.O.topk_row(sc[b, r].numpy(), n_valid, k)
                ids = np.sort(sel[sel >= 0])
                row = np.full(k, -1, dtype=np.int32)
                row[: ids.size] = ids
                idx[b, t_begin + r] = torch.from_numpy(row)
        return idx

    def dsa_gather_selected(self, sc, idx, t_begin, id_offset, stream=None):
        B, tc = sc.shape[:2]
        sel = idx[:, t_begin:t_begin + tc].long()
        cs = torch.where(sel >= 0, torch.gather(sc, 2, sel.clamp(min=0)), torch.tensor(float("-inf")))
        ci = torch.where(sel >= 0, sel + id_offset, torch.tensor(-1)).to(torch.int32)
        return cs.float(), ci

    def dsa_topk_merge(self, cs, ci, ctx_len, T, S_total, k, t_begin=0, idx=None, stream=None):
        P, B, tc, kc = cs.shape
        for b in range(B):
            for r in range(tc):
                pos = int(ctx_len[b]) - T + t_begin + r
                n_valid = 0 if pos < 0 else min(S_total, pos + 1)
                row = np.full(k, -1, dtype=np.int32)
                if n_valid <= k:
                    row[:n_valid] = np.arange(n_valid)
                else:
                    s = cs[:, b, r].reshape(-1).double().numpy()
                    i = ci[:, b, r].reshape(-1).numpy()
                    keep = i >= 0
                    s, i = s[keep], i[keep]
                    order = np.lexsort((i, -s))[:k]
                    row[:] = np.sort(i[order])
                idx[b, t_begin + r] = torch.from_numpy(row)
        return idx

    def dsa_idx_localize(self, idx, s0, s_len, stream=None):
        return torch.where((idx >= s0) & (idx < s0 + s_len), idx - s0, torch.tensor(-1, dtype=torch.int32)).to(torch.int32)

    def dsa_sparse_attn(self, q, kv, idx, sm_scale, d_v, want_lse=False, stream=None):
        O = self.O
        B, T, Hq = q.shape[:3]
        out = torch.empty((B, T, Hq, d_v), dtype=torch.bfloat16)
        lse = torch.empty((B, T, Hq), dtype=torch.float32)
        for b in range(B):
            K = kv[b].double().numpy()
            for t in range(T):
                o, l = O.sparse_attn_row(q[b, t].double().numpy(), K, K[:, :d_v], idx[b, t].numpy(), sm_scale)
                out[b, t] = torch.from_numpy(o).to(torch.bfloat16)
                lse[b, t] = torch.from_numpy(l).float()
        return out, lse

    def dsa_attn_combine(self, part_o, part_lse, want_lse=False, stream=None):
        lse = torch.logsumexp(part_lse.double(), dim=0)
        wgt = torch.exp(part_lse.double() - lse).nan_to_num(0.0)
        out = (wgt.unsqueeze(-1) * part_o.double()).sum(0)
        return out.to(torch.bfloat16), lse.float()


def _cp_inputs():
    g = torch.Generator().manual_seed(31)
    B, T, S, H, D, Hq, Dqk, Dv = 2, 6, 200, 4, 64, 4, 64, 32
    codes = torch.randint(0, 126, (B, S, D), generator=g, dtype=torch.int32).to(torch.uint8)
    q_idx = torch.randint(0, 126, (B, T, H, D), generator=g, dtype=torch.int32).to(torch.uint8)
    w = torch.randn((B, T, H), generator=g) * 0.5
    ctx = torch.tensor([200, 100], dtype=torch.int32)
    qs = [torch.randn((B, T, Hq, Dqk), generator=g).to(torch.bfloat16) for _ in range(2)]
    kvs = [torch.randn((B, S, Dqk), generator=g).to(torch.bfloat16) for _ in range(2)]
    return q_idx, w, codes, ctx, qs, kvs, 16, 1.0 / 8.0, Dv


def _cp_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q_idx, w, codes, ctx, qs, kvs, k, sm_scale, d_v = _cp_inputs()
        S = codes.shape[1]
        s0, n = cp.key_shards(S, world)[rank]
        rk = cp.Rank((s0, n), q_idx, w, codes[:, s0:s0 + n].contiguous(), ctx, [kv[:, s0:s0 + n].contiguous() for kv in kvs], S)
        idx, outs = cp.group_forward(_OracleSteps(), rk, qs, k, sm_scale, d_v, cp.nccl_all_gather(), t_chunk=4)
        q.put((rank, idx.numpy(), [(o.float().numpy(), l.numpy()) for o, l in outs]))
    finally:
        dist.destroy_process_group()


def test_key_sharded_group_over_three_cpu_ranks_matches_the_oracle():
    """Three gloo ranks (the last one holding no keys), two query chunks, ragged contexts (one
    sequence's keys all on the first rank): every rank ends with the unsharded selection of the
    oracle and its attention (bf16 parts merged by log-sum-exp)."""
    import oracle as O
    ctx_mp = mp.get_context("spawn")
    q = ctx_mp.Queue()
    port = 29700 + (os.getpid() % 1000)
    world = 3
    ps = [ctx_mp.Process(target=_cp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    got = dict((r, (i, o)) for r, i, o in (q.get(timeout=300) for _ in ps))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert cp.key_shards(200, 3)[2][1] == 0
    q_idx, w, codes, ctx, qs, kvs, k, sm_scale, d_v = _cp_inputs()
    B, T = q_idx.shape[:2]
    for b in range(B):
        kd = O.e4m3_to_f64(codes[b].numpy())
        layers = [{"q": qs[l][b].double().numpy(), "K": kvs[l][b].double().numpy(),
                   "V": kvs[l][b].double().numpy()[:, :d_v]} for l in range(2)]
        for t in range(T):
            pos = int(ctx[b]) - T + t
            idx_ref, outs_ref = O.group_forward_row(O.e4m3_to_f64(q_idx[b, t].numpy()), w[b, t].numpy(), kd, pos, k,
                                                    [dict(L, q=L["q"][t]) for L in layers], sm_scale)
            want = np.sort(idx_ref[idx_ref >= 0])
            for r in range(world):
                idx_r, outs_r = got[r]
                row = idx_r[b, t]
                assert np.array_equal(row[row >= 0], want) and (row[want.size:] == -1).all(), (r, b, t)
                for (o, l), (oref, lref) in zip(outs_r, outs_ref):
                    assert np.abs(o[b, t] - oref).max() <= 2e-2
                    assert np.abs(l[b, t] - lref).max() <= 1e-3 * max(1.0, np.abs(lref).max())


def test_group_refuses_more_candidates_than_the_merge_holds():
    """world x k above the merge's 16384 candidates per row stops at the first exchange (the
    check sees the gathered shape, so every rank stops at the same point)."""
    q_idx, w, codes, ctx, qs, kvs, _, sm_scale, d_v = _cp_inputs()
    S = codes.shape[1]
    rk = cp.Rank((0, S), q_idx, w, codes, ctx, kvs, S)
    nine = lambda t: torch.stack([t] * 9)   # noqa: E731  (nine ranks' worth of candidates)
    with pytest.raises(ValueError, match="exceed"):
        cp.group_forward(_OracleSteps(), rk, qs, 2048, sm_scale, d_v, nine, t_chunk=6)
