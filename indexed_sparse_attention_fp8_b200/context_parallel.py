"""Context parallelism: one sequence's key caches sharded over ranks, one process per GPU.

Where the query-row sharding of `shard.py` replicates the key caches, this form gives rank r
only the contiguous key rows [s0_r, s0_r + len_r) of every sequence (the indexer keys and each
layer's latent rows), for contexts whose caches or whose indexer work one GPU should not carry
alone.  The path then has two real exchange steps, both all-gathers (NCCL over NVLink in use):
  1. selection: each rank scores and selects its own keys (the ordinary indexer and top-k, with
     its context lengths shifted by -s0), turns its selection into (score, global id)
     candidates, and after the all-gather every rank merges the candidates of all ranks into the
     exact top-k of the whole row (dsa_topk_merge): the same ids as one GPU selecting over all keys;
  2. attention, per layer: each rank attends over the selected keys it holds (the others
     localised to -1), and after the all-gather of the ranks' (O, lse) every rank merges them
     (dsa_attn_combine).
Every step runs in the library's kernels (dsa.h, "Context parallelism"); this module plans the
shards and orders the calls and the exchanges.  The steps are separate functions, so a caller can
run them for all ranks in one process too (the tests do, joining the ranks' tensors in place of
the all-gather).  IndexPool is not supported here (pool 1).  The merge holds at most 16384
candidates per row, so world * k <= 16384 (eight ranks at k = 2048).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch


MERGE_MAX_CANDIDATES = 16384   # candidates per row dsa_topk_merge accepts (n_parts * kc)


def key_shards(S: int, world: int, align: int = 128) -> List[Tuple[int, int]]:
    """Contiguous key ranges (s0, length) of `world` ranks covering [0, S): lengths multiples
    of `align` (one indexer key tile) except the last, as even as that allows; ranks past the
    end get empty ranges."""
    if world < 1 or align < 1:
        raise ValueError("world and align must be positive")
    tiles = -(-S // align)
    base, extra = divmod(tiles, world)
    out, s = [], 0
    for r in range(world):
        n = (base + (1 if r < extra else 0)) * align
        e = min(S, s + n)
        out.append((s, e - s))
        s = e
    return out


class Rank:
    """One rank's share: its key shard (s0, length), its shard of the indexer keys and of every
    layer's latent rows, and its context lengths relative to the shard."""

    def __init__(self, shard: Tuple[int, int], q_idx: torch.Tensor, w: torch.Tensor, k_idx_shard: torch.Tensor,
                 ctx_len: torch.Tensor, kv_shards: Sequence[torch.Tensor], S_total: int):
        self.s0, self.len = shard
        self.q_idx, self.w, self.k_idx = q_idx, w, k_idx_shard
        self.ctx_len = ctx_len
        self.ctx_local = (ctx_len - self.s0).contiguous()   # positions relative to the shard
        self.kv = list(kv_shards)
        self.S_total = S_total


def select_candidates(dsa, rk: Rank, k: int, t_begin: int, t_count: int, idx_local: torch.Tensor,
                      stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Step 1 of a query chunk on one rank: its shard's scores and top-k, as (score, global id)
    candidates [B, t_count, k]."""
    if rk.len == 0:   # a rank past the cache's end holds no keys: no candidates
        B = rk.q_idx.shape[0]
        return (torch.full((B, t_count, k), float("-inf"), device=rk.q_idx.device),
                torch.full((B, t_count, k), -1, dtype=torch.int32, device=rk.q_idx.device))
    sc = dsa.dsa_index_scores(rk.q_idx, rk.w, rk.k_idx, rk.ctx_local, t_begin=t_begin, t_count=t_count, stream=stream)
    T = rk.q_idx.shape[1]
    dsa.dsa_topk(sc, rk.ctx_local, T, rk.len, k, t_begin=t_begin, idx=idx_local, stream=stream)
    return dsa.dsa_gather_selected(sc, idx_local, t_begin, rk.s0, stream=stream)


def merge_selection(dsa, cand_score: torch.Tensor, cand_id: torch.Tensor, ctx_len: torch.Tensor, T: int, S_total: int,
                    k: int, t_begin: int, idx: torch.Tensor, stream=None) -> torch.Tensor:
    """Step 2, on every rank after the all-gather ([world, B, t_count, k] each): the exact top-k."""
    return dsa.dsa_topk_merge(cand_score, cand_id, ctx_len, T, S_total, k, t_begin=t_begin, idx=idx, stream=stream)


def attend_local(dsa, rk: Rank, layer: int, q: torch.Tensor, idx: torch.Tensor, sm_scale: float, d_v: int,
                 stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Step 3, per layer on one rank: attention over the selected keys this rank holds
    (normalised over them, with their log-sum-exp; -inf where it holds none)."""
    if rk.len == 0:   # no keys here: an empty part (weight zero in the merge)
        B, T, Hq = q.shape[:3]
        return (torch.zeros((B, T, Hq, d_v), dtype=torch.bfloat16, device=q.device),
                torch.full((B, T, Hq), float("-inf"), device=q.device))
    loc = dsa.dsa_idx_localize(idx, rk.s0, rk.len, stream=stream)
    return dsa.dsa_sparse_attn(q, rk.kv[layer], loc, sm_scale, d_v, want_lse=True, stream=stream)


def combine(dsa, part_o: torch.Tensor, part_lse: torch.Tensor, want_lse: bool = True, stream=None):
    """Step 4, per layer on every rank after the all-gather ([world, ...] each)."""
    return dsa.dsa_attn_combine(part_o, part_lse, want_lse=want_lse, stream=stream)


def group_forward(dsa, rk: Rank, qs: Sequence[torch.Tensor], k: int, sm_scale: float, d_v: int,
                  all_gather: Callable[[torch.Tensor], torch.Tensor], t_chunk: Optional[int] = None, stream=None):
    """One IndexShare group on this rank: the selection (shared by the layers) and every
    layer's attention, each followed by its exchange.  `all_gather(t)` returns the ranks'
    tensors stacked as [world, *t.shape] (rank order), e.g. torch.distributed's
    all_gather_into_tensor.  Returns (idx [B, T, k] global ids, [(out, lse)] per layer), the
    same on every rank."""
    B, T = rk.q_idx.shape[:2]
    dev = rk.q_idx.device
    t_chunk = T if t_chunk is None else max(1, min(t_chunk, T))
    idx_local = torch.full((B, T, k), -1, dtype=torch.int32, device=dev)
    idx = torch.full((B, T, k), -1, dtype=torch.int32, device=dev)
    for t0 in range(0, T, t_chunk):
        tc = min(t_chunk, T - t0)
        cs, ci = select_candidates(dsa, rk, k, t0, tc, idx_local, stream=stream)
        cs_all, ci_all = all_gather(cs), all_gather(ci)
        if cs_all.shape[0] * k > MERGE_MAX_CANDIDATES:   # the same on every rank: all stop here
            raise ValueError(f"{cs_all.shape[0]} ranks x k={k} candidates exceed the merge's "
                             f"{MERGE_MAX_CANDIDATES} per row")
        merge_selection(dsa, cs_all, ci_all, rk.ctx_len, T, rk.S_total, k, t0, idx, stream=stream)
    outs = []
    for layer, q in enumerate(qs):
        o, lse = attend_local(dsa, rk, layer, q, idx, sm_scale, d_v, stream=stream)
        outs.append(combine(dsa, all_gather(o), all_gather(lse), stream=stream))
    return idx, outs


def nccl_all_gather(group=None) -> Callable[[torch.Tensor], torch.Tensor]:
    """An all_gather for group_forward over a torch.distributed process group (NCCL for CUDA
    tensors, gloo for CPU tensors): [world, *t.shape] in rank order."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        # flat views: NCCL takes a stacked output, gloo only the flat (concatenated) form
        dist.all_gather_into_tensor(out.view(-1), t.contiguous().view(-1), group=group)
        return out
    return gather
