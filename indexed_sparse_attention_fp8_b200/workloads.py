"""Seeded synthetic workloads for the DSA layer group (indexer -> top-k -> sparse attention).

This module only *makes inputs*: shapes, seeds and value distributions.  It holds none of
the method's arithmetic, and it is the one module that both the CUDA path's callers
(tests, bench, smoke) and the CPU oracle's callers share.  It never imports the oracle or
the native library.

Workloads (all on one GPU, synthetic data, no trained weights):

  tiny    : 1 seq, L=2048 causal; indexer H_I=4, d_I=64; top-k 256; attention 16 q heads
            over one KV head with separate K and V, d=128.
  prefill32k  : 1 seq, L=32768; indexer H_I=64, d_I=128; top-k 2048; MLA-in-MQA attention,
            128 q heads over one latent row of 576 (K) whose first 512 columns are V.
  prefill128k : as prefill32k at L=131072, with 10% of keys carrying a planted signal
            aligned with a random later query, so the top-k is non-trivial.
  decode256k  : 32 seqs x 1 new token, each with a 262144-token cache; shapes as prefill32k.
  chunk1m : 8192 new queries at the end of a 1,048,576-token cache; shapes as prefill32k;
            plus the IndexPool variant (pool 4 keys, top-512 blocks -> 2048 tokens).
  decode256k_pool : decode256k with IndexPool (pool 4 keys, top-512 blocks -> 2048 tokens).

Value distributions: indexer q/k = e4m3(N(0,1)*0.5) (round-to-nearest-even, no scale),
w = N(0,1)/2 (tiny) or N(0,1)/8 (others) in fp32, attention q/K/V = bf16(N(0,1)).
Each tensor draws from its own torch.Generator seeded from (workload seed, tensor id,
layer), on the device the tensors are made on.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int            # sequences
    T: int            # new queries per sequence (at the end of the context)
    ctx: int          # keys visible to the last query (= cache length incl. the new tokens)
    H_I: int          # indexer heads
    d_I: int          # indexer head dim
    w_std: float      # std of the indexer head weights
    topk: int         # selected keys per query
    Hq: int           # attention query heads (all share one KV head)
    d_qk: int         # q/K head dim
    d_v: int          # V head dim
    kv_latent: bool   # True: V aliases the first d_v columns of the K row (MLA latent)
    group: int = 4    # layers sharing one indexer + top-k (IndexShare)
    pool: int = 1     # IndexPool factor (1 = off)
    planted_frac: float = 0.0  # fraction of keys that carry a planted signal

    @property
    def S(self) -> int:  # rows of the key caches
        return self.ctx

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_qk)

    def pos(self, b: int, t: int) -> int:
        """Absolute position of query t of sequence b: queries sit at the end of the context."""
        return self.ctx - self.T + t

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 0, B=1, T=2048, ctx=2048, H_I=4, d_I=64, w_std=0.5, topk=256,
                     Hq=16, d_qk=128, d_v=128, kv_latent=False),
    "prefill32k": Workload("prefill32k", 1, B=1, T=32768, ctx=32768, H_I=64, d_I=128, w_std=0.125,
                           topk=2048, Hq=128, d_qk=576, d_v=512, kv_latent=True),
    "prefill128k": Workload("prefill128k", 2, B=1, T=131072, ctx=131072, H_I=64, d_I=128,
                            w_std=0.125, topk=2048, Hq=128, d_qk=576, d_v=512, kv_latent=True,
                            planted_frac=0.10),
    "decode256k": Workload("decode256k", 3, B=32, T=1, ctx=262144, H_I=64, d_I=128, w_std=0.125,
                           topk=2048, Hq=128, d_qk=576, d_v=512, kv_latent=True),
    "chunk1m": Workload("chunk1m", 4, B=1, T=8192, ctx=1048576, H_I=64, d_I=128, w_std=0.125,
                        topk=2048, Hq=128, d_qk=576, d_v=512, kv_latent=True),
}
# IndexPool variant of the 1M chunked prefill: 4 keys pooled into one, top-512 blocks.
WORKLOADS["chunk1m_pool"] = WORKLOADS["chunk1m"].replace(name="chunk1m_pool", pool=4, topk=512)
# IndexPool at decode: the 32 x 256K decode batch with 4 keys pooled into one, top-512 blocks
# (2048 tokens), so the decode indexer reads a quarter of the keys.
WORKLOADS["decode256k_pool"] = WORKLOADS["decode256k"].replace(name="decode256k_pool", pool=4, topk=512)

# Tensor ids for the per-tensor generators.
_TID = {"q_idx": 1, "w": 2, "k_idx": 3, "q": 4, "kv": 5, "v": 6, "plant": 7}


def _gen(device, seed: int, tid: int, layer: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tid * 7919 + layer * 104_729) & 0x7FFF_FFFF_FFFF)
    return g


def _randn(shape, g, device, dtype=torch.float32, chunk_elems: int = 1 << 28) -> torch.Tensor:
    """N(0,1) samples, drawn in chunks along dim 0 so no fp32 temporary exceeds ~1 GiB."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=g, device=device, dtype=torch.float32).to(dtype)
    return out


def _to_e4m3_bytes(x: torch.Tensor) -> torch.Tensor:
    """fp32 -> e4m3 codes (uint8) by torch's round-to-nearest-even cast, saturating at 448."""
    return x.clamp_(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def make_indexer_inputs(wl: Workload, device="cpu", layer: int = 0):
    """Indexer tensors of one IndexShare group (layer selects an independent draw, used by the
    per-layer-indexer comparator).

    Returns dict with q_idx [B,T,H_I,d_I] u8 (e4m3 codes), w [B,T,H_I] f32,
    k_idx [B,S,d_I] u8, ctx_len [B] i32.
    """
    B, T, S, H, D = wl.B, wl.T, wl.S, wl.H_I, wl.d_I
    q_idx = _to_e4m3_bytes(_randn((B, T, H, D), _gen(device, wl.seed, _TID["q_idx"], layer), device).mul_(0.5))
    w = _randn((B, T, H), _gen(device, wl.seed, _TID["w"], layer), device).mul_(wl.w_std)
    gk = _gen(device, wl.seed, _TID["k_idx"], layer)
    k_idx = torch.empty((B, S, D), dtype=torch.uint8, device=device)
    step = 1 << 20
    for b in range(B):
        for s0 in range(0, S, step):
            s1 = min(S, s0 + step)
            blk = torch.randn((s1 - s0, D), generator=gk, device=device).mul_(0.5)
            if wl.planted_frac > 0.0:
                _plant(wl, blk, s0, b, q_idx, w, device, layer)
            k_idx[b, s0:s1] = _to_e4m3_bytes(blk)
    ctx_len = torch.full((B,), wl.ctx, dtype=torch.int32, device=device)
    return {"q_idx": q_idx, "w": w, "k_idx": k_idx, "ctx_len": ctx_len}


def _plant(wl: Workload, kblk: torch.Tensor, s0: int, b: int, q_idx, w, device, layer: int):
    """Planted signal: a random 10% of keys s get, added to their fp32 value before e4m3
    rounding, a vector of norm 3 * (typical key norm 0.5*sqrt(d_I)) pointing along
    g = sum_j max(w[t_s,j],0) * q[t_s,j,:] for a random later query t_s in [s, L).  Planted
    pairs then span every distance.  (Input construction only.)"""
    n, D = kblk.shape
    g = _gen(device, wl.seed, _TID["plant"], layer * 65536 + b * 4096 + s0 // (1 << 20))
    chosen = torch.rand(n, generator=g, device=device) < wl.planted_frac
    rows = torch.nonzero(chosen).flatten()
    if rows.numel() == 0:
        return
    s_abs = rows + s0
    # query index (not position) of a random later query; queries are at the end of the ctx
    first_q_pos = wl.ctx - wl.T
    lo = torch.clamp(s_abs - first_q_pos, min=0)
    u = torch.rand(rows.numel(), generator=g, device=device)
    t_s = (lo + (u * (wl.T - lo).to(torch.float32)).long()).clamp_(max=wl.T - 1)
    qf = q_idx[b, t_s].view(torch.float8_e4m3fn).to(torch.float32)        # [n, H, D]
    wp = torch.clamp(w[b, t_s], min=0.0).unsqueeze(-1)                      # [n, H, 1]
    gdir = (wp * qf).sum(dim=1)                                             # [n, D]
    gdir = gdir / gdir.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    kblk[rows] += (3.0 * 0.5 * math.sqrt(D)) * gdir


def make_attn_inputs(wl: Workload, layer: int, device="cpu", dtype=torch.bfloat16):
    """Attention tensors of one layer: q [B,T,Hq,d_qk] bf16; kv [B,S,d_qk] bf16 (the latent
    row, or K); v [B,S,d_v] bf16 (None when V aliases kv[..., :d_v])."""
    B, T, S = wl.B, wl.T, wl.S
    q = _randn((B, T, wl.Hq, wl.d_qk), _gen(device, wl.seed, _TID["q"], layer), device, dtype)
    kv = _randn((B, S, wl.d_qk), _gen(device, wl.seed, _TID["kv"], layer), device, dtype)
    v = None
    if not wl.kv_latent:
        v = _randn((B, S, wl.d_v), _gen(device, wl.seed, _TID["v"], layer), device, dtype)
    return {"q": q, "kv": kv, "v": v}


def small_case(name: str = "tiny", **overrides) -> Workload:
    """A workload of the named family with some fields overridden (used for parity cases
    small enough for the oracle to finish in seconds)."""
    return WORKLOADS[name].replace(**overrides)
