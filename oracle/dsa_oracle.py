"""CPU oracle for the DSA layer group: lightning indexer -> top-k -> sparse attention,
with IndexShare and IndexPool.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU-baseline leg
may import this module.  It shares no code with the CUDA library (no headers, helpers,
tables or constants) and imports nothing from it.  It is slow on purpose: plain numpy in
float64, one query row at a time, no blocking, fusion or reordering beyond what each
definition below states.

Sources (the pages describe the method in prose only):
  [DSA]   "GLM 5.2: How Four Co-Designed Mechanisms Beat Raw Scale", section "DeepSeek
          Sparse Attention": Stage 1 (coarse scoring: an indexer scores every token of the
          context for the current query) and Stage 2 (fine selection: the top-2,048 tokens
          get full attention).
  [SHARE] same page, section "IndexShare: Amortizing the Indexer": one indexer run per
          block of 4 layers, the selection shared across the block.
  [FP8]   twiscan.com post on GLM-5.2 ("I read the GLM-5.2 report ..."): the indexer scores
          the keys and keeps the top-k, and ranking is easy enough to run in FP8.
  [POOL]  "GLM-5.3-Flash hybrid sparse-linear attention with IndexPool", section "What
          changed": IndexPool pools four indexer keys into one.
  [ATTN]  "China's First Frontier Model?", section "The Time has Come": sparse attention
          attends only to the candidates the indexer selected, up to a fixed limit.

Readings taken where the pages are silent (each is listed with its reason in the design
notes of the repository):
  * indexer score  I[t,s] = sum_j w[t,j] * max(0, sum_d q_idx[t,j,d] * k_idx[s,d]), no
    extra scale (the head weights carry it);
  * FP8 = OCP e4m3 ("e4m3fn": bias 7, no infinities, max 448) with unit scale;
  * causality: query at position p sees keys 0..p (itself included); others score -inf;
  * top-k: the k_eff = min(k, n_valid) largest scores; ties broken by lower key index;
    fewer than k valid keys -> all of them, padded with -1;
  * attention: softmax(sm_scale * q.K) over the selected keys, times V; duplicates in the
    index list count twice; -1 entries are skipped;
  * IndexPool: pooled key b = e4m3(((k[4b]+k[4b+1]) + (k[4b+2]+k[4b+3])) * 0.25) computed
    in fp32 from the decoded keys; block b is valid for query position p iff 4b <= p; the
    top blocks expand to tokens 4b..4b+3, tokens beyond p become -1.  The same mean over
    P = 2 or 8 keys (a balanced pairwise fp32 sum times 1/P; validity P*b <= p, expansion to
    P tokens) generalises the pages' factor of four.

Parity status: every function here is pinned by tests that do not re-type its formula
(library routines, closed forms, brute force on tiny inputs, invariants).
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

# ----------------------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------------------


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode OCP FP8 E4M3 codes (uint8) exactly to float64.

    Layout S.EEEE.MMM, exponent bias 7.  Exponent field 0 is subnormal: (M/8) * 2^-6.
    Otherwise (1 + M/8) * 2^(E-7).  S.1111.111 is NaN; there are no infinities, so the
    largest finite magnitude is 1.75 * 2^8 = 448.  [FP8]
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = (m / 8.0) * 2.0 ** -6
    nrm = (1.0 + m / 8.0) * np.power(2.0, (e - 7).astype(np.float64))
    val = np.where(e == 0, sub, nrm)
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def f32_to_e4m3(x: np.ndarray) -> np.ndarray:
    """Encode float32 values to E4M3 codes: round to nearest, ties to even, and saturate
    magnitudes beyond the largest finite value (448) to 448.  NaN maps to 0x7F.

    Written from the format definition: a magnitude a in [2^e, 2^(e+1)) with e >= -6 has
    spacing 2^(e-3); below 2^-6 (subnormals) the spacing is 2^-9.  np.rint rounds half to
    even.  [POOL requantisation]
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    sign = np.where(np.signbit(x), 0x80, 0x00).astype(np.int64)
    a = np.abs(np.nan_to_num(x, nan=0.0))
    # subnormal range: multiples of 2^-9; q = 8 is the smallest normal (code 0x08)
    q_sub = np.rint(np.minimum(a, 1.0) / 2.0 ** -9).astype(np.int64)
    # normal range
    a_n = np.where((a > 0) & (a < 448.0), a, 1.0)        # saturated values handled below
    _, ex = np.frexp(a_n)                                 # a = m * 2^ex, m in [0.5, 1)
    e = ex.astype(np.int64) - 1                           # a in [2^e, 2^(e+1))
    q = np.rint((a_n / np.power(2.0, e) - 1.0) * 8.0).astype(np.int64)
    carry = q == 8
    e = np.where(carry, e + 1, e)
    q = np.where(carry, 0, q)
    code_n = np.minimum(((e + 7) << 3) | q, 0x7E)
    code = np.where(a < 2.0 ** -6, q_sub, code_n)
    code = np.where(a >= 448.0, 0x7E, code)
    code = code | sign
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    """Decode bfloat16 bit patterns (uint16) exactly: they are the top half of a float32."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):
        return u.view(np.float32).astype(np.float64)


def f64_to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


# ----------------------------------------------------------------------------------------
# Stage 1: lightning indexer  [DSA Stage 1, FP8]
# ----------------------------------------------------------------------------------------


def index_scores_row(q_t: np.ndarray, w_t: np.ndarray, k: np.ndarray, pos: int,
                     pool: int = 1) -> np.ndarray:
    """Indexer scores of one query against every key row of one sequence.

    q_t : [H_I, d_I] float64 (decoded e4m3), w_t : [H_I] float, k : [S', d_I] float64
    (decoded e4m3; S' pooled rows when pool > 1), pos : the query's absolute position.

    I[s] = sum_j w_t[j] * max(0, q_t[j] . k[s]) for valid keys, -inf otherwise, rounded once
    to float32.  Key row s is valid iff pool * s <= pos (pool = 1: the causal rule s <= pos).
    """
    S = k.shape[0]
    n_valid = min(S, pos // pool + 1)
    out = np.full(S, -np.inf, dtype=np.float32)
    if n_valid <= 0:
        return out
    logits = k[:n_valid] @ q_t.T                          # [n_valid, H_I]: q_t[j] . k[s]
    relu = np.maximum(logits, 0.0)
    out[:n_valid] = f64_to_f32(relu @ np.asarray(w_t, dtype=np.float64))
    return out


def index_scores(q_idx: np.ndarray, w: np.ndarray, k_idx: np.ndarray, ctx_len: Sequence[int],
                 rows: Optional[Sequence[tuple]] = None, pool: int = 1) -> Dict[tuple, np.ndarray]:
    """Indexer scores for the requested (b, t) rows (all rows when rows is None).

    q_idx [B,T,H_I,d_I] and k_idx [B,S,d_I] are e4m3 codes (uint8); w [B,T,H_I] fp32;
    query t of sequence b sits at position ctx_len[b] - T + t.  Returns {(b,t): f32 [S']}.
    """
    B, T = q_idx.shape[0], q_idx.shape[1]
    if rows is None:
        rows = [(b, t) for b in range(B) for t in range(T)]
    out = {}
    kcache = {}
    for (b, t) in rows:
        if b not in kcache:
            kcache = {b: e4m3_to_f64(k_idx[b])}
        pos = int(ctx_len[b]) - T + t
        out[(b, t)] = index_scores_row(e4m3_to_f64(q_idx[b, t]), w[b, t], kcache[b], pos, pool)
    return out


# ----------------------------------------------------------------------------------------
# Stage 2: top-k selection  [DSA Stage 2, ATTN]
# ----------------------------------------------------------------------------------------


def topk_row(scores: np.ndarray, n_valid: int, k: int) -> np.ndarray:
    """The k_eff = min(k, n_valid) best keys of one row, ordered by (score desc, index asc);
    int32 [k], padded with -1.  Only the first n_valid entries of the row are candidates."""
    n = int(min(n_valid, scores.shape[0]))
    out = np.full(k, -1, dtype=np.int32)
    if n <= 0:
        return out
    s = np.asarray(scores[:n], dtype=np.float64)
    order = np.lexsort((np.arange(n), -s))               # primary: -score, secondary: index
    keff = min(k, n)
    out[:keff] = order[:keff].astype(np.int32)
    return out


def expand_blocks(block_ids: np.ndarray, pos: int, pool: int) -> np.ndarray:
    """IndexPool expansion: each selected block b becomes tokens pool*b .. pool*b+pool-1;
    tokens beyond the query position (and padding blocks) become -1.  [POOL]"""
    out = np.full(block_ids.shape[0] * pool, -1, dtype=np.int32)
    for i, b in enumerate(block_ids):
        if b < 0:
            continue
        for r in range(pool):
            tok = pool * int(b) + r
            out[i * pool + r] = tok if tok <= pos else -1
    return out


# ----------------------------------------------------------------------------------------
# IndexPool key pooling  [POOL]
# ----------------------------------------------------------------------------------------


def index_pool(k_idx: np.ndarray, pool: int = 4) -> np.ndarray:
    """Pool groups of `pool` consecutive indexer keys (e4m3 codes [..., S, d]) into one:
    decode to fp32, sum the group as a balanced pairwise tree in fp32 (for the pages' four:
    ((k0 + k1) + (k2 + k3))), multiply by 1/pool, requantise to e4m3 (RNE, saturating).
    pool is 4 (the pages' factor) or 2 or 8.  Groups start at key 0; S must be a multiple of
    pool."""
    if pool not in (2, 4, 8):
        raise ValueError("IndexPool pools 2, 4 or 8 keys into one")
    kf = e4m3_to_f64(k_idx).astype(np.float32)            # exact: e4m3 values fit fp32
    S = kf.shape[-2]
    if S % pool:
        raise ValueError("key count must be a multiple of the pool factor")
    g = kf.reshape(kf.shape[:-2] + (S // pool, pool, kf.shape[-1]))
    parts = [g[..., r, :] for r in range(pool)]
    while len(parts) > 1:                                 # pairwise: (k0+k1), (k2+k3), ...
        parts = [parts[2 * i] + parts[2 * i + 1] for i in range(len(parts) // 2)]
    m = parts[0] * np.float32(1.0 / pool)                 # every op in fp32
    return f32_to_e4m3(m)


# ----------------------------------------------------------------------------------------
# Sparse attention over the selected keys  [DSA Stage 2, ATTN]
# ----------------------------------------------------------------------------------------


def sparse_attn_row(q_t: np.ndarray, K: np.ndarray, V: np.ndarray, idx_row: np.ndarray,
                    sm_scale: float):
    """Attention of one query (all heads) over the selected key rows.

    q_t [Hq, d_qk], K [S, d_qk], V [S, d_v] float64; idx_row [k] int (-1 = skip).
    O[h] = sum_i p[h,i] V[idx_i] with p[h,:] = softmax_i(sm_scale * q_t[h] . K[idx_i]);
    lse[h] = log sum_i exp(sm_scale * q_t[h] . K[idx_i]).  Max-subtracted for range only.
    Returns (O [Hq, d_v] float64, lse [Hq] float64).  No selected key: O = 0, lse = -inf.
    """
    sel = np.asarray([i for i in idx_row if i >= 0], dtype=np.int64)
    Hq = q_t.shape[0]
    if sel.size == 0:
        return np.zeros((Hq, V.shape[1])), np.full(Hq, -np.inf)
    logits = (q_t @ K[sel].T) * sm_scale                  # [Hq, n]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    denom = p.sum(axis=1, keepdims=True)
    O = (p @ V[sel]) / denom
    lse = (m + np.log(denom))[:, 0]
    return O, lse


# ----------------------------------------------------------------------------------------
# IndexShare group  [SHARE]
# ----------------------------------------------------------------------------------------


def select_row(q_idx_t, w_t, k_dec, pos: int, k: int, pool: int = 1, k_pool_dec=None):
    """Indexer + top-k for one query row: returns (idx [k_tokens] int32, scores f32).

    pool == 1: scores over keys, top-k keys.  pool > 1 (IndexPool): scores over pooled
    keys (k_pool_dec, decoded pooled e4m3), top-k blocks, expanded to pool*k tokens."""
    if pool == 1:
        sc = index_scores_row(q_idx_t, w_t, k_dec, pos)
        n_valid = min(k_dec.shape[0], pos + 1)
        return topk_row(sc, n_valid, k), sc
    sc = index_scores_row(q_idx_t, w_t, k_pool_dec, pos, pool=pool)
    n_valid = min(k_pool_dec.shape[0], pos // pool + 1)
    blocks = topk_row(sc, n_valid, k)
    return expand_blocks(blocks, pos, pool), sc


def group_forward_row(q_idx_t, w_t, k_dec, pos: int, k: int, layers: List[dict],
                      sm_scale: float, pool: int = 1, k_pool_dec=None):
    """One query row of an IndexShare group: one indexer + one top-k, reused by every
    layer's attention.  layers: [{"q": [Hq,d_qk], "K": [S,d_qk], "V": [S,d_v]}] float64.
    Returns (idx, [(O, lse) per layer])."""
    idx, _ = select_row(q_idx_t, w_t, k_dec, pos, k, pool, k_pool_dec)
    outs = [sparse_attn_row(L["q"], L["K"], L["V"], idx, sm_scale) for L in layers]
    return idx, outs


def per_layer_forward_row(indexer_inputs: List[tuple], pos: int, k: int, layers: List[dict],
                          sm_scale: float):
    """The comparator without IndexShare: every layer runs its own indexer and top-k.
    indexer_inputs: per layer (q_idx_t, w_t, k_dec)."""
    res = []
    for (qi, wt, kd), L in zip(indexer_inputs, layers):
        idx, _ = select_row(qi, wt, kd, pos, k)
        res.append((idx, sparse_attn_row(L["q"], L["K"], L["V"], idx, sm_scale)))
    return res


# ----------------------------------------------------------------------------------------
# Acceptance rules (the comparison side of parity: pure functions of oracle values)
# ----------------------------------------------------------------------------------------


def topk_set_ok(gpu_idx: np.ndarray, scores_ref: np.ndarray, n_valid: int, k: int,
                pos: int, rel_band: float = 1e-3, pool: int = 1):
    """Check one GPU top-k row against oracle scores.

    Pass iff: the valid entries are distinct, within [0, n_valid), and there are exactly
    k_eff of them; every key whose oracle score exceeds the oracle's k-th score tau by more
    than rel_band*|tau| is selected; no key scoring below tau - rel_band*|tau| is selected.
    (Keys inside the band around tau are free.)  Returns (ok, message)."""
    sel = np.asarray([i for i in gpu_idx if i >= 0], dtype=np.int64)
    keff = min(k, n_valid)
    if sel.size != keff:
        return False, f"selected {sel.size}, expected {keff}"
    if np.unique(sel).size != sel.size:
        return False, "duplicate indices"
    if sel.size and (sel.min() < 0 or sel.max() >= n_valid):
        return False, f"index out of [0,{n_valid})"
    if keff == n_valid:
        return True, "all valid keys"
    s = np.asarray(scores_ref[:n_valid], dtype=np.float64)
    tau = np.sort(s)[::-1][keff - 1]
    band = rel_band * abs(tau)
    must = np.nonzero(s > tau + band)[0]
    if not np.isin(must, sel).all():
        return False, f"missed {np.setdiff1d(must, sel)[:8]} above tau={tau}"
    if (s[sel] < tau - band).any():
        bad = sel[s[sel] < tau - band]
        return False, f"selected {bad[:8]} below tau={tau}"
    return True, "ok"


def score_close(gpu: np.ndarray, ref: np.ndarray, dense_mag: np.ndarray, rel: float = 1e-3,
                floor_rel: float = 1e-5):
    """Indexer tolerance: |gpu - ref| <= rel*|ref|, or, where cancellation of signed head
    weights makes ref near zero, |gpu - ref| <= floor_rel * D with
    D = sum_j |w_j| * max(0, q_j . k) (the score's absolute magnitude).
    Returns (ok_mask, n_floor_used)."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    d = np.abs(g - r)
    rel_ok = d <= rel * np.abs(r)
    floor_ok = d <= floor_rel * np.asarray(dense_mag, dtype=np.float64)
    return rel_ok | floor_ok, int(np.count_nonzero(~rel_ok & floor_ok))


def score_magnitude_row(q_t: np.ndarray, w_t: np.ndarray, k: np.ndarray, pos: int, pool: int = 1):
    """D[s] = sum_j |w_t[j]| * max(0, q_t[j] . k[s]) for valid keys (the tolerance scale)."""
    S = k.shape[0]
    n_valid = min(S, pos // pool + 1)
    out = np.zeros(S)
    logits = k[:n_valid] @ q_t.T
    out[:n_valid] = np.maximum(logits, 0.0) @ np.abs(np.asarray(w_t, dtype=np.float64))
    return out
