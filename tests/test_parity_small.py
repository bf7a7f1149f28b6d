"""GPU parity at sizes the oracle finishes in seconds: the whole tiny workload row by row,
ragged and varlen batches, chunked prefill, IndexPool, decode-shaped split-key attention,
MLA shapes, and the degenerate cases (k >= context, all scores tied, single visible key).
Every call goes through the C ABI of libdsa_b200.so."""
import numpy as np
import pytest
import torch

import oracle as O
import indexed_sparse_attention_fp8_b200 as dsa
from indexed_sparse_attention_fp8_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def _no_device_timeouts():
    yield
    assert dsa.dsa_device_status() == 0, "a kernel gave up a bounded wait"


def _inputs(wl, layers=4):
    ind = W.make_indexer_inputs(wl, device=DEV)
    lays = [W.make_attn_inputs(wl, l, device=DEV) for l in range(layers)]
    return ind, lays


def _layer_dicts(lays, want_v):
    return [{"q": L["q"], "kv": L["kv"], "v": L["v"] if want_v else None} for L in lays]


def _run_group(wl, ind, lays, ctx_len=None, t_chunk=None, want_lse=True):
    ctx = ind["ctx_len"] if ctx_len is None else ctx_len
    return dsa.dsa_group_forward(ind["q_idx"], ind["w"], ind["k_idx"], ctx, wl.topk,
                                 _layer_dicts(lays, not wl.kv_latent), wl.sm_scale, wl.d_v, pool=wl.pool,
                                 t_chunk=t_chunk, want_lse=want_lse)


def _check_rows(wl, ind, lays, idx, outs, rows, ctx_len=None, check_scores=True):
    """Oracle comparison of the listed (b, t) rows: scores (through dsa_index_scores),
    top-k sets and every layer's attention (and lse)."""
    ctx = ind["ctx_len"] if ctx_len is None else ctx_len
    ctx_h = P.to_np(ctx)
    q_idx, w = ind["q_idx"], ind["w"]
    kdec = P.Decoded(ind["k_idx"])
    kpool_dec = None
    if wl.pool > 1:
        kpool_dec = P.Decoded(dsa.dsa_index_pool(ind["k_idx"], pool=wl.pool))
    idx_h = P.to_np(idx)
    nfloor_total = 0
    by_b = {}
    for (b, t) in rows:
        by_b.setdefault(b, []).append(t)
    for b, ts in by_b.items():
        kd = kdec[b]
        kpd = kpool_dec[b] if kpool_dec is not None else None
        if check_scores:
            keys = ind["k_idx"] if wl.pool == 1 else dsa.dsa_index_pool(ind["k_idx"], pool=wl.pool)
            sc = dsa.dsa_index_scores(q_idx, w, keys, ctx, pool=wl.pool)
            sc_h = P.to_np(sc[b])
        lay_np = [(P.bf16_np(L["kv"][b]), None if wl.kv_latent else P.bf16_np(L["v"][b])) for L in lays]
        for t in ts:
            pos = int(ctx_h[b]) - wl.T + t
            qc, wr = P.to_np(q_idx[b, t]), P.to_np(w[b, t])
            if check_scores:
                nf, msg = P.check_scores_row(sc_h[t], qc, wr, kd if wl.pool == 1 else kpd, pos, wl.pool)
                nfloor_total += nf
                assert msg is None, f"row {(b, t)}: {msg}"
            msg = P.check_topk_row(idx_h[b, t], qc, wr, kd, pos, wl.topk, wl.pool, kpd)
            assert msg is None, f"row {(b, t)}: {msg}"
            for li, (L, (o, lse)) in enumerate(zip(lays, outs)):
                K, Vsep = lay_np[li]
                V = K[:, : wl.d_v] if wl.kv_latent else Vsep
                qrow = P.bf16_np(L["q"][b, t])
                msg = P.check_attn_row(P.bf16_np(o[b, t]), qrow, K, V, idx_h[b, t], wl.sm_scale,
                                       None if lse is None else P.to_np(lse[b, t]).astype(np.float64))
                assert msg is None, f"row {(b, t)} layer {li}: {msg}"
    return nfloor_total


def test_tiny_workload_every_row():
    wl = W.WORKLOADS["tiny"]
    ind, lays = _inputs(wl)
    idx, outs = _run_group(wl, ind, lays)
    torch.cuda.synchronize()
    nfloor = _check_rows(wl, ind, lays, idx, outs, [(0, t) for t in range(wl.T)])
    # only near-zero scores may use the magnitude floor
    assert nfloor < 0.2 * wl.T * wl.T / 2


def test_indexshare_group_equals_separate_calls_bitwise():
    wl = W.WORKLOADS["tiny"].replace(T=700, ctx=700)
    ind, lays = _inputs(wl)
    idx, outs = _run_group(wl, ind, lays)
    sc = dsa.dsa_index_scores(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"])
    idx2 = dsa.dsa_topk(sc, ind["ctx_len"], wl.T, wl.S, wl.topk)
    assert torch.equal(idx, idx2)
    for L, (o, lse) in zip(lays, outs):
        o2, l2 = dsa.dsa_sparse_attn(L["q"], L["kv"], idx, wl.sm_scale, wl.d_v, v=L["v"], want_lse=True)
        assert torch.equal(o, o2) and torch.equal(lse, l2)


def test_query_chunking_does_not_change_the_selection():
    wl = W.WORKLOADS["tiny"].replace(T=900, ctx=1500)
    ind, lays = _inputs(wl, layers=1)
    idx_a, outs_a = _run_group(wl, ind, lays)
    idx_b, outs_b = _run_group(wl, ind, lays, t_chunk=97)     # ragged chunks of 97 queries
    assert torch.equal(idx_a, idx_b)
    assert torch.equal(outs_a[0][0], outs_b[0][0])


def test_chunked_prefill_and_varlen_batch():
    wl = W.WORKLOADS["tiny"].replace(B=3, T=300, ctx=1000, topk=128)
    ind, lays = _inputs(wl, layers=2)
    ctx = torch.tensor([1000, 517, 300], dtype=torch.int32, device=DEV)
    idx, outs = _run_group(wl, ind, lays, ctx_len=ctx)
    rows = [(b, t) for b in range(3) for t in (0, 1, 127, 128, 129, 200, 299)]
    _check_rows(wl, ind, lays, idx, outs, rows, ctx_len=ctx)


def test_k_exceeds_context_is_dense_causal():
    wl = W.WORKLOADS["tiny"].replace(T=100, ctx=100, topk=256)
    ind, lays = _inputs(wl, layers=1)
    idx, outs = _run_group(wl, ind, lays)
    idx_h = P.to_np(idx)
    for t in range(100):
        assert list(idx_h[0, t, : t + 1]) == list(range(t + 1)) and (idx_h[0, t, t + 1:] == -1).all()
    _check_rows(wl, ind, lays, idx, outs, [(0, t) for t in range(0, 100, 7)])


def test_all_tied_scores_select_lowest_indices():
    wl = W.WORKLOADS["tiny"].replace(T=600, ctx=600, topk=64)
    ind, lays = _inputs(wl, layers=1)
    ind["w"].zero_()                                    # every score is exactly 0
    idx, outs = _run_group(wl, ind, lays)
    idx_h = P.to_np(idx)
    for t in range(64, 600, 37):
        assert list(idx_h[0, t]) == list(range(64))


def test_indexpool_small():
    wl = W.WORKLOADS["tiny"].replace(T=512, ctx=2048, topk=64, pool=4)
    ind, lays = _inputs(wl, layers=2)
    kp = dsa.dsa_index_pool(ind["k_idx"])
    assert np.array_equal(P.to_np(kp), O.index_pool(P.to_np(ind["k_idx"])))     # bit-exact
    idx, outs = _run_group(wl, ind, lays)
    _check_rows(wl, ind, lays, idx, outs, [(0, t) for t in (0, 1, 2, 3, 100, 255, 256, 511)])


@pytest.mark.parametrize("factor", [2, 4, 8])
def test_indexpool_every_code_bit_exact(factor):
    """Pooling of keys drawn uniformly over all 254 finite e4m3 codes (so sums cancel,
    saturate and land on ties of every binade): the pooled codes equal the oracle's bit for
    bit, for the pages' factor 4 and for 2 and 8."""
    g = torch.Generator(device="cpu").manual_seed(17)
    codes = torch.randint(0, 254, (2, 1 << 17, 128), generator=g, dtype=torch.int32)
    codes = torch.where(codes >= 0x7F, codes + 1, codes).to(torch.uint8)   # skip 0x7F (NaN); 0xFF is never drawn
    kp = dsa.dsa_index_pool(codes.to(DEV), pool=factor)
    assert np.array_equal(P.to_np(kp), O.index_pool(codes.numpy(), pool=factor))


def test_mla_shapes_small_prefill():
    wl = W.WORKLOADS["prefill32k"].replace(T=2500, ctx=3000)
    ind, lays = _inputs(wl, layers=2)
    idx, outs = _run_group(wl, ind, lays, t_chunk=1024)
    rows = [(0, t) for t in (0, 1, 63, 64, 1023, 1024, 1547, 1548, 2047, 2048, 2499)]
    _check_rows(wl, ind, lays, idx, outs, rows)


def test_mla_decode_shaped_split_keys():
    wl = W.WORKLOADS["decode256k"].replace(B=5, ctx=6000)
    ind, lays = _inputs(wl, layers=2)
    assert dsa.dsa_sparse_attn_workspace_size(wl.B, 1, 128, 512, 2048) > 0   # split-key path
    ctx = torch.tensor([6000, 2049, 2048, 777, 1], dtype=torch.int32, device=DEV)
    idx, outs = _run_group(wl, ind, lays, ctx_len=ctx)
    _check_rows(wl, ind, lays, idx, outs, [(b, 0) for b in range(5)], ctx_len=ctx)


def test_attention_skips_negative_ids_anywhere():
    wl = W.WORKLOADS["tiny"].replace(T=64, ctx=64, topk=40)
    ind, lays = _inputs(wl, layers=1)
    g = torch.Generator(device="cpu").manual_seed(5)
    idx = torch.randint(0, 64, (1, 64, 40), generator=g).to(torch.int32)
    for t in range(64):
        idx[0, t][idx[0, t] > t] = -1                  # holes in the middle of rows
    idx[0, 3] = -1                                     # a row with nothing selected
    idx = idx.to(DEV)
    L = lays[0]
    out, lse = dsa.dsa_sparse_attn(L["q"], L["kv"], idx, wl.sm_scale, wl.d_v, v=L["v"], want_lse=True)
    K, V = P.bf16_np(L["kv"][0]), P.bf16_np(L["v"][0])
    idx_h = P.to_np(idx)
    for t in range(64):
        msg = P.check_attn_row(P.bf16_np(out[0, t]), P.bf16_np(L["q"][0, t]), K, V, idx_h[0, t], wl.sm_scale,
                               P.to_np(lse[0, t]).astype(np.float64))
        assert msg is None, f"row {t}: {msg}"
    assert (P.bf16_np(out[0, 3]) == 0).all() and np.isneginf(P.to_np(lse[0, 3])).all()


@pytest.mark.parametrize("q_scale", [6.0, 12.0, 20.0])
def test_mla_peaked_softmax(q_scale):
    """Logits 6-20x the unit-variance workload's (a peaked softmax: a few keys carry most of
    the weight, and the running max moves by more than the lazy-rescale threshold inside a
    row, so O is rescaled in TMEM mid-row).  Outputs reach |O| ~ 5, so the bf16 bounds are
    taken in units of max(1, max|O|); the lse bound is unchanged."""
    wl = W.WORKLOADS["prefill32k"].replace(T=256, ctx=4096)
    L = W.make_attn_inputs(wl, 0, device=DEV)
    q = (L["q"].float() * q_scale).to(torch.bfloat16)
    g = torch.Generator(device="cpu").manual_seed(11)
    idx = torch.stack([torch.randperm(4096 - 256, generator=g)[: wl.topk] for _ in range(wl.T)]).to(torch.int32)
    idx = idx.view(1, wl.T, wl.topk).to(DEV)
    out, lse = dsa.dsa_sparse_attn(q, L["kv"], idx, wl.sm_scale, wl.d_v, want_lse=True)
    K = P.bf16_np(L["kv"][0])
    idx_h = P.to_np(idx)
    for t in (0, 1, 77, 128, 255):
        msg = P.check_attn_row(P.bf16_np(out[0, t]), P.bf16_np(q[0, t]), K, K[:, : wl.d_v], idx_h[0, t], wl.sm_scale,
                               P.to_np(lse[0, t]).astype(np.float64), out_scaled=True)
        assert msg is None, f"row {t}: {msg}"


@pytest.mark.parametrize("reps", [1, 8])
def test_topk_long_rows_exact_with_ties(reps):
    """Long rows given as fp32 scores directly: the selected set must equal the oracle's
    exactly, with exact ties resolved to the lowest indices (an all-tied row, and a row of
    small integers with thousands of keys tied at the pivot), ids ascending and -1 padding; a
    row with fewer visible keys than k selects them all.  The pivot bucket is copied to shared
    memory when it fits (the every-7th and integer rows) and not for the all-tied row; five and
    forty rows."""
    S, k, T = 20000, 2048, 1
    B = 5 * reps
    g = torch.Generator(device="cpu").manual_seed(3)
    sc = torch.randn(B, T, S, generator=g)
    ctx = torch.tensor([S, S, 15000, 1500, S] * reps, dtype=torch.int32)
    for r in range(reps):
        sc[5 * r] = 0.0                                                     # all tied: ids 0..2047
        sc[5 * r + 1, 0] = torch.randint(0, 50, (S,), generator=g).float()  # heavy ties at the pivot
        sc[5 * r + 4] = 0.0
        sc[5 * r + 4, 0, ::7] = 1.0                                         # winners: every 7th id up to 14329
    idx = dsa.dsa_topk(sc.to(DEV), ctx.to(DEV), T, S, k)
    for b in range(B):
        n_valid = min(S, int(ctx[b]))
        ref = O.topk_row(sc[b, 0].numpy(), n_valid, k)
        got = P.to_np(idx[b, 0])
        valid = got[got >= 0]
        assert np.array_equal(np.sort(valid), np.sort(ref[ref >= 0])), f"row {b}"
        assert (np.diff(valid) > 0).all() and (got[valid.size:] == -1).all(), f"row {b}"


def _select_rows(B, S, g):
    """Rows of every kind the selection treats differently (fp32 scores given directly)."""
    sc = torch.randn(B, 1, S, generator=g)
    kinds = []
    for b in range(B):
        kind = b % 7
        if kind == 1:    # small integers: thousands of keys tied at the pivot
            sc[b, 0] = torch.randint(0, 50, (S,), generator=g).float()
        elif kind == 2:  # all tied: the lowest ids win
            sc[b, 0] = 0.5
        elif kind == 3:  # sparse winners: every 7th key, far fewer than the zeros around them
            sc[b, 0] = 0.0
            sc[b, 0, ::7] = 1.0
        elif kind == 4:  # ascending: every winner at the row's end (one CTA's part of a cluster)
            sc[b, 0] = torch.arange(S, dtype=torch.float32) * 1e-3
        elif kind == 5:  # the sampled blocks mislead the threshold: the first few sampled blocks
            # (16 keys every sstride) hold the row's only high scores, enough of them to set the
            # threshold above every other key, yet fewer than k keys in all
            sstride = 16 * -(-S // (16 * 512))
            nblk = -(-S // sstride)
            ns = (nblk - 1) * 16 + min(16, S - (nblk - 1) * sstride)
            r = -(-(3 * 2048 // 2) * ns // S)
            for q in range(-(-r // 16) + 1):
                sc[b, 0, q * sstride: q * sstride + 16] = 50.0
        kinds.append(kind)
    return sc, kinds


@pytest.mark.parametrize("B,S", [(300, 20000), (6, 20000), (40, 40000), (12, 65536), (4, 131072), (2, 4500)])
def test_topk_selection_paths_exact(B, S):
    """The selection's every path against the oracle's sort, set for set: one CTA per row (300
    rows), clusters of 2, 4 and 8 CTAs per row (6, 40, 12 and 4 rows), rows that fit the
    candidate buffer whole (S = 4500), rows where the sampled threshold holds (normal, integer
    ties, ascending: every winner in the last CTA's part) and rows where it cannot (all tied and
    sparse winners: too many candidates; a misleading sample: too few), which take the full-row
    path; one row of each batch sees fewer keys than k."""
    k, T = 2048, 1
    g = torch.Generator(device="cpu").manual_seed(11 + B)
    sc, kinds = _select_rows(B, S, g)
    ctx = torch.full((B,), S, dtype=torch.int32)
    ctx[B - 1] = min(S, 1500)
    if B > 2:
        ctx[B - 2] = S - 777
    idx = dsa.dsa_topk(sc.to(DEV), ctx.to(DEV), T, S, k)
    got_all = P.to_np(idx)
    for b in range(B):
        n_valid = min(S, int(ctx[b]))
        ref = O.topk_row(sc[b, 0].numpy(), n_valid, k)
        got = got_all[b, 0]
        valid = got[got >= 0]
        assert np.array_equal(np.sort(valid), np.sort(ref[ref >= 0])), f"row {b} (kind {kinds[b]})"
        assert (np.diff(valid) > 0).all() and (got[valid.size:] == -1).all(), f"row {b}"


@pytest.mark.parametrize("name", ["tiny", "prefill32k"])
def test_attention_ids_beyond_the_cache_are_skipped_and_flagged(name):
    """Selected ids at or beyond the cache length S_kv are skipped on the device like a -1 and
    reported by dsa_device_status() as DSA_ERR_INDEX_RANGE.  The cache passed is a view of the
    first S_kv rows of a larger allocation, so the rows the bad ids name are real memory and a
    missing check would show up as wrong outputs, not as a read outside any allocation."""
    wl = W.WORKLOADS[name].replace(T=48, ctx=300)
    S = wl.ctx
    big = W.make_attn_inputs(wl.replace(ctx=S + 128), 0, device=DEV)
    q = big["q"][:, :wl.T].contiguous()
    kv = big["kv"][:, :S]                                   # S_kv = S rows; 128 more rows follow in memory
    v = None if big["v"] is None else big["v"][:, :S]
    g = torch.Generator(device="cpu").manual_seed(23)
    k = min(wl.topk, 128)
    idx = torch.randint(0, S, (1, wl.T, k), generator=g).to(torch.int32)
    bad = torch.rand((1, wl.T, k), generator=g) < 0.1
    idx[bad] = (S + torch.randint(0, 128, (int(bad.sum()),), generator=g)).to(torch.int32)
    idx[0, 5] = S + 3                                       # a row where every id is out of range
    assert dsa.dsa_device_status() == 0
    out, lse = dsa.dsa_sparse_attn(q, kv, idx.to(DEV), wl.sm_scale, wl.d_v, v=v, want_lse=True)
    assert dsa.dsa_device_status() == 7                     # DSA_ERR_INDEX_RANGE, then cleared
    assert dsa.dsa_device_status() == 0
    K = P.bf16_np(kv[0])
    V = K[:, : wl.d_v] if wl.kv_latent else P.bf16_np(v[0])
    skipped = idx[0].numpy().copy()
    skipped[skipped >= S] = -1                              # what the oracle must see
    for t in (0, 1, 5, 17, wl.T - 1):
        msg = P.check_attn_row(P.bf16_np(out[0, t]), P.bf16_np(q[0, t]), K, V, skipped[t], wl.sm_scale,
                               P.to_np(lse[0, t]).astype(np.float64))
        assert msg is None, f"row {t}: {msg}"
    assert (P.bf16_np(out[0, 5]) == 0).all() and np.isneginf(P.to_np(lse[0, 5])).all()


@pytest.mark.parametrize("factor,topk", [(2, 96), (8, 24)])
def test_indexpool_factors_2_and_8(factor, topk):
    """IndexPool over 2 and 8 keys: pooled keys bit-exact against the oracle, then the pooled
    indexer, block top-k and expansion to P tokens per block, and the attention over them."""
    wl = W.WORKLOADS["tiny"].replace(T=512, ctx=2048, topk=topk, pool=factor)
    ind, lays = _inputs(wl, layers=2)
    kp = dsa.dsa_index_pool(ind["k_idx"], pool=factor)
    kp_h = P.to_np(kp)
    assert kp_h.shape[1] == 2048 // factor
    assert np.array_equal(kp_h, O.index_pool(P.to_np(ind["k_idx"]), pool=factor))
    idx, outs = _run_group(wl, ind, lays)
    _check_rows(wl, ind, lays, idx, outs, [(0, t) for t in (0, 1, factor - 1, factor, 100, 255, 256, 511)])


@pytest.mark.parametrize("factor", [2, 4, 8])
def test_pooled_cache_tail_refresh_equals_full_pool(factor):
    """A pooled cache kept by dsa_index_pool_tail: after keys are appended (ragged contexts, one
    and several new rows, blocks left partly filled and then completed), the refreshed cache is
    the full pool of the current keys bit for bit, and the oracle's; blocks away from the new
    rows are not written."""
    g = torch.Generator(device="cpu").manual_seed(23 + factor)
    B, S, D = 3, 4096, 128
    codes = torch.randint(0, 254, (B, S, D), generator=g, dtype=torch.int32)
    k = torch.where(codes >= 0x7F, codes + 1, codes).to(torch.uint8).to(DEV)
    ctx = torch.tensor([1000, 2049, 37], dtype=torch.int32, device=DEV)
    kp = dsa.dsa_index_pool(k, pool=factor)
    for T in (1, 1, 3, factor, 5 * factor + 1, 1):
        ctx += T
        for b in range(B):   # the append: new rows ctx-T .. ctx-1
            c = int(ctx[b])
            k[b, c - T:c] = torch.randint(0, 127, (T, D), generator=g, dtype=torch.int32).to(torch.uint8).to(DEV)
        before = kp.clone()
        dsa.dsa_index_pool_tail(k, ctx, T, kp, pool=factor)
        full = dsa.dsa_index_pool(k, pool=factor)
        assert torch.equal(kp, full)
        for b in range(B):   # untouched outside the new rows' blocks
            c = int(ctx[b])
            lo, hi = (c - T) // factor, (c - 1) // factor + 1
            assert torch.equal(kp[b, :lo], before[b, :lo]) and torch.equal(kp[b, hi:], before[b, hi:])
    assert dsa.dsa_device_status() == 0
    assert np.array_equal(P.to_np(kp), O.index_pool(P.to_np(k), pool=factor))


def test_group_with_kept_pooled_cache_equals_pooling_in_the_call():
    """The group call reading a caller-kept pooled cache gives the ids and outputs of the call
    that pools the keys itself, bit for bit (decode shape, ragged contexts)."""
    wl = W.WORKLOADS["decode256k_pool"].replace(B=3, ctx=9000)
    ind, lays = _inputs(wl, layers=2)
    ctx = torch.tensor([9000, 4097, 2051], dtype=torch.int32, device=DEV)
    layers = lambda: [{"q": L["q"], "kv": L["kv"], "v": L["v"]} for L in lays]   # noqa: E731
    idx0, outs0 = dsa.dsa_group_forward(ind["q_idx"], ind["w"], ind["k_idx"], ctx, wl.topk, layers(), wl.sm_scale,
                                        wl.d_v, pool=wl.pool, want_lse=True)
    kp = dsa.dsa_index_pool(ind["k_idx"], pool=wl.pool)
    idx1, outs1 = dsa.dsa_group_forward(ind["q_idx"], ind["w"], ind["k_idx"], ctx, wl.topk, layers(), wl.sm_scale,
                                        wl.d_v, pool=wl.pool, want_lse=True, k_pooled=kp)
    assert torch.equal(idx0, idx1)
    for (o0, l0), (o1, l1) in zip(outs0, outs1):
        assert torch.equal(o0, o1) and torch.equal(l0, l1)


def test_decode_step_replays_as_a_cuda_graph():
    """A decode step (pooled-cache refresh, indexer, top-k, split-key attention and its combine
    for two layers) captured once as a CUDA graph and replayed gives the eager step's ids,
    outputs and lse bit for bit: no call synchronises the host or allocates while capturing."""
    wl = W.WORKLOADS["decode256k_pool"].replace(B=3, ctx=9000)
    ind, lays = _inputs(wl, layers=2)
    ctx = torch.tensor([9000, 4097, 2051], dtype=torch.int32, device=DEV)
    kp = dsa.dsa_index_pool(ind["k_idx"], pool=wl.pool)
    layers = [{"q": L["q"], "kv": L["kv"], "v": L["v"]} for L in lays]
    g = dsa.Group(ind["q_idx"], ind["w"], ind["k_idx"], ctx, wl.topk, layers, wl.sm_scale, wl.d_v, pool=wl.pool,
                  want_lse=True, k_pooled=kp)
    ws = torch.empty(g.workspace_size(wl.T), dtype=torch.uint8, device=DEV)

    def step(stream):
        dsa.dsa_index_pool_tail(ind["k_idx"], ctx, wl.T, kp, pool=wl.pool, stream=stream)
        return g.forward(ws, stream)

    idx, outs = step(torch.cuda.current_stream())
    eager = (idx.clone(), [(o.clone(), l.clone()) for o, l in outs])
    for o, l in outs:
        o.zero_()
        l.zero_()
    idx.fill_(-7)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream())
    graph.replay()
    torch.cuda.synchronize()
    assert dsa.dsa_device_status() == 0
    assert torch.equal(idx, eager[0])
    for (o, l), (oe, le) in zip(outs, eager[1]):
        assert torch.equal(o, oe) and torch.equal(l, le)


def test_pooled_decode_small():
    """The decode-shaped pooled path (one query per sequence, QB=1 indexer over pooled keys,
    top-512 blocks, split-key MLA attention), at a cache size the oracle checks in seconds."""
    wl = W.WORKLOADS["decode256k_pool"].replace(B=3, ctx=9000)
    ind, lays = _inputs(wl, layers=2)
    ctx = torch.tensor([9000, 4097, 2051], dtype=torch.int32, device=DEV)
    idx, outs = _run_group(wl, ind, lays, ctx_len=ctx)
    _check_rows(wl, ind, lays, idx, outs, [(b, 0) for b in range(3)], ctx_len=ctx)


def _run_box(wl, ind, lays, box):
    """One shard box (b0, b1, t0, t1) as its own group call: rows t0..t1-1 of sequences
    b0..b1-1, with ctx_len moved to the chunk's end so every row keeps its position."""
    b0, b1, t0, t1 = box
    sl = lambda x: x[b0:b1, t0:t1].contiguous()      # noqa: E731
    ctx = ind["ctx_len"][b0:b1] - (wl.T - t1)
    layers = [{"q": sl(L["q"]), "kv": L["kv"][b0:b1], "v": None if L["v"] is None else L["v"][b0:b1]} for L in lays]
    return dsa.dsa_group_forward(sl(ind["q_idx"]), sl(ind["w"]), ind["k_idx"][b0:b1], ctx, wl.topk, layers,
                                 wl.sm_scale, wl.d_v, pool=wl.pool, want_lse=True)


@pytest.mark.parametrize("name,over", [("tiny", {}), ("decode256k", {"B": 5, "ctx": 3000})])
def test_sharded_plan_reproduces_the_single_call_bitwise(name, over):
    """The 2-rank sharding plan (zig-zag row chunks for prefill, batch slices for decode), its
    boxes run one after another on this GPU, gives the single call's ids, outputs and lse bit
    for bit (both sides use the same key split here, so even the fp32 sums agree)."""
    from indexed_sparse_attention_fp8_b200 import shard
    wl = W.WORKLOADS[name].replace(**over)
    ind, lays = _inputs(wl, layers=2)
    idx, outs = _run_group(wl, ind, lays)
    seen = 0
    for rank in range(2):
        for box in shard.plan(wl, 2, rank):
            b0, b1, t0, t1 = box
            idx_c, outs_c = _run_box(wl, ind, lays, box)
            assert torch.equal(idx_c, idx[b0:b1, t0:t1]), box
            for (o, l), (oc, lc) in zip(outs, outs_c):
                assert torch.equal(oc, o[b0:b1, t0:t1]) and torch.equal(lc, l[b0:b1, t0:t1]), box
            seen += (b1 - b0) * (t1 - t0)
    assert seen == wl.B * wl.T


def _to_pages(x, page_size, table, num_pages):
    """A per-sequence cache [B, S, W] copied into a page pool [num_pages, page_size, W] along
    the block table [B, pages_per_seq]; pages not in the table hold noise."""
    B, S, W = x.shape
    if x.dtype == torch.uint8:                              # e4m3 codes: any byte but NaN (0x7F, 0xFF)
        pool = torch.randint(0, 0x7F, (num_pages, page_size, W), dtype=torch.uint8, device=x.device)
    else:
        pool = torch.randn((num_pages, page_size, W), device=x.device).to(x.dtype)
    for b in range(B):
        for j in range(table.shape[1]):
            rows = x[b, j * page_size:(j + 1) * page_size]
            pool[int(table[b, j]), : rows.shape[0]] = rows
    return pool


def _page_table(B, S, page_size, spare, seed):
    pps = (S + page_size - 1) // page_size
    g = torch.Generator(device="cpu").manual_seed(seed)
    perm = torch.randperm(B * pps + spare, generator=g)[: B * pps].to(torch.int32)
    return perm.view(B, pps).to(DEV), B * pps + spare


@pytest.mark.parametrize("name,over,page_size", [
    ("tiny", {"B": 2, "T": 300, "ctx": 1000}, 128),
    ("decode256k", {"B": 3, "ctx": 3000}, 256),
    ("decode256k_pool", {"B": 2, "ctx": 5000}, 128),
])
def test_paged_caches_reproduce_the_contiguous_call_bitwise(name, over, page_size):
    """Paged KV (the serving form of decode and chunked prefill): the indexer keys and every
    layer's latent (or K and V) rows live in shuffled pages of shared pools, addressed through
    a block table; the group call gives the contiguous call's ids, outputs and lse bit for bit
    (the indexer, the pool kernel and both attention kernels read through the table)."""
    wl = W.WORKLOADS[name].replace(**over)
    ind, lays = _inputs(wl, layers=2)
    ctx = torch.tensor([wl.ctx - 37 * b for b in range(wl.B)], dtype=torch.int32, device=DEV)
    idx, outs = _run_group(wl, ind, lays, ctx_len=ctx)
    table, num_pages = _page_table(wl.B, wl.S, page_size, spare=3, seed=7)
    pg = dsa.paging(table, page_size, num_pages)
    kp = _to_pages(ind["k_idx"], page_size, table.cpu(), num_pages)
    layers = [{"q": L["q"], "kv": _to_pages(L["kv"], page_size, table.cpu(), num_pages),
               "v": None if L["v"] is None else _to_pages(L["v"], page_size, table.cpu(), num_pages)} for L in lays]
    idx_p, outs_p = dsa.dsa_group_forward(ind["q_idx"], ind["w"], kp, ctx, wl.topk, layers, wl.sm_scale, wl.d_v,
                                          pool=wl.pool, want_lse=True, paging=pg)
    assert dsa.dsa_device_status() == 0
    assert torch.equal(idx_p, idx)
    for (o, l), (op, lp) in zip(outs, outs_p):
        assert torch.equal(op, o) and torch.equal(lp, l)


def test_paged_bad_page_ids_are_skipped_and_flagged():
    """A block-table entry outside [0, num_pages) is never followed: the attention skips the
    rows on that page (like -1 ids), the indexer reads zeros for them, and the status reports
    DSA_ERR_INDEX_RANGE.  The bad entries here point just past the pool and at -1."""
    wl = W.WORKLOADS["decode256k"].replace(B=2, ctx=1024)
    ind, lays = _inputs(wl, layers=1)
    table, num_pages = _page_table(wl.B, wl.S, 256, spare=0, seed=9)
    bad = table.clone()
    bad[0, 1] = num_pages                                   # rows 256..511 of sequence 0
    bad[1, 3] = -1                                          # rows 768..1023 of sequence 1
    pg = dsa.paging(bad, 256, num_pages)
    kv_pool = _to_pages(lays[0]["kv"], 256, table.cpu(), num_pages)
    g = torch.Generator(device="cpu").manual_seed(4)
    sel = torch.randint(0, 1024, (wl.B, 1, 300), generator=g).to(torch.int32).to(DEV)
    out, lse = dsa.dsa_sparse_attn(lays[0]["q"], kv_pool, sel, wl.sm_scale, wl.d_v, want_lse=True, paging=pg)
    assert dsa.dsa_device_status() == 7
    K = [P.bf16_np(lays[0]["kv"][b]) for b in range(wl.B)]
    sel_h = P.to_np(sel).copy()
    sel_h[0][(sel_h[0] >= 256) & (sel_h[0] < 512)] = -1     # what the oracle must see
    sel_h[1][sel_h[1] >= 768] = -1
    for b in range(wl.B):
        msg = P.check_attn_row(P.bf16_np(out[b, 0]), P.bf16_np(lays[0]["q"][b, 0]), K[b], K[b][:, : wl.d_v],
                               sel_h[b, 0], wl.sm_scale, P.to_np(lse[b, 0]).astype(np.float64))
        assert msg is None, f"sequence {b}: {msg}"
    kp = _to_pages(ind["k_idx"], 256, table.cpu(), num_pages)
    sc = dsa.dsa_index_scores(ind["q_idx"], ind["w"], kp, ind["ctx_len"], paging=pg)
    assert dsa.dsa_device_status() == 7
    assert (P.to_np(sc[0, 0, 256:512]) == 0).all()          # zero keys score exactly 0
    ref = dsa.dsa_index_scores(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"])
    assert torch.equal(sc[0, 0, :256], ref[0, 0, :256]) and torch.equal(sc[1, 0, :768], ref[1, 0, :768])


def _unfused_ids(wl, ind, keys, t_begin=0, t_count=None):
    tc = wl.T - t_begin if t_count is None else t_count
    sc = dsa.dsa_index_scores(ind["q_idx"], ind["w"], keys, ind["ctx_len"], pool=wl.pool, t_begin=t_begin,
                              t_count=tc)
    return dsa.dsa_topk(sc, ind["ctx_len"], wl.T, keys.shape[1], wl.topk, pool=wl.pool, t_begin=t_begin)


@pytest.mark.parametrize("name,over", [
    ("tiny", {"T": 4096, "ctx": 16384}),                       # rows with n <= k, n <= 8192 and n > 8192
    ("prefill32k", {"T": 1024, "ctx": 20480}),                 # the 64-head, 4-query-block indexer
    ("decode256k", {"B": 4, "ctx": 40960}),                    # one query per sequence
    ("chunk1m_pool", {"T": 256, "ctx": 65536}),                # pooled blocks, top-512
])
def test_fused_selection_equals_full_score_rows_bitwise(name, over):
    """The fused selection (sampled threshold, candidate append, top-k on the candidates) gives
    exactly the ids of full score rows + the row top-k, in every row regime: all visible keys
    kept (n <= k), threshold -inf (n <= 8192 candidates), sampled threshold; and the oracle
    accepts sampled rows of each regime."""
    wl = W.WORKLOADS[name].replace(**over)
    ind, lays = _inputs(wl, layers=1)
    keys = ind["k_idx"] if wl.pool == 1 else dsa.dsa_index_pool(ind["k_idx"], pool=wl.pool)
    assert keys.shape[1] % 16 == 0                          # the fused path applies
    got = dsa.dsa_index_select(ind["q_idx"], ind["w"], keys, ind["ctx_len"], wl.topk, pool=wl.pool)
    ref = _unfused_ids(wl, ind, keys)
    assert torch.equal(got, ref)
    # through the group call too (fused and default selection), with a workspace small enough for
    # several query chunks
    for fused in (True, False):
        idx, outs = dsa.dsa_group_forward(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], wl.topk,
                                          [{"q": lays[0]["q"], "kv": lays[0]["kv"], "v": lays[0]["v"]}], wl.sm_scale,
                                          wl.d_v, pool=wl.pool, t_chunk=max(1, wl.T // 3), fused_select=fused)
        assert torch.equal(idx, ref)
    kdec = P.Decoded(ind["k_idx"])
    kpd = P.Decoded(keys) if wl.pool > 1 else None
    idx_h = P.to_np(idx)
    for b in sorted({0, wl.B - 1}):
        for t in sorted({0, wl.T // 2, wl.T - 1}):
            pos = wl.ctx - wl.T + t
            msg = P.check_topk_row(idx_h[b, t], P.to_np(ind["q_idx"][b, t]), P.to_np(ind["w"][b, t]), kdec[b], pos,
                                   wl.topk, wl.pool, kpd[b] if kpd else None)
            assert msg is None, f"row {(b, t)}: {msg}"


def test_fused_selection_repair_when_the_sample_misleads():
    """Keys at multiples of 16 (exactly the sampled ones) score far above all others, so each
    row's threshold (the r-th largest sample) is met by only r = 32 < k keys and every long row
    is redone by the repair pass;
    an all-tied row overflows the candidate buffer and is redone too.  The ids still equal the
    full-row selection, and the oracle accepts them."""
    wl = W.WORKLOADS["tiny"].replace(T=64, ctx=16384, topk=256)
    ind = W.make_indexer_inputs(wl, device=DEV)
    v = torch.zeros(wl.d_I, device=DEV)
    v[:8] = 2.0
    codes = v.to(torch.float8_e4m3fn).view(torch.uint8)
    ind["q_idx"][:] = codes                                 # every head of every query looks along v
    ind["w"].abs_()                                         # positive head weights
    kf = ind["k_idx"][0, ::16].view(torch.float8_e4m3fn).float()
    kf[:, :8] += 4.0                                        # the sampled keys align with v (distinct scores)
    ind["k_idx"][0, ::16] = kf.to(torch.float8_e4m3fn).view(torch.uint8)
    ind["w"][0, 10] = 0.0                                   # row 10: every score is 0 (all tied)
    got = dsa.dsa_index_select(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], wl.topk)
    ref = _unfused_ids(wl, ind, ind["k_idx"])
    assert torch.equal(got, ref)
    assert list(P.to_np(got[0, 10])) == list(range(256))   # all tied: the lowest ids
    kdec = P.Decoded(ind["k_idx"])
    for t in (0, 10, 63):
        msg = P.check_topk_row(P.to_np(got[0, t]), P.to_np(ind["q_idx"][0, t]), P.to_np(ind["w"][0, t]), kdec[0],
                               wl.ctx - wl.T + t, wl.topk)
        assert msg is None, f"row {t}: {msg}"
