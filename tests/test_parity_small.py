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
        kpool_dec = P.Decoded(dsa.dsa_index_pool(ind["k_idx"]))
    idx_h = P.to_np(idx)
    nfloor_total = 0
    by_b = {}
    for (b, t) in rows:
        by_b.setdefault(b, []).append(t)
    for b, ts in by_b.items():
        kd = kdec[b]
        kpd = kpool_dec[b] if kpool_dec is not None else None
        if check_scores:
            keys = ind["k_idx"] if wl.pool == 1 else dsa.dsa_index_pool(ind["k_idx"])
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


def test_indexpool_every_code_bit_exact():
    """Pooling of keys drawn uniformly over all 254 finite e4m3 codes (so sums cancel,
    saturate and land on ties of every binade): the pooled codes equal the oracle's bit for
    bit."""
    g = torch.Generator(device="cpu").manual_seed(17)
    codes = torch.randint(0, 254, (2, 1 << 17, 128), generator=g, dtype=torch.int32)
    codes = torch.where(codes >= 0x7F, codes + 1, codes).to(torch.uint8)   # skip 0x7F (NaN); 0xFF is never drawn
    kp = dsa.dsa_index_pool(codes.to(DEV))
    assert np.array_equal(P.to_np(kp), O.index_pool(codes.numpy()))


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
