"""The comparison side of the GPU parity tests, on the CPU: the helpers in tests/parity.py
accept outputs that meet the stated tolerances and reject each kind of violation (a score off
by more than 1e-3 relative, an unmasked tail, ids out of order or misplaced padding, a wrong
key or a missing token of a pooled block, attention beyond 2e-2 max or 1e-2 mean, an lse off by
more than 1e-3).  Stand-in "GPU" outputs are the oracle's own values, rounded the way the
device stores them, then perturbed."""
import numpy as np
import torch

import oracle as O
from tests import parity as P

rng = np.random.default_rng(99)


def codes(shape, scale=0.5):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
    return x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def bf16_round(x):
    return torch.from_numpy(np.asarray(x, np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def _indexer_case(S=300, pos=200, H=4, D=64):
    q, k = codes((H, D)), codes((S, D))
    w = rng.standard_normal(H).astype(np.float32)
    kdec = O.e4m3_to_f64(k)
    ref = O.index_scores_row(O.e4m3_to_f64(q), w, kdec, pos)
    return q, w, kdec, ref


def test_scores_helper():
    q, w, kdec, ref = _indexer_case()
    n_valid = 201
    gpu = ref.copy()                              # -inf up to the tile end (256) and beyond
    assert P.check_scores_row(gpu, q, w, kdec, 200)[1] is None
    bad = gpu.copy(); j = int(np.argmax(np.abs(ref[:n_valid]))); bad[j] *= np.float32(1 + 2e-3)
    assert P.check_scores_row(bad, q, w, kdec, 200)[1] is not None
    ok = gpu.copy(); ok[j] *= np.float32(1 + 5e-4)
    assert P.check_scores_row(ok, q, w, kdec, 200)[1] is None
    tail = gpu.copy(); tail[230] = 0.0            # inside the diagonal tile: must stay -inf
    assert "masked tail" in P.check_scores_row(tail, q, w, kdec, 200)[1]
    beyond = gpu.copy(); beyond[280] = 0.0        # past the tile that holds the last visible key
    assert P.check_scores_row(beyond, q, w, kdec, 200)[1] is None


def test_scores_helper_floor_for_cancelling_weights():
    # two heads with opposite weights on identical logits: the score is exactly 0, its
    # magnitude is not; an error of 1e-6 of that magnitude is accepted, 1e-4 is not
    D = 64
    qh = codes((1, D)); q = np.concatenate([qh, qh]); w = np.array([1.0, -1.0], np.float32)
    k = codes((40, D)); kdec = O.e4m3_to_f64(k)
    ref = O.index_scores_row(O.e4m3_to_f64(q), w, kdec, 39)
    assert (ref[:40] == 0).all()
    mag = O.score_magnitude_row(O.e4m3_to_f64(q), w, kdec, 39)
    j = int(np.argmax(mag))
    gpu = ref.copy(); gpu[j] = np.float32(1e-6 * mag[j])
    nfloor, msg = P.check_scores_row(gpu, q, w, kdec, 39)
    assert msg is None and nfloor >= 1
    gpu[j] = np.float32(1e-4 * mag[j])
    assert P.check_scores_row(gpu, q, w, kdec, 39)[1] is not None


def test_topk_helper():
    q, w, kdec, ref = _indexer_case()
    k = 16
    sel = np.sort(O.topk_row(ref, 201, k))
    assert P.check_topk_row(sel, q, w, kdec, 200, k) is None
    assert P.check_topk_row(sel[::-1].copy(), q, w, kdec, 200, k) == "ids not strictly ascending"
    order = np.argsort(-ref[:201].astype(np.float64), kind="stable")
    assert order[100] not in sel
    wrong = np.sort(np.r_[sel[1:], order[100]])    # a mid-ranked key instead of a winner
    assert P.check_topk_row(wrong, q, w, kdec, 200, k) is not None
    short = np.r_[sel[:-1], -1]
    assert P.check_topk_row(short, q, w, kdec, 200, k) is not None
    pad_mid = np.r_[sel[:5], -1, sel[5:-1]]
    assert P.check_topk_row(pad_mid, q, w, kdec, 200, k) is not None


def test_topk_helper_pooled():
    kp = codes((64, 64)); q = codes((4, 64)); w = np.abs(rng.standard_normal(4)).astype(np.float32)
    kpd = O.e4m3_to_f64(kp)
    pos, k = 201, 8                                # block 50 (tokens 200..203) is partly visible
    blocks = O.topk_row(O.index_scores_row(O.e4m3_to_f64(q), w, kpd, pos, 4), pos // 4 + 1, k)
    toks = O.expand_blocks(blocks, pos, 4)
    gpu = np.full(k * 4, -1, np.int64)
    v = np.sort(toks[toks >= 0]); gpu[: v.size] = v
    assert P.check_topk_row(gpu, q, w, None, pos, k, pool=4, kpool_dec=kpd) is None
    drop = gpu.copy(); drop[0] = -1; drop = np.r_[drop[1:], -1]   # one token of a block missing
    assert P.check_topk_row(drop, q, w, None, pos, k, pool=4, kpool_dec=kpd) is not None


def _attn_case(Hq=8, D=32, Dv=16, S=50):
    q = rng.standard_normal((Hq, D)); K = rng.standard_normal((S, D)); V = K[:, :Dv]
    idx = rng.permutation(S)[:20]
    o, lse = O.sparse_attn_row(q, K, V, idx, 0.2)
    return q, K, V, idx, o, lse


def test_attention_helper():
    q, K, V, idx, o, lse = _attn_case()
    g = bf16_round(o)
    assert P.check_attn_row(g, q, K, V, idx, 0.2, lse) is None
    one = g.copy(); one[3, 5] += 0.03                                  # max bound 2e-2
    assert "attention" in P.check_attn_row(one, q, K, V, idx, 0.2, lse)
    all_ = g + 0.011                                                   # mean bound 1e-2
    assert "attention" in P.check_attn_row(all_, q, K, V, idx, 0.2, lse)
    off = lse + 2e-3 * max(1.0, np.abs(lse).max())
    assert "lse" in P.check_attn_row(g, q, K, V, idx, 0.2, off)
    inf = lse.copy(); inf[0] = -np.inf
    assert P.check_attn_row(g, q, K, V, idx, 0.2, inf) == "lse finiteness differs"


def test_attention_helper_scaled_outputs():
    # outputs of size ~5: an error of 0.05 is 1e-2 of the scale (accepted only when the bounds
    # are read in units of max(1, max|O|))
    q, K, V, idx, o, lse = _attn_case()
    V5 = V * 5.0
    o5, l5 = O.sparse_attn_row(q, K, V5, idx, 0.2)
    g = o5.copy(); g[0, 0] += 0.05 * np.sign(g[0, 0])
    assert P.check_attn_row(g, q, K, V5, idx, 0.2, l5) is not None
    assert P.check_attn_row(g, q, K, V5, idx, 0.2, l5, out_scaled=True) is None
