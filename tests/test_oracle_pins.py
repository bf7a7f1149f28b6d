"""Pins of the CPU oracle against things other than itself (CPU only).

Every check below gets its expected value from outside the oracle: a library routine
(torch's fp8/bf16 casts, torch matmul, torch scaled_dot_product_attention), a closed form,
a hand-worked example under tests/golden/, brute force in pure Python on tiny inputs, or an
invariant of the definition.  test_oracle_mutants.py plants mistakes in the oracle and
checks that these pins catch them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# ---------------------------------------------------------------- helpers (independent)

def torch_e4m3(codes):
    """e4m3 decode by torch's own float8_e4m3fn type (a library routine)."""
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def rand_codes(shape, scale=0.5):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * scale)
    return x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def brute_scores(q_codes, w, k_codes, pos, pool=1):
    """Pure-Python loops over heads and dims, torch decode; float64 then one f32 rounding."""
    qf, kf = torch_e4m3(q_codes), torch_e4m3(k_codes)
    H, D = qf.shape
    out = []
    for s in range(kf.shape[0]):
        if pool * s > pos:
            out.append(float("-inf"))
            continue
        tot = 0.0
        for j in range(H):
            dot = 0.0
            for d in range(D):
                dot += qf[j, d] * kf[s, d]
            tot += float(w[j]) * (dot if dot > 0 else 0.0)
        out.append(float(np.float32(tot)))
    return np.array(out, dtype=np.float32)


# ---------------------------------------------------------------- number formats

def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    a, b = O.e4m3_to_f64(codes), torch_e4m3(codes)
    assert np.array_equal(np.isnan(a), np.isnan(b))
    m = ~np.isnan(a)
    assert np.array_equal(a[m], b[m])
    assert np.array_equal(np.signbit(a[m]), np.signbit(b[m]))


def test_e4m3_decode_format_values():
    # OCP FP8 E4M3: bias 7, subnormal step 2^-9, max finite 448, S.1111.111 = NaN
    v = O.e4m3_to_f64(np.array([0x38, 0x7E, 0x01, 0x08, 0x07, 0xFE, 0x44, 0x30], dtype=np.uint8))
    assert list(v) == [1.0, 448.0, 2.0 ** -9, 2.0 ** -6, 7 * 2.0 ** -9, -448.0, 3.0, 0.5]
    assert math.isnan(O.e4m3_to_f64(np.array([0x7F], dtype=np.uint8))[0])


def test_e4m3_encode_matches_torch_in_range():
    x = (rng.standard_normal(200_000) * np.exp(rng.standard_normal(200_000) * 3)).astype(np.float32)
    x = np.clip(x, -447.0, 447.0)
    # exact ties between neighbours in several binades, both parities
    ties = np.array([(2 * m + 1) * 2.0 ** (e - 4) for e in range(-6, 8) for m in range(8, 16)], dtype=np.float32)
    sub_ties = np.array([(2 * m + 1) * 2.0 ** -10 for m in range(0, 8)], dtype=np.float32)
    x = np.concatenate([x, ties, -ties, sub_ties, -sub_ties, [0.0, -0.0]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.f32_to_e4m3(x), ref)


def test_e4m3_encode_every_rounding_class():
    """Every decision the encoder makes, enumerated: for each fp32 exponent from far below the
    e4m3 subnormals to beyond saturation, every value of the 5 leading mantissa bits (what an
    e4m3 normal keeps plus the round bit; more for subnormals, covered by the exponent sweep),
    a zero, a 1-ulp and a full sticky tail, both signs.  Compared with torch's RNE cast."""
    bits = []
    for e in range(127 - 20, 127 + 10):          # 2^-20 .. 2^9
        for head in range(32):
            for tail in (0, 1, (1 << 18) - 1):
                bits.append((e << 23) | (head << 18) | tail)
    u = np.array(bits, dtype=np.uint32)
    x = np.concatenate([u, u | np.uint32(0x80000000)]).view(np.float32)
    x = x[np.abs(x) < 464.0]                     # beyond 464 both sides saturate (pinned below)
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert x.size > 5_000
    assert np.array_equal(O.f32_to_e4m3(x), ref)


def test_e4m3_encode_saturates():
    x = np.array([448.0, 455.9, 464.0, 479.0, 1e9, np.inf, -600.0, -np.inf], dtype=np.float32)
    assert list(O.f32_to_e4m3(x)) == [0x7E] * 6 + [0xFE] * 2
    assert O.f32_to_e4m3(np.array([np.nan], dtype=np.float32))[0] == 0x7F


def test_bf16_decode_matches_torch():
    u = rng.integers(0, 1 << 16, 50_000, dtype=np.uint16)
    t = torch.from_numpy(u.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    a = O.bf16_to_f64(u)
    m = ~np.isnan(t)
    assert np.array_equal(a[m], t[m]) and np.isnan(a[~m]).all()


# ---------------------------------------------------------------- indexer

def test_indexer_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "indexer_hand.json")))
    q = np.array(g["q_idx_codes"], dtype=np.uint8)[None]          # [1,T,H,d]
    w = np.array(g["w"], dtype=np.float32)[None]
    k = np.array(g["k_idx_codes"], dtype=np.uint8)[None]
    T = q.shape[1]
    ctx = [g["positions"][-1] + 1]
    assert [ctx[0] - T + t for t in range(T)] == g["positions"]
    res = O.index_scores(q, w, k, ctx)
    for t in range(T):
        exp = np.array([float(v) for v in g["expected"][t]], dtype=np.float32)
        assert np.array_equal(res[(0, t)], exp)
        n_valid = g["positions"][t] + 1
        assert list(O.topk_row(res[(0, t)], n_valid, 2)) == g["expected_top2"][t]


def test_indexer_brute_force_tiny():
    for trial in range(4):
        H, D, S = [(3, 5, 9), (4, 64, 13), (1, 8, 5), (6, 3, 11)][trial]
        q = rand_codes((H, D)); k = rand_codes((S, D)); w = rng.standard_normal(H).astype(np.float32)
        for pos in [0, S // 2, S - 1]:
            a = O.index_scores_row(O.e4m3_to_f64(q), w, O.e4m3_to_f64(k), pos)
            b = brute_scores(q, w, k, pos)
            fin = np.isfinite(b)
            assert np.array_equal(np.isfinite(a), fin)
            np.testing.assert_allclose(a[fin], b[fin], rtol=2e-7, atol=1e-30)


def test_indexer_single_head_unit_weight_is_relu_dot():
    q = rand_codes((1, 128)); k = rand_codes((300, 128))
    ref = torch.relu(torch.from_numpy(torch_e4m3(k)) @ torch.from_numpy(torch_e4m3(q)).T)[:, 0].numpy()
    a = O.index_scores_row(O.e4m3_to_f64(q), np.ones(1, np.float32), O.e4m3_to_f64(k), 299)
    np.testing.assert_allclose(a, ref.astype(np.float32), rtol=1e-7)
    assert (a >= 0).all() and (a == 0).any()   # the ReLU clips some keys to exactly 0


def test_indexer_power_of_two_weight_scaling_is_exact():
    q = rand_codes((4, 64)); k = rand_codes((50, 64)); w = rng.standard_normal(4).astype(np.float32)
    a = O.index_scores_row(O.e4m3_to_f64(q), w, O.e4m3_to_f64(k), 49)
    b = O.index_scores_row(O.e4m3_to_f64(q), w * np.float32(8.0), O.e4m3_to_f64(k), 49)
    assert np.array_equal(b, a * np.float32(8.0))


def test_indexer_causal_rule_includes_self():
    q = rand_codes((2, 16)); k = rand_codes((10, 16)); w = np.abs(rng.standard_normal(2)).astype(np.float32)
    for pos in range(10):
        a = O.index_scores_row(O.e4m3_to_f64(q), w, O.e4m3_to_f64(k), pos)
        assert np.isfinite(a[: pos + 1]).all() and np.isneginf(a[pos + 1:]).all()


def test_indexer_positions_follow_context_end():
    # T queries at the end of a context of length ctx: query t sits at ctx - T + t
    q = rand_codes((1, 3, 2, 8)); k = rand_codes((1, 7, 8)); w = rng.standard_normal((1, 3, 2)).astype(np.float32)
    res = O.index_scores(q, w, k, [7])
    for t in range(3):
        assert np.count_nonzero(np.isfinite(res[(0, t)])) == 7 - 3 + t + 1


# ---------------------------------------------------------------- top-k

def test_topk_brute_force_sort():
    for _ in range(30):
        n = int(rng.integers(1, 80)); k = int(rng.integers(1, 40))
        s = rng.integers(-5, 6, size=n).astype(np.float32)      # many ties on purpose
        n_valid = int(rng.integers(1, n + 1))
        ref = sorted(range(n_valid), key=lambda i: (-float(s[i]), i))[:k]
        got = O.topk_row(s, n_valid, k)
        assert list(got[: len(ref)]) == ref and (got[len(ref):] == -1).all()


def test_topk_all_keys_when_k_exceeds_valid():
    s = rng.standard_normal(10).astype(np.float32)
    got = O.topk_row(s, 6, 8)
    assert sorted(got[:6]) == list(range(6)) and list(got[6:]) == [-1, -1]


def test_topk_acceptance_rule():
    s = rng.standard_normal(500).astype(np.float32)
    idx = O.topk_row(s, 500, 50)
    assert O.topk_set_ok(idx, s, 500, 50, 499)[0]
    bad = idx.copy(); bad[0] = int(np.argsort(s)[0])             # the worst key instead of the best
    assert not O.topk_set_ok(bad, s, 500, 50, 499)[0]
    dup = idx.copy(); dup[1] = dup[0]
    assert not O.topk_set_ok(dup, s, 500, 50, 499)[0]
    # inside the tie band anything goes: swap the k-th for the (k+1)-th when they are close
    s2 = s.copy(); order = np.argsort(-s2); s2[order[50]] = s2[order[49]] * (1 - 1e-4 * np.sign(s2[order[49]]))
    idx2 = O.topk_row(s2, 500, 50); sw = idx2.copy(); sw[list(idx2).index(order[49])] = order[50]
    assert O.topk_set_ok(sw, s2, 500, 50, 499)[0]
    # missing a key far above the k-th score is wrong even when its replacement sits inside
    # the band (nothing selected lies below tau - band, so only the "missed" rule rejects it)
    miss = idx2.copy(); miss[list(idx2).index(order[0])] = order[50]
    assert not O.topk_set_ok(miss, s2, 500, 50, 499)[0]
    assert not O.topk_set_ok(np.where(np.arange(50) == 49, -1, idx), s, 500, 50, 499)[0]   # one short
    assert not O.topk_set_ok(np.r_[idx[:49], 500], s, 500, 50, 499)[0]                    # beyond n_valid
    # fewer valid keys than k: every valid key, nothing else
    assert O.topk_set_ok(np.r_[np.arange(7), [-1] * 3], s, 7, 10, 6)[0]
    assert not O.topk_set_ok(np.r_[np.arange(6), [-1] * 4], s, 7, 10, 6)[0]


def test_score_tolerance_rule_closed_form():
    # relative rule: |gpu - ref| <= 1e-3 |ref|; floor rule: |gpu - ref| <= 1e-5 * D where D is
    # the score's absolute magnitude sum_j |w_j| relu(q_j . k)
    ref = np.array([1000.0, 1000.0, 1.0, 0.0, 0.0, -50.0])
    gpu = np.array([1000.9, 1001.1, 1.01, 0.009, 0.011, -50.04])
    mag = np.array([1000.0, 1000.0, 1.0, 1000.0, 1000.0, 60.0])
    ok, nfloor = O.score_close(gpu, ref, mag, rel=1e-3, floor_rel=1e-5)
    assert list(ok) == [True, False, False, True, False, True] and nfloor == 1


def test_score_magnitude_closed_form():
    # two heads, w = (1, -2): D = |1| relu(q0.k) + |-2| relu(q1.k)
    q = np.array([[1.0, 0.0], [0.0, 1.0]]); w = np.array([1.0, -2.0], np.float32)
    k = np.array([[3.0, 2.0], [-1.0, 5.0], [2.0, -4.0], [9.0, 9.0]])
    assert list(O.score_magnitude_row(q, w, k, pos=2)) == [3 + 2 * 2, 0 + 2 * 5, 2 + 0, 0.0]


# ---------------------------------------------------------------- IndexPool

def test_pool_of_identical_keys_is_identity():
    k = rand_codes((5, 32))
    rep = np.repeat(k, 4, axis=0)
    assert np.array_equal(O.index_pool(rep), k)


def test_pool_brute_force_and_library_requantisation():
    k = rand_codes((2, 64, 16))
    got = O.index_pool(k)
    kt = torch.from_numpy(k).view(torch.float8_e4m3fn).to(torch.float32)
    for b in range(2):
        for g in range(16):
            for d in range(16):
                a, bb, c, e = [kt[b, 4 * g + r, d] for r in range(4)]
                m = ((a + bb) + (c + e)) * 0.25                    # torch fp32 scalar ops
                ref = m.reshape(1).to(torch.float8_e4m3fn).view(torch.uint8).item()
                assert got[b, g, d] == ref


def test_pool_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "indexpool_hand.json")))
    k = np.array(g["groups_codes"], dtype=np.uint8).reshape(-1, 1)     # [4 * groups, d = 1]
    assert list(O.index_pool(k)[:, 0]) == g["expected_codes"]


def test_pool_mean_is_exact_then_one_rounding():
    """Four e4m3 values are integer multiples of 2^-9 below 2^11 in magnitude, so their fp32
    sum and its quarter are exact: the pooled code is the exact rational mean rounded once by
    torch's e4m3 cast, whatever order the four keys come in."""
    from fractions import Fraction
    k = rand_codes((32, 24), scale=40.0)                       # wide range: subnormals to 448
    got = O.index_pool(k)
    kv = torch_e4m3(k)
    for g in range(8):
        for d in range(24):
            mean = sum(Fraction(float(kv[4 * g + r, d])) for r in range(4)) / 4
            ref = torch.tensor([float(mean)], dtype=torch.float64).to(torch.float32).to(torch.float8_e4m3fn)
            assert float(mean) == float(np.float32(float(mean)))     # exact in fp32
            assert got[g, d] == ref.view(torch.uint8).item()
    perm = k.reshape(8, 4, 24)[:, [2, 0, 3, 1]].reshape(32, 24)
    assert np.array_equal(O.index_pool(perm), got)


@pytest.mark.parametrize("P", [2, 8])
def test_pool_factors_2_and_8_identity_brute_force_and_exact_mean(P):
    """Pool factors 2 and 8 (the pages' factor is 4): identical keys pool to themselves; each
    pooled code equals torch fp32 scalar arithmetic (pairwise sum, times 1/P) cast by torch to
    e4m3; and, since P e4m3 values (integer multiples of 2^-9 below 2^9 in magnitude) sum
    exactly in fp32 for P <= 8, the code is the exact rational mean rounded once, whatever
    order the keys come in."""
    from fractions import Fraction
    k = rand_codes((5, 32))
    assert np.array_equal(O.index_pool(np.repeat(k, P, axis=0), pool=P), k)
    k = rand_codes((P * 6, 12), scale=40.0)
    got = O.index_pool(k, pool=P)
    assert got.shape == (6, 12)
    kt = torch.from_numpy(k).view(torch.float8_e4m3fn).to(torch.float32)
    for g in range(6):
        for d in range(12):
            vals = [kt[P * g + r, d] for r in range(P)]
            while len(vals) > 1:
                vals = [vals[2 * i] + vals[2 * i + 1] for i in range(len(vals) // 2)]
            ref = (vals[0] * (1.0 / P)).reshape(1).to(torch.float8_e4m3fn).view(torch.uint8).item()
            assert got[g, d] == ref
            mean = sum(Fraction(float(kt[P * g + r, d])) for r in range(P)) / P
            assert float(mean) == float(np.float32(float(mean)))          # exact in fp32
            ex = torch.tensor([float(mean)], dtype=torch.float64).to(torch.float32).to(torch.float8_e4m3fn)
            assert got[g, d] == ex.view(torch.uint8).item()
    rng = np.random.default_rng(P)
    perm = np.stack([rng.permutation(P) for _ in range(6)])
    shuffled = np.concatenate([k[P * g + perm[g]] for g in range(6)])
    assert np.array_equal(O.index_pool(shuffled, pool=P), got)
    with pytest.raises(ValueError):
        O.index_pool(rand_codes((12, 4)), pool=3)


@pytest.mark.parametrize("P", [2, 8])
def test_pool_factor_validity_and_expansion(P):
    # block b is a candidate iff P*b <= pos; it expands to tokens P*b .. P*b+P-1, those beyond
    # pos becoming -1
    D = 16
    q = np.zeros((1, D)); q[0, 0] = 1.0; w = np.ones(1, np.float32)
    kp = np.zeros((6, D)); kp[:, 0] = [1.0, 2.0, 3.0, 100.0, 0.5, 0.25]     # block 3 scores highest
    pos = 3 * P                                                              # block 3's first token
    idx, sc = O.select_row(q, w, None, pos, 2, pool=P, k_pool_dec=kp)
    assert list(idx[:P]) == [3 * P] + [-1] * (P - 1)
    assert list(idx[P:2 * P]) == list(range(2 * P, 3 * P))                   # runner-up block 2, whole
    assert np.isneginf(sc[4:]).all() and np.isfinite(sc[:4]).all()
    idx, _ = O.select_row(q, w, None, pos - 1, 2, pool=P, k_pool_dec=kp)     # block 3 not yet visible
    assert list(idx[:P]) == list(range(2 * P, 3 * P))


def test_select_row_pool_last_block_visible_from_its_first_token():
    # block b is a candidate from position 4b on (its first token visible), never before; the
    # expanded ids keep only tokens <= pos
    D = 16
    q = np.zeros((1, D)); q[0, 0] = 1.0; w = np.ones(1, np.float32)
    kp = np.zeros((6, D)); kp[:, 0] = [1.0, 2.0, 3.0, 100.0, 0.5, 0.25]     # block 3 scores highest
    for pos, want in [(12, [12, -1, -1, -1]), (13, [12, 13, -1, -1]), (15, [12, 13, 14, 15]), (11, [8, 9, 10, 11])]:
        idx, sc = O.select_row(q, w, None, pos, 2, pool=4, k_pool_dec=kp)
        assert list(idx[:4]) == want, (pos, list(idx))
        assert np.isneginf(sc[pos // 4 + 1:]).all()


def test_pool_validity_and_expansion():
    # block b is valid iff 4b <= pos; tokens beyond pos in the last block become -1
    kp = rand_codes((6, 8)); q = rand_codes((2, 8)); w = np.ones(2, np.float32)
    sc = O.index_scores_row(O.e4m3_to_f64(q), w, O.e4m3_to_f64(kp), pos=9, pool=4)
    assert np.isfinite(sc[:3]).all() and np.isneginf(sc[3:]).all()
    assert list(O.expand_blocks(np.array([2, 0, -1]), 9, 4)) == [8, 9, -1, -1, 0, 1, 2, 3, -1, -1, -1, -1]


# ---------------------------------------------------------------- attention

def _attn_inputs(Hq, D, Dv, S, latent):
    q = rng.standard_normal((Hq, D)); K = rng.standard_normal((S, D))
    V = K[:, :Dv] if latent else rng.standard_normal((S, Dv))
    return q, K, V


def test_attention_dense_when_all_keys_selected_matches_torch_sdpa():
    # k >= context: sparse attention over every causal key is dense causal attention
    T, Hq, D, Dv = 12, 4, 16, 8
    q = rng.standard_normal((T, Hq, D)); K = rng.standard_normal((T, D)); V = rng.standard_normal((T, Dv))
    scale = 1 / math.sqrt(D)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).permute(1, 0, 2)[None], torch.from_numpy(K)[None, None].expand(1, Hq, T, D),
        torch.from_numpy(V)[None, None].expand(1, Hq, T, Dv), is_causal=True, scale=scale)[0].permute(1, 0, 2).numpy()
    for t in range(T):
        sc = rng.standard_normal(T).astype(np.float32)
        idx = O.topk_row(sc, t + 1, 64)                        # k=64 > t+1: all causal keys
        o, lse = O.sparse_attn_row(q[t], K, V, idx, scale)
        np.testing.assert_allclose(o, ref[t], rtol=1e-10, atol=1e-12)
        lref = torch.logsumexp(torch.from_numpy(q[t] @ K[: t + 1].T * scale), dim=1).numpy()
        np.testing.assert_allclose(lse, lref, rtol=1e-12)


def test_attention_single_key_returns_v():
    q, K, V = _attn_inputs(8, 32, 16, 20, latent=False)
    o, lse = O.sparse_attn_row(q, K, V, np.array([-1, 7, -1]), 0.3)
    assert np.array_equal(o, np.repeat(V[7:8], 8, axis=0))
    np.testing.assert_allclose(lse, 0.3 * q @ K[7], rtol=1e-14)


def test_attention_zero_query_is_mean_of_v_and_duplicates_count():
    _, K, V = _attn_inputs(4, 16, 8, 30, latent=True)
    q = np.zeros((4, 16))
    idx = np.array([3, 5, 5, 11])
    o, _ = O.sparse_attn_row(q, K, V, idx, 1.0)
    np.testing.assert_allclose(o, np.repeat(((V[3] + 2 * V[5] + V[11]) / 4)[None], 4, axis=0), rtol=1e-14)


def test_attention_hand_worked_example():
    from fractions import Fraction
    g = json.load(open(os.path.join(GOLDEN, "attention_hand.json")))
    K, V, q = (np.array(g[n], dtype=np.float64) for n in ("K", "V", "q"))
    for r, idx in enumerate(g["idx"]):
        o, lse = O.sparse_attn_row(q, K, V, np.array(idx), math.log(2.0))
        exp_o = np.array([[float(Fraction(x)) for x in h] for h in g["expected_O"][r]])
        np.testing.assert_allclose(o, exp_o, rtol=1e-13, atol=1e-13)
        for h, z in enumerate(g["expected_lse_of"][r]):
            if z == 0:
                assert lse[h] == -np.inf
            else:
                assert abs(lse[h] - math.log(z)) < 1e-13


def test_attention_huge_logits_pick_the_argmax_key():
    # logit gaps of ~1000 (exp(-1000) is 0 in float64): the output is exactly V of the
    # best key and lse is exactly the best logit
    K = np.zeros((5, 4)); K[:, 0] = [1.0, 3.0, -2.0, 2.0, 0.0]
    V = rng.standard_normal((5, 3))
    q = np.array([[1000.0, 0, 0, 0], [-1000.0, 0, 0, 0]])
    o, lse = O.sparse_attn_row(q, K, V, np.array([0, 1, 2, 3, 4]), 1.0)
    assert np.array_equal(o[0], V[1]) and np.array_equal(o[1], V[2])
    assert list(lse) == [3000.0, 2000.0]


def test_attention_brute_force_and_permutation():
    q, K, V = _attn_inputs(3, 6, 4, 15, latent=True)
    idx = rng.permutation(15)[:9]
    o, lse = O.sparse_attn_row(q, K, V, idx, 0.7)
    for h in range(3):
        logits = [0.7 * sum(q[h, d] * K[i, d] for d in range(6)) for i in idx]
        ex = [math.exp(l) for l in logits]
        z = sum(ex)
        for c in range(4):
            assert abs(o[h, c] - sum(e * V[i, c] for e, i in zip(ex, idx)) / z) < 1e-12
        assert abs(lse[h] - math.log(z)) < 1e-12
    o2, _ = O.sparse_attn_row(q, K, V, idx[::-1], 0.7)
    np.testing.assert_allclose(o, o2, rtol=1e-13)


# ---------------------------------------------------------------- IndexShare group

def test_indexshare_group_reuses_one_selection():
    S, H, D, Hq, Dq, Dv, k = 40, 2, 8, 4, 12, 6, 7
    qi = O.e4m3_to_f64(rand_codes((H, D))); kd = O.e4m3_to_f64(rand_codes((S, D)))
    w = rng.standard_normal(H).astype(np.float32)
    layers = [dict(zip("qKV", _attn_inputs(Hq, Dq, Dv, S, latent=True))) for _ in range(4)]
    idx, outs = O.group_forward_row(qi, w, kd, 33, k, layers, 0.25)
    sel_only, _ = O.select_row(qi, w, kd, 33, k)
    assert np.array_equal(idx, sel_only)
    for L, (o, lse) in zip(layers, outs):
        o2, l2 = O.sparse_attn_row(L["q"], L["K"], L["V"], idx, 0.25)
        assert np.array_equal(o, o2) and np.array_equal(lse, l2)
    # the comparator with the same indexer inputs at every layer selects the same keys
    per = O.per_layer_forward_row([(qi, w, kd)] * 4, 33, k, layers, 0.25)
    assert all(np.array_equal(p[0], idx) for p in per)


def test_per_layer_comparator_selects_with_each_layers_own_indexer():
    # layer l's keys are built so that key 5l+3 dominates its own indexer: each layer's
    # selection must contain its own planted key, and the layers' selections differ
    S, H, D, Hq, Dq, Dv, k = 30, 1, 4, 2, 6, 3, 3
    q = np.zeros((H, D)); q[0, 0] = 1.0; w = np.ones(H, np.float32)
    ins = []
    for l in range(4):
        kd = np.zeros((S, D)); kd[:, 0] = rng.uniform(-1, 1, S); kd[5 * l + 3, 0] = 50.0
        ins.append((q, w, kd))
    layers = [dict(zip("qKV", _attn_inputs(Hq, Dq, Dv, S, latent=False))) for _ in range(4)]
    per = O.per_layer_forward_row(ins, 29, k, layers, 0.5)
    for l, (idx, (o, lse)) in enumerate(per):
        assert 5 * l + 3 in set(idx.tolist())
        o2, l2 = O.sparse_attn_row(layers[l]["q"], layers[l]["K"], layers[l]["V"], idx, 0.5)
        assert np.array_equal(o, o2) and np.array_equal(lse, l2)
    assert len({tuple(p[0].tolist()) for p in per}) == 4
