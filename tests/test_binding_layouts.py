"""The Python binding's marshalling checks, on CPU tensors: a tensor whose dtype, shape or
strides differ from the layout the C ABI assumes is rejected with a ValueError naming it,
before any pointer is taken; a well-formed call gets as far as the device check (the library
has no CPU path)."""
import pytest
import torch

import indexed_sparse_attention_fp8_b200 as dsa
from indexed_sparse_attention_fp8_b200 import build as dsa_build

B, T, S, H, D = 2, 8, 64, 4, 64
HQ, DQK, DV, K = 16, 128, 128, 32


@pytest.fixture(scope="module", autouse=True)
def lib():
    dsa_build.build()
    return dsa._lib()


def _indexer():
    return (torch.zeros(B, T, H, D, dtype=torch.uint8), torch.zeros(B, T, H), torch.zeros(B, S, D, dtype=torch.uint8),
            torch.full((B,), S, dtype=torch.int32))


def _attn():
    return (torch.zeros(B, T, HQ, DQK, dtype=torch.bfloat16), torch.zeros(B, S, DQK, dtype=torch.bfloat16),
            torch.zeros(B, S, DV, dtype=torch.bfloat16), torch.zeros(B, T, K, dtype=torch.int32))


def test_well_formed_calls_reach_the_device_check():
    q_idx, w, k_idx, ctx = _indexer()
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.dsa_index_scores(q_idx, w, k_idx, ctx)
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.dsa_topk(torch.zeros(B, T, S), ctx, T, S, K)
    q, kv, v, idx = _attn()
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.dsa_sparse_attn(q, kv, idx, 0.1, DV, v=v, want_lse=True)
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.dsa_index_pool(k_idx)
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.Group(q_idx, w, k_idx, ctx, K, [{"q": q, "kv": kv, "v": v}] * 2, 0.1, DV)


def test_indexer_layouts():
    q_idx, w, k_idx, ctx = _indexer()
    with pytest.raises(ValueError, match="q_idx: dtype"):
        dsa.dsa_index_scores(q_idx.float(), w, k_idx, ctx)
    with pytest.raises(ValueError, match="w: shape"):
        dsa.dsa_index_scores(q_idx, w[:, :, :2], k_idx, ctx)
    with pytest.raises(ValueError, match="k_idx: must be contiguous"):
        dsa.dsa_index_scores(q_idx, w, k_idx.transpose(0, 1).contiguous().transpose(0, 1), ctx)
    with pytest.raises(ValueError, match="ctx_len: dtype"):
        dsa.dsa_index_scores(q_idx, w, k_idx, ctx.long())
    # a scores buffer whose batch stride is not t_count * ld (a slice of a taller buffer)
    tall = torch.empty(B, 2 * T, S)
    with pytest.raises(ValueError, match="scores: strides"):
        dsa.dsa_index_scores(q_idx, w, k_idx, ctx, scores=tall[:, :T])
    with pytest.raises(ValueError, match="scores: strides"):
        dsa.dsa_topk(tall[:, :T], ctx, T, S, K)
    with pytest.raises(ValueError, match="idx: shape"):
        dsa.dsa_topk(torch.zeros(B, T, S), ctx, T, S, K, pool=4, idx=torch.zeros(B, T, K, dtype=torch.int32))
    with pytest.raises(ValueError, match="k_pool: shape"):
        dsa.dsa_index_pool(k_idx, k_pool=torch.zeros(B, S, D, dtype=torch.uint8))


def test_attention_layouts():
    q, kv, v, idx = _attn()
    with pytest.raises(ValueError, match="q: must be contiguous"):
        dsa.dsa_sparse_attn(q.transpose(1, 2).contiguous().transpose(1, 2), kv, idx, 0.1, DV, v=v)
    with pytest.raises(ValueError, match="kv: dtype"):
        dsa.dsa_sparse_attn(q, kv.half(), idx, 0.1, DV, v=v)
    with pytest.raises(ValueError, match="kv: shape"):
        dsa.dsa_sparse_attn(q, kv[:, :, :64], idx, 0.1, DV, v=v)          # narrower than d_qk
    wide = torch.zeros(B, S, DQK + 4, dtype=torch.bfloat16)                 # row stride 132: not 16 B
    with pytest.raises(ValueError, match="kv: shape"):
        dsa.dsa_sparse_attn(q, wide[:, :, :DQK], idx, 0.1, DV, v=v)
    with pytest.raises(ValueError, match="v: strides"):
        dsa.dsa_sparse_attn(q, kv, idx, 0.1, DV, v=v.transpose(1, 2).contiguous().transpose(1, 2))
    with pytest.raises(ValueError, match="idx: dtype"):
        dsa.dsa_sparse_attn(q, kv, idx.long(), 0.1, DV, v=v)
    with pytest.raises(ValueError, match="out: shape"):
        dsa.dsa_sparse_attn(q, kv, idx, 0.1, DV, v=v, out=torch.zeros(B, T, HQ, DQK + 8, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="lse: dtype"):
        dsa.dsa_sparse_attn(q, kv, idx, 0.1, DV, v=v, lse=torch.zeros(B, T, HQ, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="q: dtype"):
        dsa.dsa_sparse_attn_noalloc(q.float(), kv, idx, 0.1, DV, v=v)
    # row-strided caches with 16-byte aligned strides are accepted (a latent row of 576 holding V in its first 512)
    lat = torch.zeros(B, S, 576, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.dsa_sparse_attn(torch.zeros(B, T, 128, 576, dtype=torch.bfloat16), lat, idx, 0.1, 512)


def test_group_layers_share_one_set_of_strides():
    q_idx, w, k_idx, ctx = _indexer()
    q, kv, v, _ = _attn()
    other = torch.zeros(B, S, DQK + 8, dtype=torch.bfloat16)[:, :, :DQK]     # valid, but a different row stride
    with pytest.raises(ValueError, match="layer 1: q shape or kv strides"):
        dsa.Group(q_idx, w, k_idx, ctx, K, [{"q": q, "kv": kv, "v": v}, {"q": q, "kv": other, "v": v}], 0.1, DV)
    with pytest.raises(ValueError, match="layer 1: v presence"):
        dsa.Group(q_idx, w, k_idx, ctx, K, [{"q": q, "kv": kv, "v": v}, {"q": q, "kv": kv, "v": None}], 0.1, DV)
    with pytest.raises(ValueError, match="idx: shape"):
        dsa.Group(q_idx, w, k_idx, ctx, K, [{"q": q, "kv": kv, "v": v}], 0.1, DV, pool=4,
                  idx=torch.zeros(B, T, K, dtype=torch.int32))


@pytest.mark.parametrize("name,over", [
    ("tiny", dict(T=64, ctx=128)),
    ("prefill32k", dict(T=16, ctx=64)),
    ("decode256k", dict(B=3, ctx=64)),
    ("chunk1m_pool", dict(T=16, ctx=256)),
])
def test_workload_tensors_pass_the_layout_checks(name, over):
    """The seeded workload tensors the tests and the bench hand to the binding (built here on
    the CPU at reduced sizes) have the layouts it accepts: every call gets to the device check."""
    from indexed_sparse_attention_fp8_b200 import workloads as W
    wl = W.WORKLOADS[name].replace(**over)
    ind = W.make_indexer_inputs(wl, device="cpu")
    lays = [W.make_attn_inputs(wl, l, device="cpu") for l in range(2)]
    args = [{"q": L["q"], "kv": L["kv"], "v": None if wl.kv_latent else L["v"]} for L in lays]
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.Group(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], wl.topk, args, wl.sm_scale, wl.d_v,
                  pool=wl.pool)
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.dsa_index_scores(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], t_begin=0, t_count=1)
    idx = torch.zeros(wl.B, wl.T, wl.topk * wl.pool, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA device"):
        dsa.dsa_sparse_attn(lays[0]["q"], lays[0]["kv"], idx, wl.sm_scale, wl.d_v, v=args[0]["v"], want_lse=True)
