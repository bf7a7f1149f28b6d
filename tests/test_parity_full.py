"""GPU parity at the full workload sizes, in the launch configuration the benchmark times
(dsa_group_forward over the whole workload with an 8 GiB score workspace), checked on sampled
rows the oracle can compute one by one: indexer scores (via dsa_index_scores on the sampled
rows), the top-k set, and every layer's attention output and log-sum-exp.

Workloads: prefill 32K, prefill 128K (planted signal), decode 32 x 256K, chunked prefill 8192
queries against 1M keys, and its IndexPool variant.  Also the per-layer-indexer comparator."""
import numpy as np
import pytest
import torch

import oracle as O
import indexed_sparse_attention_fp8_b200 as dsa
from indexed_sparse_attention_fp8_b200 import workloads as W
from tests import parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DEV = "cuda"
SCORE_WS_BYTES = 8 << 30


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    assert dsa.dsa_device_status() == 0, "a kernel gave up a bounded wait"
    torch.cuda.empty_cache()


def _t_chunk(wl):
    return max(1, min(wl.T, SCORE_WS_BYTES // (wl.B * ((wl.S // wl.pool + 3) // 4 * 4) * 4)))


def _sample_rows(wl, n_random=3):
    """Query rows checked against the oracle: every sequence of a decode batch (one row each), and
    for prefill the first rows, both sides of the 128-row tile edge, the middle, the last rows and
    a few random ones."""
    rng = np.random.default_rng(wl.seed + 77)
    ts = sorted({0, 1, min(127, wl.T - 1), min(128, wl.T - 1), wl.T // 2, wl.T - 2, wl.T - 1,
                 *[int(x) for x in rng.integers(0, wl.T, n_random)]})
    bs = list(range(wl.B)) if wl.T == 1 else sorted({0, wl.B - 1, int(rng.integers(0, wl.B))})
    return [(b, t) for b in bs for t in ts if 0 <= t < wl.T]


def _check(wl, ind, lays, idx, outs, rows):
    kdec = P.Decoded(ind["k_idx"])
    kp = dsa.dsa_index_pool(ind["k_idx"], pool=wl.pool) if wl.pool > 1 else None
    kpdec = P.Decoded(kp) if kp is not None else None
    idx_h = P.to_np(idx)
    for (b, t) in rows:
        pos = wl.ctx - wl.T + t
        qc, wr = P.to_np(ind["q_idx"][b, t]), P.to_np(ind["w"][b, t])
        keys = ind["k_idx"] if wl.pool == 1 else kp
        # a window of up to 8 queries around t, so the multi-query indexer path is the one checked
        tb = min(t, max(0, wl.T - 8))
        sc = dsa.dsa_index_scores(ind["q_idx"], ind["w"], keys, ind["ctx_len"], pool=wl.pool, t_begin=tb,
                                  t_count=min(8, wl.T - tb))
        _, msg = P.check_scores_row(P.to_np(sc[b, t - tb]), qc, wr, kdec[b] if wl.pool == 1 else kpdec[b], pos,
                                    wl.pool)
        assert msg is None, f"scores {(b, t)}: {msg}"
        msg = P.check_topk_row(idx_h[b, t], qc, wr, kdec[b], pos, wl.topk, wl.pool, kpdec[b] if kpdec else None)
        assert msg is None, f"top-k {(b, t)}: {msg}"
        row = idx_h[b, t]
        sel = row[row >= 0]
        for li, (L, (o, lse)) in enumerate(zip(lays, outs)):
            # the oracle reads only the selected rows: decode just those
            Ksub = P.bf16_np(L["kv"][b, torch.as_tensor(sel, device=DEV, dtype=torch.long)])
            Vsub = Ksub[:, : wl.d_v]
            msg = P.check_attn_row(P.bf16_np(o[b, t]), P.bf16_np(L["q"][b, t]), Ksub, Vsub,
                                   np.arange(sel.size), wl.sm_scale, P.to_np(lse[b, t]).astype(np.float64))
            assert msg is None, f"attention {(b, t)} layer {li}: {msg}"


def _run(name):
    wl = W.WORKLOADS[name]
    ind = W.make_indexer_inputs(wl, device=DEV)
    lays = [W.make_attn_inputs(wl, l, device=DEV) for l in range(wl.group)]
    layer_args = [{"q": L["q"], "kv": L["kv"], "v": None} for L in lays]
    idx, outs = dsa.dsa_group_forward(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], wl.topk, layer_args,
                                      wl.sm_scale, wl.d_v, pool=wl.pool, t_chunk=_t_chunk(wl), want_lse=True)
    torch.cuda.synchronize()
    _check(wl, ind, lays, idx, outs, _sample_rows(wl))


@pytest.mark.parametrize("name", ["prefill32k", "prefill128k", "decode256k", "decode256k_pool", "chunk1m", "chunk1m_pool"])
def test_full_size_group_sampled_rows(name):
    _run(name)


def test_per_layer_indexer_comparator_prefill32k():
    """Without IndexShare each layer runs its own indexer and top-k on its own inputs."""
    wl = W.WORKLOADS["prefill32k"]
    rows = _sample_rows(wl, n_random=1)
    for layer in range(2):
        ind = W.make_indexer_inputs(wl, device=DEV, layer=layer)
        lay = W.make_attn_inputs(wl, layer, device=DEV)
        idx, outs = dsa.dsa_group_forward(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], wl.topk,
                                          [{"q": lay["q"], "kv": lay["kv"], "v": None}], wl.sm_scale, wl.d_v,
                                          t_chunk=_t_chunk(wl), want_lse=True)
        torch.cuda.synchronize()
        _check(wl, ind, [lay], idx, outs, rows)
        del ind, lay, idx, outs
        torch.cuda.empty_cache()
