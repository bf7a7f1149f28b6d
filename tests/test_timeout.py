"""Failure detection without a GPU fault: a device wait whose limit runs out reports
DSA_ERR_TIMEOUT through the status word, and the context stays usable afterwards."""
import pytest
import torch

import indexed_sparse_attention_fp8_b200 as dsa
from indexed_sparse_attention_fp8_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout():
    assert dsa.dsa_device_status() == 0                 # nothing pending
    dsa.dsa_debug_wait_timeout(1_000_000)               # 1 ms limit on a barrier nothing completes
    assert dsa.dsa_device_status() == 6                 # DSA_ERR_TIMEOUT
    assert dsa.dsa_device_status() == 0                 # read-and-clear
    # the context still runs the real kernels correctly
    wl = W.WORKLOADS["tiny"].replace(T=64, ctx=64)
    ind = W.make_indexer_inputs(wl, device="cuda")
    sc = dsa.dsa_index_scores(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"])
    assert torch.isfinite(sc[0, 63, :64]).all()
    assert dsa.dsa_device_status() == 0


def test_timeout_probe_rejects_bad_limits():
    with pytest.raises(dsa.DSAError):
        dsa.dsa_debug_wait_timeout(0)
    with pytest.raises(dsa.DSAError):
        dsa.dsa_debug_wait_timeout(5_000_000_000)


@pytest.mark.parametrize("shape", ["prefill", "decode"])
def test_real_kernels_give_up_their_waits_drain_and_recover(shape):
    """With the wait limit of the real kernels cut to 1 ns (every wait that is not ready at its first
    non-blocking check gives up at once), the tensor-core indexer's and the MLA attention's waits
    run out: each launch sets the status word, drains its copies and MMAs,
    frees TMEM and returns, and dsa_device_status() reports DSA_ERR_TIMEOUT.  With the default
    limit restored, the same calls give exactly the results they gave before.  Both shapes: a
    prefill block (4-query indexer blocks, one CTA per SM; attention in one key split) and
    decode (one-query blocks, two indexer CTAs per SM; attention in key splits with the
    combine)."""
    if shape == "prefill":
        wl = W.WORKLOADS["prefill32k"].replace(T=256, ctx=4096)
    else:
        wl = W.WORKLOADS["decode256k"].replace(B=4, T=1, ctx=20000)
    ind = W.make_indexer_inputs(wl, device="cuda")
    lay = W.make_attn_inputs(wl, 0, device="cuda")
    g = torch.Generator(device="cpu").manual_seed(3)
    idx = torch.stack([torch.randperm(wl.ctx - wl.T, generator=g)[: wl.topk] for _ in range(wl.B * wl.T)])
    idx = idx.to(torch.int32).view(wl.B, wl.T, wl.topk).cuda()
    # score entries past a row's last visible key tile are not written: both calls start from
    # the same sentinel so the comparison covers exactly what the indexer writes
    S = ind["k_idx"].shape[1]

    def scores():
        sc = torch.full((wl.B, wl.T, S), 12345.0, dtype=torch.float32, device="cuda")
        return dsa.dsa_index_scores(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"], scores=sc)
    ref_sc = scores()
    ref_o, ref_l = dsa.dsa_sparse_attn(lay["q"], lay["kv"], idx, wl.sm_scale, wl.d_v, want_lse=True)
    assert dsa.dsa_device_status() == 0
    dsa.dsa_debug_set_wait_limit(1)
    try:
        dsa.dsa_index_scores(ind["q_idx"], ind["w"], ind["k_idx"], ind["ctx_len"])
        st_indexer = dsa.dsa_device_status()
        dsa.dsa_sparse_attn(lay["q"], lay["kv"], idx, wl.sm_scale, wl.d_v, want_lse=True)
        st_attn = dsa.dsa_device_status()
    finally:
        dsa.dsa_debug_set_wait_limit(0)
    assert st_indexer == 6 and st_attn == 6                  # DSA_ERR_TIMEOUT from each kernel
    sc = scores()
    o, l = dsa.dsa_sparse_attn(lay["q"], lay["kv"], idx, wl.sm_scale, wl.d_v, want_lse=True)
    assert dsa.dsa_device_status() == 0
    assert torch.equal(sc, ref_sc) and torch.equal(o, ref_o) and torch.equal(l, ref_l)


def test_wait_limit_hook_rejects_bad_limits():
    with pytest.raises(dsa.DSAError):
        dsa.dsa_debug_set_wait_limit(5_000_000_000)          # above 2 s
