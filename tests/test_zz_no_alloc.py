"""The workspace-free attention entry point (dsa_sparse_attn_noalloc), for callers that can
neither allocate device memory nor pass a workspace.  It must give the same results as
dsa_sparse_attn on split-key (decode-shaped) problems, on two calls in a row with different
inputs (the shared scratch keeps the previous call's contents), with and without the lse
output, at both split counts the MLA kernel picks for decode batches (4 splits up to 18
queries, 2 from 19 to 37), and for a 32-query decode batch whose default split needs more
partials than the scratch holds (the call then runs at fewer splits instead of failing).
Called through the C ABI.  This file is collected last."""
import numpy as np
import pytest
import torch

import indexed_sparse_attention_fp8_b200 as dsa
from indexed_sparse_attention_fp8_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu


def _decode_case(seed_layer, B, ctx, wl_name="decode256k"):
    wl = W.WORKLOADS[wl_name].replace(B=B, T=1, ctx=ctx)
    lay = W.make_attn_inputs(wl, seed_layer, device="cuda")
    g = torch.Generator(device="cpu").manual_seed(100 + seed_layer)
    idx = torch.randint(0, ctx, (B, 1, wl.topk), generator=g).to(torch.int32)
    idx[:, :, -37:] = -1                                   # a ragged tail of skipped ids
    return wl, lay, idx.cuda()


def _compare(wl, lay, idx, want_lse):
    ref, ref_lse = dsa.dsa_sparse_attn(lay["q"], lay["kv"], idx, wl.sm_scale, wl.d_v, v=lay["v"], want_lse=want_lse)
    got, got_lse = dsa.dsa_sparse_attn_noalloc(lay["q"], lay["kv"], idx, wl.sm_scale, wl.d_v, v=lay["v"],
                                               want_lse=want_lse)
    torch.cuda.synchronize()
    d = np.abs(P.bf16_np(got) - P.bf16_np(ref))
    assert d.max() <= P.ATTN_MAX and d.mean() <= P.ATTN_MEAN
    if want_lse:
        np.testing.assert_allclose(P.to_np(got_lse), P.to_np(ref_lse), rtol=1e-5, atol=1e-5)
    else:
        assert got_lse is None
    assert dsa.dsa_device_status() == 0


@pytest.mark.parametrize("wl_name,B,ctx", [("decode256k", 3, 5000), ("tiny", 4, 700)])
def test_noalloc_matches_workspace_entry_on_two_calls(wl_name, B, ctx):
    lib = dsa._lib()
    assert lib.dsa_noalloc_scratch_bytes() == 16 << 20
    for call in range(2):                                  # second call sees the first call's scratch
        wl, lay, idx = _decode_case(call, B, ctx, wl_name)
        assert dsa.dsa_sparse_attn_workspace_size(B, 1, wl.Hq, wl.d_v, wl.topk) > 0   # split-key path
        _compare(wl, lay, idx, want_lse=True)


@pytest.mark.parametrize("B,want_lse", [(3, False), (24, True), (24, False)])
def test_noalloc_both_mla_split_counts_with_and_without_lse(B, want_lse):
    """B=3 takes 4 key splits, B=24 takes 2; the lse output is optional."""
    wl, lay, idx = _decode_case(2, B, 4100)
    need = dsa.dsa_sparse_attn_workspace_size(B, 1, wl.Hq, wl.d_v, wl.topk)
    assert 0 < need <= dsa._lib().dsa_noalloc_scratch_bytes()
    _compare(wl, lay, idx, want_lse)


def test_noalloc_decode_batch_beyond_its_scratch_runs_at_fewer_splits():
    """32 decode queries: the default split's partials exceed the fixed scratch, so the call
    runs at fewer splits and still matches the workspace entry point."""
    wl, lay, idx = _decode_case(3, 32, 4096)
    need = dsa.dsa_sparse_attn_workspace_size(wl.B, 1, wl.Hq, wl.d_v, wl.topk)
    assert need > dsa._lib().dsa_noalloc_scratch_bytes()
    for want_lse in (True, False):
        _compare(wl, lay, idx, want_lse)
