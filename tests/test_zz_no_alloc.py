"""The workspace-free attention entry point (dsa_sparse_attn_noalloc), for callers that can
neither allocate device memory nor pass a workspace.  It must give the same results as
dsa_sparse_attn on split-key (decode-shaped) problems, on two calls in a row with different
inputs (the shared scratch keeps the previous call's contents), and reject problems larger
than its fixed scratch.  Called through the C ABI."""
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


@pytest.mark.parametrize("wl_name,B,ctx", [("decode256k", 3, 5000), ("tiny", 4, 700)])
def test_noalloc_matches_workspace_entry_on_two_calls(wl_name, B, ctx):
    lib = dsa._lib()
    assert lib.dsa_noalloc_scratch_bytes() == 16 << 20
    for call in range(2):                                  # second call sees the first call's scratch
        wl, lay, idx = _decode_case(call, B, ctx, wl_name)
        assert dsa.dsa_sparse_attn_workspace_size(B, 1, wl.Hq, wl.d_v, wl.topk) > 0   # split-key path
        ref, ref_lse = dsa.dsa_sparse_attn(lay["q"], lay["kv"], idx, wl.sm_scale, wl.d_v, v=lay["v"], want_lse=True)
        got, got_lse = dsa.dsa_sparse_attn_noalloc(lay["q"], lay["kv"], idx, wl.sm_scale, wl.d_v, v=lay["v"],
                                                   want_lse=True)
        torch.cuda.synchronize()
        d = np.abs(P.bf16_np(got) - P.bf16_np(ref))
        assert d.max() <= P.ATTN_MAX and d.mean() <= P.ATTN_MEAN
        np.testing.assert_allclose(P.to_np(got_lse), P.to_np(ref_lse), rtol=1e-5, atol=1e-5)
        assert dsa.dsa_device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    wl = W.WORKLOADS["decode256k"].replace(B=32, T=1, ctx=4096)   # two splits: 16.8 MB of partials
    need = dsa.dsa_sparse_attn_workspace_size(wl.B, 1, wl.Hq, wl.d_v, wl.topk)
    assert need > dsa._lib().dsa_noalloc_scratch_bytes()
    q = torch.zeros((wl.B, 1, wl.Hq, wl.d_qk), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((wl.B, 64, wl.d_qk), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((wl.B, 1, wl.topk), dtype=torch.int32, device="cuda")
    with pytest.raises(dsa.DSAError) as ei:
        dsa.dsa_sparse_attn_noalloc(q, kv, idx, wl.sm_scale, wl.d_v)
    assert ei.value.status == 4                            # DSA_ERR_WORKSPACE_TOO_SMALL, nothing enqueued
