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
