"""Shared parity helpers: run oracle rows on inputs read back from the device and compare with
the CUDA path's outputs under the stated tolerances.

Tolerances (all written here, used by every parity test):
  * indexer scores: |gpu - ref| <= 1e-3 |ref|, or <= 1e-5 * D where D = sum_j |w_j| relu(q_j.k)
    (near-zero scores from cancelling signed head weights; the count using the floor is kept);
  * top-k: the GPU set has k_eff distinct valid keys, contains every key scoring above
    tau + 1e-3|tau| (tau = the oracle's k-th score) and none below tau - 1e-3|tau|;
  * attention (bf16 out): max |gpu - ref| <= 2e-2 and mean |gpu - ref| <= 1e-2, where ref is
    the oracle's attention over the GPU's own index set (so tie-band choices do not leak in).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

SCORE_REL, SCORE_FLOOR = 1e-3, 1e-5
TOPK_BAND = 1e-3
ATTN_MAX, ATTN_MEAN = 2e-2, 1e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> float64 via the oracle's own decoder of the raw bits."""
    return O.bf16_to_f64(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


class Decoded:
    """Per-sequence decoded key caches (float64), built lazily from device tensors."""

    def __init__(self, k_idx: torch.Tensor):
        self.k_idx = k_idx
        self.cache = {}

    def __getitem__(self, b):
        if b not in self.cache:
            self.cache = {b: O.e4m3_to_f64(to_np(self.k_idx[b]))}
        return self.cache[b]


def check_scores_row(gpu_row: np.ndarray, q_codes, w_row, kdec, pos, pool=1):
    """Returns (n_floor_used, message or None)."""
    qd = O.e4m3_to_f64(q_codes)
    ref = O.index_scores_row(qd, w_row, kdec, pos, pool)
    S = kdec.shape[0]
    n_valid = min(S, pos // pool + 1)
    mag = O.score_magnitude_row(qd, w_row, kdec, pos, pool)
    ok, nfloor = O.score_close(gpu_row[:n_valid], ref[:n_valid], mag[:n_valid], SCORE_REL, SCORE_FLOOR)
    if not ok.all():
        bad = np.nonzero(~ok)[0][:5]
        return nfloor, f"scores differ at {bad}: gpu {gpu_row[bad]} ref {ref[bad]}"
    tile_end = min(S, (n_valid + 127) // 128 * 128)
    if not np.isneginf(gpu_row[n_valid:tile_end]).all():
        return nfloor, "masked tail of the diagonal tile is not -inf"
    return nfloor, None


def check_topk_row(gpu_idx: np.ndarray, q_codes, w_row, kdec, pos, k, pool=1, kpool_dec=None):
    """GPU top-k row (token ids, ascending, -1 padded) against the oracle's scores."""
    valid = gpu_idx[gpu_idx >= 0]
    if valid.size and not (np.diff(valid) > 0).all():
        return "ids not strictly ascending"
    if (gpu_idx[valid.size:] >= 0).any() and pool == 1:
        return "padding not at the end"
    qd = O.e4m3_to_f64(q_codes)
    if pool == 1:
        ref = O.index_scores_row(qd, w_row, kdec, pos)
        n_valid = min(kdec.shape[0], pos + 1)
        ok, msg = O.topk_set_ok(gpu_idx, ref, n_valid, k, pos, TOPK_BAND)
        return None if ok else msg
    ref = O.index_scores_row(qd, w_row, kpool_dec, pos, pool)
    n_valid = min(kpool_dec.shape[0], pos // pool + 1)
    blocks = np.unique(valid // pool)
    ok, msg = O.topk_set_ok(np.concatenate([blocks, -np.ones(k - blocks.size, np.int64)]), ref, n_valid, k, pos,
                            TOPK_BAND)
    if not ok:
        return "blocks: " + msg
    exp = O.expand_blocks(np.concatenate([blocks, -np.ones(k - blocks.size, np.int64)]), pos, pool)
    if not np.array_equal(np.sort(exp[exp >= 0]), valid):
        return "expansion of the selected blocks differs"
    return None


def check_attn_row(gpu_out: np.ndarray, q_row, K, V, idx_row, sm_scale, gpu_lse=None, out_scaled=False):
    """gpu_out [Hq, d_v] float64 (decoded bf16); q_row [Hq, d_qk], K, V float64.
    out_scaled: the bf16 bounds apply to the output measured in units of max(1, max|O|)
    (outputs far from unit scale carry bf16 rounding in proportion to their size)."""
    ref, lse = O.sparse_attn_row(q_row, K, V, idx_row, sm_scale)
    d = np.abs(gpu_out - ref)
    if out_scaled:
        d = d / max(1.0, float(np.abs(ref).max()))
    if d.max() > ATTN_MAX or d.mean() > ATTN_MEAN:
        return f"attention max {d.max():.3e} mean {d.mean():.3e}"
    if gpu_lse is not None:
        fin = np.isfinite(lse)
        if not np.array_equal(fin, np.isfinite(gpu_lse)):
            return "lse finiteness differs"
        if fin.any() and np.abs(gpu_lse[fin] - lse[fin]).max() > 1e-3 * max(1.0, np.abs(lse[fin]).max()):
            return f"lse differs by {np.abs(gpu_lse[fin] - lse[fin]).max():.3e}"
    return None
