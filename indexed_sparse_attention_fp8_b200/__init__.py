"""B200 (sm_100a) DSA layer group: FP8 lightning indexer -> top-k -> sparse MQA/MLA attention,
with IndexShare (one selection per group of layers) and IndexPool.

This module is a thin ctypes binding over the C ABI of libdsa_b200.so (include/dsa.h): it
only marshals torch tensors into pointers and sizes.  Every step of the computation runs in
the library's CUDA kernels; there is no CPU or PyTorch fallback.  Functions keep the C names.
PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa_b200.so")

_c_int, _c_i64, _c_p, _c_sz, _c_f = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float

STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED_SHAPE", 3: "DSA_ERR_MISALIGNED",
          4: "DSA_ERR_WORKSPACE_TOO_SMALL", 5: "DSA_ERR_CUDA", 6: "DSA_ERR_TIMEOUT", 7: "DSA_ERR_INDEX_RANGE"}


class DSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} -> {STATUS.get(status, status)}: {_lib().dsa_status_string(status).decode()}"
        if status == 5:
            msg += f" (cudaError {_lib().dsa_last_cuda_error()})"
        super().__init__(msg)


class Paging(ctypes.Structure):
    """Mirror of dsa_paging in include/dsa.h: logical row s of sequence b lives at physical row
    block_table[b, s // page_size] * page_size + s % page_size of each page pool."""
    _fields_ = [("block_table", _c_p), ("page_size", ctypes.c_int32), ("pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


def paging(block_table: torch.Tensor, page_size: int, num_pages: int) -> Paging:
    """A page map for the calls below: block_table [B, pages_per_seq] int32 on the device (kept
    alive by the returned object), page_size a power of two >= 128, num_pages pages per pool."""
    _layout("block_table", block_table, torch.int32, (-1, -1))
    p = Paging(block_table=_ptr(block_table), page_size=int(page_size), pages_per_seq=int(block_table.shape[1]),
               num_pages=int(num_pages))
    p._table = block_table
    return p


def _paging_ref(p: Optional[Paging]):
    return None if p is None else ctypes.byref(p)


class GroupArgs(ctypes.Structure):
    """Mirror of dsa_group_args in include/dsa.h."""
    _fields_ = [
        ("q_idx", _c_p), ("w", _c_p), ("k_idx", _c_p), ("ctx_len", _c_p),
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("S_max", ctypes.c_int32), ("H_I", ctypes.c_int32),
        ("d_I", ctypes.c_int32), ("topk", ctypes.c_int32), ("pool", ctypes.c_int32),
        ("group_size", ctypes.c_int32),
        ("q", ctypes.POINTER(_c_p)), ("kv", ctypes.POINTER(_c_p)), ("v", ctypes.POINTER(_c_p)),
        ("out", ctypes.POINTER(_c_p)), ("lse", ctypes.POINTER(_c_p)),
        ("kv_row_stride", _c_i64), ("kv_batch_stride", _c_i64), ("v_row_stride", _c_i64),
        ("v_batch_stride", _c_i64),
        ("Hq", ctypes.c_int32), ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32), ("sm_scale", _c_f),
        ("idx", _c_p), ("paging", Paging), ("fused_select", ctypes.c_int32), ("k_pooled", _c_p),
    ]


_LIB = None

# name -> (restype, argtypes)
_SIGS = {
    "dsa_status_string": (ctypes.c_char_p, [_c_int]),
    "dsa_last_cuda_error": (_c_int, []),
    "dsa_launch_count": (ctypes.c_uint64, []),
    "dsa_device_status": (_c_int, [_c_p]),
    "dsa_debug_wait_timeout": (_c_int, [ctypes.c_uint64, _c_p]),
    "dsa_debug_set_wait_limit": (_c_int, [ctypes.c_uint64]),
    "dsa_index_scores": (_c_int, [_c_p, _c_p, _c_p, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                  _c_int, _c_int, _c_p, _c_i64, ctypes.POINTER(Paging), _c_p]),
    "dsa_topk": (_c_int, [_c_p, _c_i64, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_p, _c_p]),
    "dsa_index_select_workspace_size": (_c_sz, [_c_int, _c_int, _c_int, _c_int]),
    "dsa_index_select": (_c_int, [_c_p, _c_p, _c_p, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                  _c_int, _c_int, _c_p, _c_p, _c_sz, ctypes.POINTER(Paging), _c_p]),
    "dsa_sparse_attn_workspace_size": (_c_sz, [_c_int, _c_int, _c_int, _c_int, _c_int]),
    "dsa_sparse_attn": (_c_int, [_c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_int, _c_p, _c_int, _c_int,
                                 _c_int, _c_int, _c_int, _c_int, _c_f, _c_p, _c_p, _c_p, _c_sz, ctypes.POINTER(Paging),
                                 _c_p]),
    "dsa_index_pool": (_c_int, [_c_p, _c_int, _c_int, _c_int, _c_int, _c_p, ctypes.POINTER(Paging), _c_p]),
    "dsa_index_pool_tail": (_c_int, [_c_p, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_p, ctypes.POINTER(Paging),
                                     _c_p]),
    "dsa_noalloc_scratch_bytes": (_c_sz, []),
    "dsa_sparse_attn_noalloc": (_c_int, [_c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_int, _c_p, _c_int,
                                         _c_int, _c_int, _c_int, _c_int, _c_int, _c_f, _c_p, _c_p,
                                         ctypes.POINTER(Paging), _c_p]),
    "dsa_group_workspace_size": (_c_sz, [ctypes.POINTER(GroupArgs), _c_int]),
    "dsa_group_forward": (_c_int, [ctypes.POINTER(GroupArgs), _c_p, _c_sz, _c_p]),
    "dsa_gather_selected": (_c_int, [_c_p, _c_i64, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_p, _c_p,
                                     _c_p]),
    "dsa_topk_merge": (_c_int, [_c_p, _c_p, _c_int, _c_i64, _c_int, _c_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                _c_int, _c_p, _c_p]),
    "dsa_idx_localize": (_c_int, [_c_p, _c_i64, _c_int, _c_int, _c_p, _c_p]),
    "dsa_attn_combine": (_c_int, [_c_p, _c_p, _c_int, _c_i64, _c_int, _c_p, _c_p, _c_p]),
}


def _lib() -> ctypes.CDLL:
    """Load libdsa_b200.so (raises if it has not been built: there is no fallback)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m indexed_sparse_attention_fp8_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _LIB = lib
    return _LIB


def _check(fn: str, status: int):
    if status != 0:
        raise DSAError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device (the library has no CPU path)")
    return t.data_ptr()


def _layout(name: str, t: Optional[torch.Tensor], dtype: torch.dtype, shape: Sequence[int],
            strides: Optional[Sequence[int]] = None) -> None:
    """Checks that a tensor has the dtype, shape and element strides the C ABI assumes for it
    (row-major contiguous unless `strides` is given; -1 in `shape` or `strides` matches any)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.dim() != len(shape) or any(want not in (-1, got) for want, got in zip(shape, t.shape)):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if strides is None:
        if not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous (strides {t.stride()})")
    elif any(want not in (-1, got) for want, got in zip(strides, t.stride())):
        raise ValueError(f"{name}: strides {t.stride()}, expected {tuple(strides)}")


def _kv_layout(name: str, t: Optional[torch.Tensor], B: int, width: int, pg: Optional[Paging] = None) -> None:
    """A K or V cache [B, S, >= width] bf16 with unit inner stride and row / batch strides that
    are multiples of 8 elements (16 bytes); with paging, a page pool [num_pages, page_size,
    >= width] whose pages follow each other at the row stride."""
    if t is None:
        return
    if pg is not None:
        _layout(name, t, torch.bfloat16, (pg.num_pages, pg.page_size, -1), (-1, -1, 1))
        if t.stride(0) != pg.page_size * t.stride(1):
            raise ValueError(f"{name}: pages must follow each other at the row stride (strides {t.stride()})")
        B = pg.num_pages
    else:
        _layout(name, t, torch.bfloat16, (B, -1, -1), (-1, -1, 1))
    if t.shape[2] < width or t.stride(1) < width or t.stride(1) % 8 or t.stride(0) % 8:
        raise ValueError(f"{name}: shape {tuple(t.shape)} strides {t.stride()} cannot hold {width}-wide rows "
                         "at 16-byte aligned row and batch strides")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def launch_count() -> int:
    return int(_lib().dsa_launch_count())


def dsa_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the kernels' device status: 0, 6
    (DSA_ERR_TIMEOUT) when a bounded device wait gave up, or 7 (DSA_ERR_INDEX_RANGE) when a
    call met an id beyond what it may read (attention: a selected id past its cache; the
    context-parallel gather and merge: an id past the score row or the row's visible keys)
    and skipped it."""
    return int(_lib().dsa_device_status(_stream(stream)))


def dsa_debug_set_wait_limit(limit_ns: int) -> None:
    """Time limit of the real kernels' bounded waits (1 ns .. 2 s; 0 = the default 2 s)."""
    _check("dsa_debug_set_wait_limit", _lib().dsa_debug_set_wait_limit(int(limit_ns)))


def dsa_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    """Enqueue the bounded-wait probe: its wait runs out after limit_ns and sets the status."""
    _check("dsa_debug_wait_timeout", _lib().dsa_debug_wait_timeout(int(limit_ns), _stream(stream)))


# ---------------------------------------------------------------------------------- calls


def dsa_index_scores(q_idx: torch.Tensor, w: torch.Tensor, k_idx: torch.Tensor, ctx_len: torch.Tensor,
                     pool: int = 1, t_begin: int = 0, t_count: Optional[int] = None,
                     scores: Optional[torch.Tensor] = None, paging: Optional[Paging] = None,
                     stream=None) -> torch.Tensor:
    """Indexer scores [B, t_count, ld] fp32 of queries t_begin.. (see dsa_index_scores in dsa.h).
    q_idx [B,T,H_I,d_I] uint8 (e4m3), w [B,T,H_I] f32, k_idx [B,S,d_I] uint8 (or its page pool
    [num_pages, page_size, d_I] with `paging`), ctx_len [B] i32."""
    B, T, H, D = q_idx.shape
    S = k_idx.shape[1] if paging is None else paging.pages_per_seq * paging.page_size
    tc = T - t_begin if t_count is None else t_count
    ld = (S + 3) // 4 * 4
    _layout("q_idx", q_idx, torch.uint8, (B, T, H, D))
    _layout("w", w, torch.float32, (B, T, H))
    if paging is None:
        _layout("k_idx", k_idx, torch.uint8, (B, S, D))
    else:
        _layout("k_idx", k_idx, torch.uint8, (paging.num_pages, paging.page_size, D))
    _layout("ctx_len", ctx_len, torch.int32, (B,))
    if scores is None:
        scores = torch.empty((B, tc, ld), dtype=torch.float32, device=q_idx.device)
    else:
        ld = scores.stride(1)
        _layout("scores", scores, torch.float32, (B, tc, -1), (tc * ld, ld, 1))
    _check("dsa_index_scores", _lib().dsa_index_scores(
        _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(ctx_len), B, T, S, H, D, pool, t_begin, tc, _ptr(scores), ld,
        _paging_ref(paging), _stream(stream)))
    return scores


def dsa_topk(scores: torch.Tensor, ctx_len: torch.Tensor, T: int, S_max: int, k: int, pool: int = 1,
             t_begin: int = 0, idx: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Top-k token ids [B, T, k*pool] int32 (rows t_begin .. t_begin + scores.shape[1] written)."""
    B, tc, ld = scores.shape
    _layout("scores", scores, torch.float32, (B, tc, -1), (tc * scores.stride(1), -1, 1))
    _layout("ctx_len", ctx_len, torch.int32, (B,))
    if idx is None:
        idx = torch.full((B, T, k * pool), -1, dtype=torch.int32, device=scores.device)
    _layout("idx", idx, torch.int32, (B, T, k * pool))
    _check("dsa_topk", _lib().dsa_topk(_ptr(scores), scores.stride(1), _ptr(ctx_len), B, T, S_max, pool, t_begin,
                                       tc, k, _ptr(idx), _stream(stream)))
    return idx


def _cache_rows(kv: torch.Tensor, v: Optional[torch.Tensor], pg: Optional[Paging] = None) -> int:
    """Rows per sequence of the K/V caches (logical rows when paged): selected ids at or beyond
    it are skipped on the device."""
    if pg is not None:
        return pg.pages_per_seq * pg.page_size
    return int(kv.shape[1] if v is None else min(kv.shape[1], v.shape[1]))


def dsa_index_select_workspace_size(B: int, t_chunk: int, S_max: int, pool: int = 1) -> int:
    return int(_lib().dsa_index_select_workspace_size(B, t_chunk, S_max, pool))


def dsa_index_select(q_idx: torch.Tensor, w: torch.Tensor, k_idx: torch.Tensor, ctx_len: torch.Tensor, k: int,
                     pool: int = 1, t_begin: int = 0, t_count: Optional[int] = None, idx: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None, t_chunk: Optional[int] = None, paging: Optional[Paging] = None,
                     stream=None) -> torch.Tensor:
    """Indexer + top-k of rows t_begin.. in one call (fused: no full score rows where the keys
    allow it).  Same ids as dsa_index_scores followed by dsa_topk.  Returns idx [B, T, k*pool]."""
    B, T, H, D = q_idx.shape
    S = k_idx.shape[1] if paging is None else paging.pages_per_seq * paging.page_size
    tc = T - t_begin if t_count is None else t_count
    _layout("q_idx", q_idx, torch.uint8, (B, T, H, D))
    _layout("w", w, torch.float32, (B, T, H))
    if paging is None:
        _layout("k_idx", k_idx, torch.uint8, (B, S, D))
    else:
        _layout("k_idx", k_idx, torch.uint8, (paging.num_pages, paging.page_size, D))
    _layout("ctx_len", ctx_len, torch.int32, (B,))
    if idx is None:
        idx = torch.full((B, T, k * pool), -1, dtype=torch.int32, device=q_idx.device)
    _layout("idx", idx, torch.int32, (B, T, k * pool))
    if ws is None:
        ws = torch.empty(dsa_index_select_workspace_size(B, t_chunk or tc, S, pool), dtype=torch.uint8,
                         device=q_idx.device)
    _check("dsa_index_select", _lib().dsa_index_select(
        _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(ctx_len), B, T, S, H, D, pool, t_begin, tc, k, _ptr(idx), _ptr(ws),
        ws.numel() * ws.element_size(), _paging_ref(paging), _stream(stream)))
    return idx


def _attn_layouts(q, kv, v, idx, d_v, out, lse, pg: Optional[Paging] = None) -> None:
    B, T, Hq, Dqk = q.shape
    _layout("q", q, torch.bfloat16, (B, T, Hq, Dqk))
    _kv_layout("kv", kv, B, Dqk, pg)
    _kv_layout("v", v, B, d_v, pg)
    _layout("idx", idx, torch.int32, (B, T, -1))
    _layout("out", out, torch.bfloat16, (B, T, Hq, d_v))
    _layout("lse", lse, torch.float32, (B, T, Hq))


def dsa_sparse_attn_workspace_size(B: int, T: int, Hq: int, d_v: int, k: int) -> int:
    return int(_lib().dsa_sparse_attn_workspace_size(B, T, Hq, d_v, k))


def dsa_sparse_attn(q: torch.Tensor, kv: torch.Tensor, idx: torch.Tensor, sm_scale: float, d_v: int,
                    v: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                    lse: Optional[torch.Tensor] = None, want_lse: bool = False,
                    ws: Optional[torch.Tensor] = None, paging: Optional[Paging] = None, stream=None):
    """Sparse attention: q [B,T,Hq,d_qk] bf16, kv [B,S,*] bf16 (K rows; V = kv[..., :d_v] when v is None;
    page pools [num_pages, page_size, *] with `paging`), idx [B,T,k] int32.
    Returns (out [B,T,Hq,d_v] bf16, lse [B,T,Hq] f32 or None)."""
    B, T, Hq, Dqk = q.shape
    k = idx.shape[-1]
    _attn_layouts(q, kv, v, idx, d_v, out, lse, paging)
    if out is None:
        out = torch.empty((B, T, Hq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, T, Hq), dtype=torch.float32, device=q.device)
    need = dsa_sparse_attn_workspace_size(B, T, Hq, d_v, k)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    v_rs = v.stride(1) if v is not None else 0
    v_bs = v.stride(0) if v is not None else 0
    _check("dsa_sparse_attn", _lib().dsa_sparse_attn(
        _ptr(q), _ptr(kv), _ptr(v), kv.stride(1), kv.stride(0), v_rs, v_bs, _cache_rows(kv, v, paging), _ptr(idx), B,
        T, Hq, Dqk, d_v, k,
        float(sm_scale), _ptr(out), _ptr(lse), _ptr(ws), wsb, _paging_ref(paging), _stream(stream)))
    return out, lse


def dsa_sparse_attn_noalloc(q: torch.Tensor, kv: torch.Tensor, idx: torch.Tensor, sm_scale: float, d_v: int,
                            v: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                            lse: Optional[torch.Tensor] = None, want_lse: bool = False,
                            paging: Optional[Paging] = None, stream=None):
    """dsa_sparse_attn without a workspace: split partials use the library's fixed scratch
    (dsa_noalloc_scratch_bytes() per GPU; problems whose default split would not fit run at fewer
    splits).  For callers that cannot allocate device memory; calls that may overlap on one GPU
    share that scratch and must be serialised."""
    B, T, Hq, Dqk = q.shape
    k = idx.shape[-1]
    _attn_layouts(q, kv, v, idx, d_v, out, lse, paging)
    if out is None:
        out = torch.empty((B, T, Hq, d_v), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, T, Hq), dtype=torch.float32, device=q.device)
    v_rs = v.stride(1) if v is not None else 0
    v_bs = v.stride(0) if v is not None else 0
    _check("dsa_sparse_attn_noalloc", _lib().dsa_sparse_attn_noalloc(
        _ptr(q), _ptr(kv), _ptr(v), kv.stride(1), kv.stride(0), v_rs, v_bs, _cache_rows(kv, v, paging), _ptr(idx),
        B, T, Hq, Dqk, d_v, k,
        float(sm_scale), _ptr(out), _ptr(lse), _paging_ref(paging), _stream(stream)))
    return out, lse


def dsa_index_pool(k_idx: torch.Tensor, pool: int = 4, k_pool: Optional[torch.Tensor] = None,
                   paging: Optional[Paging] = None, B: Optional[int] = None, stream=None):
    """IndexPool: [B, S, d_I] e4m3 keys (or their page pool [num_pages, page_size, d_I] with
    `paging`, for B sequences) -> [B, S/pool, d_I] pooled e4m3 keys (pool 2, 4 or 8)."""
    if paging is None:
        B, S, D = k_idx.shape
        _layout("k_idx", k_idx, torch.uint8, (B, S, D))
    else:
        D = k_idx.shape[2]
        S = paging.pages_per_seq * paging.page_size
        B = int(B if B is not None else paging._table.shape[0])
        _layout("k_idx", k_idx, torch.uint8, (paging.num_pages, paging.page_size, D))
    if k_pool is None:
        k_pool = torch.empty((B, S // pool, D), dtype=torch.uint8, device=k_idx.device)
    _layout("k_pool", k_pool, torch.uint8, (B, S // pool, D))
    _check("dsa_index_pool", _lib().dsa_index_pool(_ptr(k_idx), B, S, D, pool, _ptr(k_pool), _paging_ref(paging),
                                                   _stream(stream)))
    return k_pool


def dsa_index_pool_tail(k_idx: torch.Tensor, ctx_len: torch.Tensor, T: int, k_pool: torch.Tensor, pool: int = 4,
                        paging: Optional[Paging] = None, B: Optional[int] = None, stream=None) -> torch.Tensor:
    """Refresh of a pooled key cache after T keys were appended to every sequence (ctx_len
    [B] int32 after the append): the pooled blocks holding the new rows are recomputed in
    k_pool [B, S/pool, d_I], the rest untouched."""
    if paging is None:
        B, S, D = k_idx.shape
        _layout("k_idx", k_idx, torch.uint8, (B, S, D))
    else:
        D = k_idx.shape[2]
        S = paging.pages_per_seq * paging.page_size
        B = int(B if B is not None else paging._table.shape[0])
        _layout("k_idx", k_idx, torch.uint8, (paging.num_pages, paging.page_size, D))
    _layout("ctx_len", ctx_len, torch.int32, (B,))
    _layout("k_pool", k_pool, torch.uint8, (B, S // pool, D))
    _check("dsa_index_pool_tail", _lib().dsa_index_pool_tail(_ptr(k_idx), _ptr(ctx_len), B, int(T), S, D, pool,
                                                             _ptr(k_pool), _paging_ref(paging), _stream(stream)))
    return k_pool


class Group:
    """Marshalled arguments of one IndexShare group (keeps the pointer arrays alive)."""

    def __init__(self, q_idx, w, k_idx, ctx_len, topk: int, layers: Sequence[dict], sm_scale: float,
                 d_v: int, pool: int = 1, idx: Optional[torch.Tensor] = None, want_lse: bool = False,
                 paging: Optional[Paging] = None, fused_select: bool = False,
                 k_pooled: Optional[torch.Tensor] = None):
        B, T, H, D = q_idx.shape
        S = k_idx.shape[1] if paging is None else paging.pages_per_seq * paging.page_size
        L = len(layers)
        self.layers = list(layers)
        q0, kv0 = layers[0]["q"], layers[0]["kv"]
        Hq, Dqk = q0.shape[2], q0.shape[3]
        _layout("q_idx", q_idx, torch.uint8, (B, T, H, D))
        _layout("w", w, torch.float32, (B, T, H))
        if paging is None:
            _layout("k_idx", k_idx, torch.uint8, (B, S, D))
        else:
            _layout("k_idx", k_idx, torch.uint8, (paging.num_pages, paging.page_size, D))
            _layout("block_table", paging._table, torch.int32, (B, -1))
        _layout("ctx_len", ctx_len, torch.int32, (B,))
        _layout("idx", idx, torch.int32, (B, T, topk * pool))
        if k_pooled is not None:
            if pool == 1:
                raise ValueError("k_pooled needs pool > 1")
            _layout("k_pooled", k_pooled, torch.uint8, (B, S // pool, D))
        v0 = layers[0].get("v")
        for l, lay in enumerate(self.layers):
            # one set of K/V strides describes every layer's caches
            _attn_layouts(lay["q"], lay["kv"], lay.get("v"), torch.empty((B, T, 0), dtype=torch.int32), d_v,
                          lay.get("out"), lay.get("lse"), paging)
            if lay["q"].shape != q0.shape or lay["kv"].stride() != kv0.stride():
                raise ValueError(f"layer {l}: q shape or kv strides differ from layer 0's")
            vl = lay.get("v")
            if (vl is None) != (v0 is None) or (vl is not None and vl.stride() != v0.stride()):
                raise ValueError(f"layer {l}: v presence or strides differ from layer 0's")
        for lay in self.layers:
            if lay.get("out") is None:
                lay["out"] = torch.empty((B, T, Hq, d_v), dtype=torch.bfloat16, device=q0.device)
            if want_lse and lay.get("lse") is None:
                lay["lse"] = torch.empty((B, T, Hq), dtype=torch.float32, device=q0.device)
        self.idx = idx if idx is not None else torch.empty((B, T, topk * pool), dtype=torch.int32, device=q0.device)
        arr = lambda xs: (_c_p * L)(*[_ptr(x) for x in xs])  # noqa: E731
        self._q = arr([l["q"] for l in self.layers])
        self._kv = arr([l["kv"] for l in self.layers])
        vs = [l.get("v") for l in self.layers]
        self._v = arr(vs) if any(v is not None for v in vs) else None
        self._out = arr([l["out"] for l in self.layers])
        lses = [l.get("lse") for l in self.layers]
        self._lse = arr(lses) if any(x is not None for x in lses) else None
        v_any = next((v for v in vs if v is not None), None)
        self.args = GroupArgs(
            q_idx=_ptr(q_idx), w=_ptr(w), k_idx=_ptr(k_idx), ctx_len=_ptr(ctx_len),
            B=B, T=T, S_max=S, H_I=H, d_I=D, topk=topk, pool=pool, group_size=L,
            q=self._q, kv=self._kv, v=self._v, out=self._out, lse=self._lse,
            kv_row_stride=kv0.stride(1), kv_batch_stride=kv0.stride(0),
            v_row_stride=v_any.stride(1) if v_any is not None else 0,
            v_batch_stride=v_any.stride(0) if v_any is not None else 0,
            Hq=Hq, d_qk=Dqk, d_v=d_v, sm_scale=float(sm_scale), idx=_ptr(self.idx),
            paging=paging if paging is not None else Paging(), fused_select=1 if fused_select else 0,
            k_pooled=_ptr(k_pooled))
        self._paging = paging
        self._k_pooled = k_pooled
        self.device = q0.device

    def workspace_size(self, t_chunk: int) -> int:
        return int(_lib().dsa_group_workspace_size(ctypes.byref(self.args), int(t_chunk)))

    def forward(self, ws: torch.Tensor, stream=None):
        _check("dsa_group_forward", _lib().dsa_group_forward(
            ctypes.byref(self.args), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
        return self.idx, [(l["out"], l.get("lse")) for l in self.layers]


def dsa_group_forward(q_idx, w, k_idx, ctx_len, topk: int, layers: Sequence[dict], sm_scale: float, d_v: int,
                      pool: int = 1, t_chunk: Optional[int] = None, ws: Optional[torch.Tensor] = None,
                      want_lse: bool = False, paging: Optional[Paging] = None, fused_select: bool = False,
                      k_pooled: Optional[torch.Tensor] = None, stream=None):
    """One IndexShare group: indexer + top-k once, then attention for each layer dict
    {"q", "kv", optional "v", "out", "lse"}; with `paging`, k_idx and every layer's kv (and v)
    are page pools sharing its block table; with pool > 1 and `k_pooled`, the indexer reads
    that pooled cache (kept current by dsa_index_pool_tail) instead of pooling k_idx.
    Returns (idx, [(out, lse) per layer])."""
    g = Group(q_idx, w, k_idx, ctx_len, topk, layers, sm_scale, d_v, pool, want_lse=want_lse, paging=paging,
              fused_select=fused_select, k_pooled=k_pooled)
    if ws is None:
        ws = torch.empty(g.workspace_size(t_chunk or q_idx.shape[1]), dtype=torch.uint8, device=g.device)
    return g.forward(ws, stream)


# ---------------------------------------------------------------- context parallelism (see dsa.h)

def dsa_gather_selected(scores: torch.Tensor, idx: torch.Tensor, t_begin: int, id_offset: int,
                        cand_score: Optional[torch.Tensor] = None, cand_id: Optional[torch.Tensor] = None,
                        stream=None):
    """A shard's selection (rows t_begin.. of idx [B, T, k], local ids) as candidates
    (score [B, t_count, k] f32, global id [B, t_count, k] i32), from scores [B, t_count, ld]."""
    B, tc, ld = scores.shape
    _, T, k = idx.shape
    _layout("scores", scores, torch.float32, (B, tc, -1), (tc * scores.stride(1), -1, 1))
    _layout("idx", idx, torch.int32, (B, T, k))
    if cand_score is None:
        cand_score = torch.empty((B, tc, k), dtype=torch.float32, device=scores.device)
    if cand_id is None:
        cand_id = torch.empty((B, tc, k), dtype=torch.int32, device=scores.device)
    _layout("cand_score", cand_score, torch.float32, (B, tc, k))
    _layout("cand_id", cand_id, torch.int32, (B, tc, k))
    _check("dsa_gather_selected", _lib().dsa_gather_selected(_ptr(scores), scores.stride(1), _ptr(idx), B, T, t_begin,
                                                             tc, k, id_offset, _ptr(cand_score), _ptr(cand_id),
                                                             _stream(stream)))
    return cand_score, cand_id


def dsa_topk_merge(cand_score: torch.Tensor, cand_id: torch.Tensor, ctx_len: torch.Tensor, T: int, S_total: int, k: int,
                   t_begin: int = 0, idx: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The exact top-k of the union of n_parts shard selections: cand_score / cand_id
    [n_parts, B, t_count, kc] -> idx [B, T, k] (rows t_begin.. written)."""
    P, B, tc, kc = cand_score.shape
    _layout("cand_score", cand_score, torch.float32, (P, B, tc, kc))
    _layout("cand_id", cand_id, torch.int32, (P, B, tc, kc))
    _layout("ctx_len", ctx_len, torch.int32, (B,))
    if idx is None:
        idx = torch.full((B, T, k), -1, dtype=torch.int32, device=cand_score.device)
    _layout("idx", idx, torch.int32, (B, T, k))
    _check("dsa_topk_merge", _lib().dsa_topk_merge(_ptr(cand_score), _ptr(cand_id), P, B * tc * kc, kc, _ptr(ctx_len),
                                                   B, T, S_total, t_begin, tc, k, _ptr(idx), _stream(stream)))
    return idx


def dsa_idx_localize(idx: torch.Tensor, s0: int, s_len: int, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Global key ids -> ids into the shard [s0, s0 + s_len) (others -1), same shape."""
    _layout("idx", idx, torch.int32, tuple(idx.shape))
    if out is None:
        out = torch.empty_like(idx)
    _layout("out", out, torch.int32, tuple(idx.shape))
    _check("dsa_idx_localize", _lib().dsa_idx_localize(_ptr(idx), idx.numel(), s0, s_len, _ptr(out), _stream(stream)))
    return out


def dsa_attn_combine(part_o: torch.Tensor, part_lse: torch.Tensor, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, want_lse: bool = False, stream=None):
    """Merge of attention results over disjoint key sets: part_o [n, ..., d_v] bf16, part_lse
    [n, ...] f32 -> (out [..., d_v] bf16, lse [...] f32 or None)."""
    n, d_v = part_o.shape[0], part_o.shape[-1]
    _layout("part_o", part_o, torch.bfloat16, tuple(part_o.shape))
    _layout("part_lse", part_lse, torch.float32, tuple(part_o.shape[:-1]))
    rows = part_lse[0].numel()
    if out is None:
        out = torch.empty(part_o.shape[1:], dtype=torch.bfloat16, device=part_o.device)
    _layout("out", out, torch.bfloat16, tuple(part_o.shape[1:]))
    if lse is None and want_lse:
        lse = torch.empty(part_lse.shape[1:], dtype=torch.float32, device=part_o.device)
    if lse is not None:
        _layout("lse", lse, torch.float32, tuple(part_lse.shape[1:]))
    _check("dsa_attn_combine", _lib().dsa_attn_combine(_ptr(part_o), _ptr(part_lse), n, rows, d_v, _ptr(out), _ptr(lse),
                                                       _stream(stream)))
    return out, lse
