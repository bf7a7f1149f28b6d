"""The C ABI without a GPU: the library builds, loads, exports every function include/dsa.h
declares, and rejects bad arguments before any CUDA call (fake pointers are never touched:
every call here fails validation, which happens before the first launch)."""
import ctypes
import os
import re

import pytest

import indexed_sparse_attention_fp8_b200 as dsa
from indexed_sparse_attention_fp8_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, WS_SMALL = 0, 1, 2, 3, 4
A = 0x10000  # a 16-byte aligned fake address; never dereferenced by the calls below


@pytest.fixture(scope="module")
def lib():
    dsa_build.build()
    return dsa._lib()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|int|size_t|uint64_t)\s+(dsa_\w+)\s*\(", src, re.M)))


def test_header_declares_the_four_calls_and_helpers():
    names = declared_functions()
    for n in ["dsa_index_scores", "dsa_topk", "dsa_sparse_attn", "dsa_group_forward", "dsa_index_pool",
              "dsa_group_workspace_size", "dsa_sparse_attn_workspace_size", "dsa_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_is_the_in_tree_native_build(lib):
    assert os.path.dirname(dsa.LIB_PATH) == os.path.dirname(dsa.__file__)
    assert lib._name == dsa.LIB_PATH


def test_status_strings(lib):
    for code in range(7):
        assert lib.dsa_status_string(code)
    assert lib.dsa_status_string(99) == b"unknown status"


def test_index_scores_validation(lib):
    f = lib.dsa_index_scores
    good = dict(q=A, w=A, k=A, c=A, B=1, T=8, S=8, H=64, D=128, pool=1, tb=0, tc=8, sc=A, ld=8, pg=None)

    def call(**kw):
        a = {**good, **kw}
        return f(a["q"], a["w"], a["k"], a["c"], a["B"], a["T"], a["S"], a["H"], a["D"], a["pool"], a["tb"], a["tc"],
                 a["sc"], a["ld"], a["pg"], None)
    assert call(H=8) == UNSUPPORTED
    assert call(H=64, D=64) == UNSUPPORTED
    assert call(pool=3) == UNSUPPORTED
    assert call(pool=16) == UNSUPPORTED
    assert call(tb=4, tc=5) == INVALID
    assert call(ld=6) == INVALID            # ld not a multiple of 4
    assert call(ld=4) == INVALID            # ld < S_max
    assert call(q=None) == INVALID
    assert call(k=A + 8) == MISALIGNED
    assert call(tc=0) == OK                 # empty chunk: nothing to launch


def test_topk_validation(lib):
    f = lib.dsa_topk
    assert f(A, 8, A, 1, 8, 8, 1, 0, 8, 0, A, None) == UNSUPPORTED      # k = 0
    assert f(A, 8, A, 1, 8, 8, 1, 0, 8, 4096, A, None) == UNSUPPORTED   # k > 2048
    assert f(A, 8, A, 1, 8, 8, 3, 0, 8, 4, A, None) == UNSUPPORTED      # pool 3
    assert f(A + 4, 8, A, 1, 8, 8, 1, 0, 8, 4, A, None) == MISALIGNED
    assert f(A, 8, None, 1, 8, 8, 1, 0, 8, 4, A, None) == INVALID
    assert f(A, 8, A, 0, 8, 8, 1, 0, 8, 4, A, None) == OK               # B = 0


def test_sparse_attn_validation(lib):
    f = lib.dsa_sparse_attn

    def call(Hq=128, dqk=576, dv=512, v=None, kv_rs=576, k=2048, B=1, T=4, ws=None, wsb=0, q=A, S_kv=64, pg=None):
        return f(q, A, v, kv_rs, 576 * 64, 0, 0, S_kv, A, B, T, Hq, dqk, dv, k, 0.04, A, None, ws, wsb, pg, None)
    assert call(Hq=64) == UNSUPPORTED
    assert call(dqk=512) == UNSUPPORTED
    assert call(v=A) == UNSUPPORTED         # MLA shapes read V from the latent row
    assert call(kv_rs=500) == INVALID
    assert call(kv_rs=580) == MISALIGNED    # row stride not a multiple of 16 bytes
    assert call(q=A + 2) == MISALIGNED
    assert call(k=0) == INVALID
    assert call(S_kv=0) == INVALID           # the cache length bounds every selected id
    # decode-shaped problems split the keys and need a workspace
    need = lib.dsa_sparse_attn_workspace_size(32, 1, 128, 512, 2048)
    assert need > 0
    assert call(B=32, T=1, ws=A, wsb=need - 1) == WS_SMALL
    # long prefill needs none
    assert lib.dsa_sparse_attn_workspace_size(1, 32768, 128, 512, 2048) == 0


def test_noalloc_validation_matches_workspace_entry(lib):
    """The workspace-free entry point checks arguments exactly as dsa_sparse_attn does, before
    looking at its scratch: a bad shape or pointer reports the same status there."""
    f, g = lib.dsa_sparse_attn_noalloc, lib.dsa_sparse_attn

    def both(Hq=128, dqk=576, dv=512, v=None, kv_rs=576, k=2048, B=32, T=1, q=A, S_kv=64):
        a = f(q, A, v, kv_rs, 576 * 64, 0, 0, S_kv, A, B, T, Hq, dqk, dv, k, 0.04, A, None, None, None)
        ws_need = lib.dsa_sparse_attn_workspace_size(max(B, 1), max(T, 1), Hq, dv, k) if Hq in (16, 128) else 0
        b = g(q, A, v, kv_rs, 576 * 64, 0, 0, S_kv, A, B, T, Hq, dqk, dv, k, 0.04, A, None, A, ws_need, None, None)
        return a, b
    for kw, want in [({"v": A}, UNSUPPORTED), ({"Hq": 64}, UNSUPPORTED), ({"kv_rs": 500}, INVALID),
                     ({"kv_rs": 580}, MISALIGNED), ({"q": A + 2}, MISALIGNED), ({"k": 0}, INVALID),
                     ({"S_kv": 0}, INVALID), ({"B": -1}, INVALID), ({"B": 0}, OK)]:
        assert both(**kw) == (want, want), kw


def test_index_pool_validation(lib):
    f = lib.dsa_index_pool
    assert f(A, 1, 10, 128, 4, A, None, None) == UNSUPPORTED    # S not a multiple of 4
    assert f(A, 1, 16, 128, 3, A, None, None) == UNSUPPORTED    # pool factors are 2, 4 and 8
    assert f(A, 1, 16, 128, 1, A, None, None) == UNSUPPORTED
    assert f(A, 1, 12, 128, 8, A, None, None) == UNSUPPORTED    # S not a multiple of 8
    assert f(A, 1, 16, 24, 4, A, None, None) == UNSUPPORTED     # d_I not a multiple of 16
    assert f(A + 1, 1, 16, 128, 4, A, None, None) == MISALIGNED
    assert f(A, 0, 16, 128, 4, A, None, None) == OK


def _group_args(pool=1, topk=2048, S=32768, T=32768, B=1, group=4, d_I=128, H_I=64):
    P = ctypes.c_void_p
    arr = (P * group)(*([A] * group))
    return dsa.GroupArgs(q_idx=A, w=A, k_idx=A, ctx_len=A, B=B, T=T, S_max=S, H_I=H_I, d_I=d_I, topk=topk,
                         pool=pool, group_size=group, q=arr, kv=arr, v=None, out=arr, lse=None,
                         kv_row_stride=576, kv_batch_stride=576 * S, v_row_stride=0, v_batch_stride=0,
                         Hq=128, d_qk=576, d_v=512, sm_scale=0.04, idx=A), arr


def test_index_select_validation(lib):
    f = lib.dsa_index_select

    def call(k=2048, pool=1, ws=A, wsb=1 << 30, idx=A, S=4096, tc=8):
        return f(A, A, A, A, 1, 8, S, 64, 128, pool, 0, tc, k, idx, ws, wsb, None, None)
    assert call(k=0) == UNSUPPORTED
    assert call(k=4096) == UNSUPPORTED
    assert call(pool=3) == UNSUPPORTED
    assert call(idx=None) == INVALID
    assert call(wsb=100) == WS_SMALL
    assert call(ws=A + 4) == MISALIGNED
    assert call(tc=0) == OK                                  # nothing to select


def test_paging_validation(lib):
    """A page map is checked before anything is launched: page sizes are powers of two >= 128,
    the table covers the rows the call needs, and pooled indexer keys are never paged."""
    def pg(page_size=256, pps=4, num_pages=16, table=A):
        return ctypes.byref(dsa.Paging(block_table=table, page_size=page_size, pages_per_seq=pps, num_pages=num_pages))
    f = lib.dsa_sparse_attn

    def attn(p, S_kv=1024):
        return f(A, A, None, 576, 0, 0, 0, S_kv, A, 1, 4, 128, 576, 512, 2048, 0.04, A, None, None, 0, p, None)
    assert attn(pg(page_size=192)) == UNSUPPORTED            # not a power of two
    assert attn(pg(page_size=64)) == UNSUPPORTED             # below one indexer tile
    assert attn(pg(pps=0)) == INVALID
    assert attn(pg(num_pages=0)) == INVALID
    assert attn(pg(pps=3)) == INVALID                        # 3 x 256 rows < S_kv = 1024
    assert attn(pg(num_pages=1 << 30)) == INVALID            # pool rows beyond int32
    assert attn(pg(), S_kv=0) == INVALID
    g = lib.dsa_index_scores
    assert g(A, A, A, A, 1, 8, 1024, 64, 128, 4, 0, 8, A, 1024, pg(), None) == UNSUPPORTED   # pooled keys
    assert g(A, A, A, A, 1, 8, 2048, 64, 128, 1, 0, 8, A, 2048, pg(), None) == INVALID      # table too short
    assert lib.dsa_index_pool(A, 1, 2048, 128, 4, A, pg(), None) == INVALID
    assert lib.dsa_index_pool(A, 1, 1024, 128, 4, A, pg(page_size=100), None) == UNSUPPORTED
    bad, keep = _group_args(S=4096, T=4096)
    bad.paging = dsa.Paging(block_table=A, page_size=256, pages_per_seq=8, num_pages=64)   # 2048 < 4096 rows
    assert lib.dsa_group_forward(ctypes.byref(bad), A, 1 << 40, None) == INVALID


def _fused_row_bytes(S):
    """Selection workspace of one query row on the fused path: a full score row (kept for the
    repair pass), the 1/16 samples, 8192 (score, id) candidates, and tau, count and flag
    (each piece rounded to 256 bytes)."""
    r = lambda x: (x + 255) // 256 * 256                    # noqa: E731
    return r(S * 4) + r((S // 16 + 3) // 4 * 4 * 4) + r(8192 * 8) + 3 * r(4)


def test_group_workspace_and_validation(lib):
    args, keep = _group_args()
    args.fused_select = 0                                   # the default: full score rows + top-k
    one = lib.dsa_group_workspace_size(ctypes.byref(args), 1)
    big = lib.dsa_group_workspace_size(ctypes.byref(args), 1024)
    assert one == 32768 * 4 and big == 1024 * 32768 * 4     # a chunk of fp32 score rows
    args.fused_select = 1                                   # fused selection
    one = lib.dsa_group_workspace_size(ctypes.byref(args), 1)
    assert one == _fused_row_bytes(32768)
    assert lib.dsa_index_select_workspace_size(1, 1, 32768, 1) == one
    assert lib.dsa_index_select_workspace_size(1, 1, 32760, 1) == (32760 * 4 + 255) // 256 * 256   # full rows only
    # too small a workspace is refused before any launch
    assert lib.dsa_group_forward(ctypes.byref(args), A, one - 16, None) == WS_SMALL
    bad, keep2 = _group_args(topk=4096)
    assert lib.dsa_group_forward(ctypes.byref(bad), A, 1 << 40, None) == UNSUPPORTED
    pool_args, keep3 = _group_args(pool=4, topk=512, S=1048576, T=8192)
    need = lib.dsa_group_workspace_size(ctypes.byref(pool_args), 1)
    assert need == (1048576 // 4) * 128 + (1048576 // 4) * 4    # pooled keys + one full score row
    pool_args.fused_select = 1
    need = lib.dsa_group_workspace_size(ctypes.byref(pool_args), 1)
    assert need == (1048576 // 4) * 128 + _fused_row_bytes(1048576 // 4)   # pooled keys + one selection row
    odd, keep4 = _group_args(pool=4, topk=512, S=1048574, T=8192)
    assert lib.dsa_group_forward(ctypes.byref(odd), A, 1 << 40, None) == UNSUPPORTED
    # a caller-kept pooled cache: no pooled keys in the workspace; only with pool > 1, aligned
    pool_args.fused_select = 0
    pool_args.k_pooled = A
    assert lib.dsa_group_workspace_size(ctypes.byref(pool_args), 1) == (1048576 // 4) * 4
    pool_args.k_pooled = A + 8
    assert lib.dsa_group_forward(ctypes.byref(pool_args), A, 1 << 40, None) == MISALIGNED
    args.k_pooled = A
    assert lib.dsa_group_forward(ctypes.byref(args), A, 1 << 40, None) == INVALID


def test_index_pool_tail_validation(lib):
    f = lib.dsa_index_pool_tail   # k_idx, ctx_len, B, T, S_max, d_I, pool, k_pool, paging, stream
    assert f(A, A, 1, 1, 16, 128, 3, A, None, None) == UNSUPPORTED     # pool factors are 2, 4 and 8
    assert f(A, A, 1, 1, 10, 128, 4, A, None, None) == UNSUPPORTED     # S not a multiple of 4
    assert f(A, A, 1, 0, 16, 128, 4, A, None, None) == INVALID         # nothing appended
    assert f(A, None, 1, 1, 16, 128, 4, A, None, None) == INVALID
    assert f(A, A, 1, 1, 16, 128, 4, A + 4, None, None) == MISALIGNED
    assert f(A, A, 0, 1, 16, 128, 4, A, None, None) == OK              # no sequences


def test_context_parallel_calls_validation(lib):
    """The four calls around the key-sharded exchange reject bad sizes before any launch."""
    g = lib.dsa_gather_selected   # scores, ld, idx, B, T, t_begin, t_count, k, id_offset, cs, ci, stream
    assert g(A, 4096, A, 1, 8, 4, 8, 2048, 0, A, A, None) == INVALID      # rows past T
    assert g(A, 4096, A, 1, 8, 0, 8, 4096, 0, A, A, None) == INVALID      # k > 2048
    assert g(A, 4096, A, 1, 8, 0, 8, 2048, -1, A, A, None) == INVALID     # negative offset
    assert g(None, 4096, A, 1, 8, 0, 8, 2048, 0, A, A, None) == INVALID
    assert g(A, 4096, A, 1, 8, 0, 0, 2048, 0, A, A, None) == OK           # nothing to gather
    m = lib.dsa_topk_merge   # cs, ci, n_parts, part_stride, kc, ctx, B, T, S, t_begin, t_count, k, idx, stream
    stride = 8 * 2048
    assert m(A, A, 2, stride, 2048, A, 1, 8, 9000, 0, 8, 4096, A, None) == UNSUPPORTED   # k > 2048
    assert m(A, A, 2, stride, 1024, A, 1, 8, 9000, 0, 8, 2048, A, None) == UNSUPPORTED   # kc < k
    assert m(A, A, 9, stride, 2048, A, 1, 8, 9000, 0, 8, 2048, A, None) == UNSUPPORTED   # 9 x 2048 > 16384
    assert m(A, A, 2, stride - 1, 2048, A, 1, 8, 9000, 0, 8, 2048, A, None) == INVALID  # parts overlap
    assert m(A, A, 0, stride, 2048, A, 1, 8, 9000, 0, 8, 2048, A, None) == INVALID
    assert m(A, A, 2, stride, 2048, None, 1, 8, 9000, 0, 8, 2048, A, None) == INVALID
    assert m(A, A, 2, stride, 2048, A, 1, 8, 9000, 0, 0, 2048, A, None) == OK           # no rows
    loc = lib.dsa_idx_localize   # idx, n, s0, s_len, out, stream
    assert loc(A, -1, 0, 10, A, None) == INVALID
    assert loc(A, 10, -1, 10, A, None) == INVALID
    assert loc(None, 10, 0, 10, A, None) == INVALID
    assert loc(A, 0, 0, 10, A, None) == OK
    c = lib.dsa_attn_combine   # part_o, part_lse, n_parts, rows, d_v, out, lse, stream
    assert c(A, A, 17, 8, 512, A, None, None) == INVALID      # more than 16 parts
    assert c(A, A, 2, 8, 511, A, None, None) == INVALID       # odd d_v
    assert c(A + 2, A, 2, 8, 512, A, None, None) == MISALIGNED
    assert c(A, A, 2, 0, 512, A, None, None) == OK            # no rows
