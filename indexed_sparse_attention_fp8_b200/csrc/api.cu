// C ABI of the DSA library: argument validation, workspace sizing and launch sequencing.
// Every entry point validates everything before its first launch, so a non-zero status
// (other than DSA_ERR_CUDA) means nothing was enqueued.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

static thread_local int g_last_cuda_error = 0;
static thread_local uint64_t g_launches = 0;

void set_cuda_error(cudaError_t e) { g_last_cuda_error = static_cast<int>(e); }
void count_launch() { ++g_launches; }

int num_sms() {
  static int cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// A dsa_paging (NULL or a NULL table: contiguous caches) whose sequences can hold S rows.
int check_paging(const dsa_paging* p, int S) {
  if (p == nullptr || p->block_table == nullptr) return DSA_OK;
  const int ps = p->page_size;
  if (ps < 128 || (ps & (ps - 1))) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (p->pages_per_seq < 1 || p->num_pages < 1) return DSA_ERR_INVALID_ARG;
  if ((int64_t)p->num_pages * ps > (int64_t)INT32_MAX / 2) return DSA_ERR_INVALID_ARG;   // rows fit in int32
  if ((int64_t)p->pages_per_seq * ps < S) return DSA_ERR_INVALID_ARG;                  // logical capacity
  return DSA_OK;
}

// Argument and shape checks of one attention call at `splits` key splits (0 = the default
// count); nothing is launched.
int check_sparse_attn(const uint16_t* q, const uint16_t* kv, const uint16_t* v, int64_t kv_rs, int64_t kv_bs,
                      int64_t v_rs, int64_t v_bs, int S_kv, const int32_t* idx, int B, int T, int Hq, int d_qk,
                      int d_v, int k, const uint16_t* out, const void* ws, size_t ws_bytes, const dsa_paging* paging,
                      int splits) {
  if (B < 0 || T < 0 || k < 1 || k > 8192 || S_kv < 1 || splits < 0) return DSA_ERR_INVALID_ARG;
  if (const int st = check_paging(paging, S_kv)) return st;
  if (!(Hq == 128 && d_qk == 576 && d_v == 512) && !(Hq == 16 && d_qk == 128 && d_v == 128))
    return DSA_ERR_UNSUPPORTED_SHAPE;
  if (Hq == 128 && v != nullptr) return DSA_ERR_UNSUPPORTED_SHAPE;  // MLA: V is part of the K row
  if (kv_rs < d_qk || kv_bs < 0 || (v && (v_rs < d_v || v_bs < 0))) return DSA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return DSA_OK;
  if (!q || !kv || !idx || !out) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out) || (v && !aligned16(v)))
    return DSA_ERR_MISALIGNED;
  if ((kv_rs & 7) || (kv_bs & 7) || (v && ((v_rs & 7) || (v_bs & 7)))) return DSA_ERR_MISALIGNED;
  const size_t need = attn_workspace_bytes(B, T, Hq, d_v, k, splits);
  if (ws_bytes < need) return DSA_ERR_WORKSPACE_TOO_SMALL;
  if (need > 0 && (!ws || !aligned16(ws))) return ws ? DSA_ERR_MISALIGNED : DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

namespace {

bool indexer_shape_ok(int H_I, int d_I) { return (H_I == 64 && d_I == 128) || (H_I == 4 && d_I == 64); }
// IndexPool factors: 1 (off), the pages' 4, and 2 and 8.
bool pool_ok(int pool) { return pool == 1 || pool == 2 || pool == 4 || pool == 8; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int check_index_scores(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                       const int32_t* ctx_len, int B, int T, int S_max, int H_I, int d_I, int pool,
                       int t_begin, int t_count, const float* scores, int64_t ld, const dsa_paging* paging) {
  if (B < 0 || T < 1 || S_max < 1 || t_begin < 0 || t_count < 0 || t_begin + t_count > T)
    return DSA_ERR_INVALID_ARG;
  if (!pool_ok(pool)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (const int st = check_paging(paging, S_max)) return st;
  if (paging && paging->block_table && pool > 1) return DSA_ERR_UNSUPPORTED_SHAPE;   // pooled keys are contiguous
  if (!indexer_shape_ok(H_I, d_I)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (ld < S_max || (ld & 3)) return DSA_ERR_INVALID_ARG;
  if (B == 0 || t_count == 0) return DSA_OK;
  if (!q_idx || !w || !k_idx || !ctx_len || !scores) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(w) || !aligned16(k_idx) || !aligned16(scores)) return DSA_ERR_MISALIGNED;
  return DSA_OK;
}

int check_topk(const float* scores, int64_t ld, const int32_t* ctx_len, int B, int T, int S_max,
               int pool, int t_begin, int t_count, int k, const int32_t* idx) {
  if (B < 0 || T < 1 || S_max < 1 || t_begin < 0 || t_count < 0 || t_begin + t_count > T)
    return DSA_ERR_INVALID_ARG;
  if (!pool_ok(pool)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (k < 1 || k > 2048) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (ld < S_max || (ld & 3)) return DSA_ERR_INVALID_ARG;
  if (B == 0 || t_count == 0) return DSA_OK;
  if (!scores || !ctx_len || !idx) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores)) return DSA_ERR_MISALIGNED;
  return DSA_OK;
}

// ---- selection (indexer + top-k) of a chunk of queries
// Fused where the keys allow it: a sampling pass scores every kSampleStride-th key row, the
// r-th largest sample of a row is its threshold, the indexer appends only the keys scoring at
// least the threshold, and the exact top-k runs on those candidates; rows left with fewer
// than k candidates (or more than kCandCap) are redone from full score rows by a repair pass
// that runs only their work items.  Otherwise the full score rows go through the workspace.
constexpr int kSampleStride = 16;
constexpr int kCandCap = 8192;   // candidates per row (the top-k's shared-memory buffer)

// Workspace of one chunk of `rows` = B * t_chunk query rows, carved in this order.
struct SelectWs {
  bool fused;
  int64_t ld, lds;
  size_t scores, samples, cand, small;   // bytes of each piece (small: tau, cnt, fail)
  size_t total() const { return scores + samples + cand + 3 * small; }
};

SelectWs select_ws(int64_t rows, int S_eff, bool fused) {
  SelectWs w;
  w.fused = fused;
  w.ld = (int64_t)round_up((size_t)S_eff, 4);
  w.lds = (int64_t)round_up((size_t)(S_eff / kSampleStride), 4);
  w.scores = round_up((size_t)rows * w.ld * sizeof(float), 256);
  w.samples = fused ? round_up((size_t)rows * w.lds * sizeof(float), 256) : 0;
  w.cand = fused ? round_up((size_t)rows * kCandCap * sizeof(float2), 256) : 0;
  w.small = fused ? round_up((size_t)rows * sizeof(int), 256) : 0;
  return w;
}

// The fused path needs contiguous keys whose sequences hold whole sampled rows.
bool select_fused_ok(int S_eff, const PageMap& key_pm, int fused_select) {
  return fused_select != 0 && key_pm.bt == nullptr && S_eff >= kSampleStride && S_eff % kSampleStride == 0;
}

// Largest chunk of queries (<= T) whose selection workspace fits `bytes`; 0 if none does.
int select_chunk(size_t bytes, int B, int T, int S_eff, bool fused) {
  int lo = 0, hi = T;
  while (lo < hi) {
    const int mid = lo + (hi - lo + 1) / 2;
    if (select_ws((int64_t)B * mid, S_eff, fused).total() <= bytes) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Selection of rows t0 .. t0+tc-1 of every sequence into idx, using the chunk workspace `ws`.
int run_select(const uint8_t* q_idx, const float* w, const uint8_t* keys, const int32_t* ctx_len, int B, int T,
               int S_eff, int H_I, int d_I, int pool, int t0, int tc, int k, int32_t* idx, uint8_t* ws, bool fused,
               const PageMap& key_pm, cudaStream_t s) {
  const int64_t rows = (int64_t)B * tc;
  const SelectWs L = select_ws(rows, S_eff, fused);
  float* scores = reinterpret_cast<float*>(ws);
  if (!fused) {
    int st = launch_index_scores(q_idx, w, keys, ctx_len, B, T, S_eff, H_I, d_I, pool, t0, tc, scores, L.ld, key_pm, s);
    if (st != DSA_OK) return st;
    return launch_topk(scores, L.ld, ctx_len, B, T, S_eff, pool, t0, tc, k, idx, s);
  }
  float* samples = reinterpret_cast<float*>(ws + L.scores);
  float2* cand = reinterpret_cast<float2*>(ws + L.scores + L.samples);
  float* tau = reinterpret_cast<float*>(ws + L.scores + L.samples + L.cand);
  int* cnt = reinterpret_cast<int*>(ws + L.scores + L.samples + L.cand + L.small);
  int* fail = reinterpret_cast<int*>(ws + L.scores + L.samples + L.cand + 2 * L.small);
  // about 2k candidates expected per row (every kSampleStride-th key scored, r = k/8 of them
  // above the threshold), so falling below k is a rare event even for small k
  const int r = std::min(std::max(k / 8, 32), kCandCap / kSampleStride);
  IndexerMode sample;
  sample.kstride = kSampleStride;
  int st = launch_index_scores(q_idx, w, keys, ctx_len, B, T, S_eff / kSampleStride, H_I, d_I, pool * kSampleStride,
                               t0, tc, samples, L.lds, key_pm, s, sample);
  if (st != DSA_OK) return st;
  if ((st = launch_sample_threshold(samples, L.lds, ctx_len, B, T, S_eff, pool, kSampleStride, t0, tc, r, kCandCap,
                                    tau, s)) != DSA_OK)
    return st;
  if (cudaMemsetAsync(cnt, 0, (size_t)rows * sizeof(int), s) != cudaSuccess) return check_launch();
  IndexerMode cm;
  cm.tau = tau;
  cm.cand = cand;
  cm.cnt = cnt;
  cm.cap = kCandCap;
  if ((st = launch_index_scores(q_idx, w, keys, ctx_len, B, T, S_eff, H_I, d_I, pool, t0, tc, nullptr, L.ld, key_pm, s,
                                cm)) != DSA_OK)
    return st;
  if ((st = launch_topk_cand(cand, cnt, kCandCap, ctx_len, B, T, S_eff, pool, t0, tc, k, idx, fail, s)) != DSA_OK)
    return st;
  // repair: full score rows and the row top-k, for the flagged rows only
  IndexerMode rep;
  rep.row_flag = fail;
  if ((st = launch_index_scores(q_idx, w, keys, ctx_len, B, T, S_eff, H_I, d_I, pool, t0, tc, scores, L.ld, key_pm, s,
                                rep)) != DSA_OK)
    return st;
  return launch_topk(scores, L.ld, ctx_len, B, T, S_eff, pool, t0, tc, k, idx, s, fail);
}

// Workspace pieces of a group call: pooled keys, attention partials, then a selection chunk.
struct GroupWs {
  size_t pool_bytes, attn_bytes, fixed_bytes;
  int S_eff;
  bool fused;
};

GroupWs group_ws(const dsa_group_args* a) {
  GroupWs g;
  g.S_eff = a->pool > 1 ? a->S_max / a->pool : a->S_max;
  g.pool_bytes = a->pool > 1 && !a->k_pooled ? round_up((size_t)a->B * g.S_eff * a->d_I, 256) : 0;
  g.attn_bytes = round_up(attn_workspace_bytes(a->B, a->T, a->Hq, a->d_v, a->topk * a->pool), 256);
  g.fixed_bytes = g.pool_bytes + g.attn_bytes;
  const PageMap key_pm = a->pool > 1 ? PageMap{nullptr, 0, 0, 0} : page_map(&a->paging);
  g.fused = select_fused_ok(g.S_eff, key_pm, a->fused_select);
  return g;
}

int check_group(const dsa_group_args* a) {
  if (!a) return DSA_ERR_INVALID_ARG;
  if (a->group_size < 1 || a->group_size > 16 || !a->q || !a->kv || !a->out || !a->idx)
    return DSA_ERR_INVALID_ARG;
  if (!pool_ok(a->pool)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (a->pool > 1 && (a->S_max % a->pool)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (a->topk < 1 || a->topk > 2048) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (a->topk * a->pool > 8192) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (a->k_pooled && a->pool == 1) return DSA_ERR_INVALID_ARG;
  if (a->k_pooled && !aligned16(a->k_pooled)) return DSA_ERR_MISALIGNED;
  const int S_eff = a->pool > 1 ? a->S_max / a->pool : a->S_max;
  const int64_t ld = (int64_t)round_up((size_t)S_eff, 4);
  int st = check_index_scores(a->q_idx, a->w, a->k_idx, a->ctx_len, a->B, a->T, S_eff, a->H_I,
                              a->d_I, a->pool, 0, a->T, reinterpret_cast<const float*>(16), ld, nullptr);
  if (st != DSA_OK) return st;
  if ((st = check_paging(&a->paging, a->S_max)) != DSA_OK) return st;
  // the attention workspace is carved from the group workspace: only shapes are checked here
  for (int l = 0; l < a->group_size; ++l) {
    const uint16_t* v = a->v ? a->v[l] : nullptr;
    st = check_sparse_attn(a->q[l], a->kv[l], v, a->kv_row_stride, a->kv_batch_stride, a->v_row_stride,
                           a->v_batch_stride, a->S_max, a->idx, a->B, a->T, a->Hq, a->d_qk, a->d_v,
                           a->topk * a->pool, a->out[l], reinterpret_cast<const void*>(256), (size_t)-1,
                           &a->paging);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(int status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DSA_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA launch failed";
    case DSA_ERR_TIMEOUT: return "bounded device wait timed out";
    case DSA_ERR_INDEX_RANGE: return "a selected id was at or beyond the cache length (skipped)";
    default: return "unknown status";
  }
}

int dsa_last_cuda_error(void) { return g_last_cuda_error; }

int dsa_device_status(void* stream) {
  const cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return DSA_ERR_CUDA;
  }
  const unsigned int st =
      indexer_take_status() | attn_tc_take_status() | attn_mma_take_status() | pool_take_status() |
      cp_take_status() | merge_take_status();
  if (st & 1u) return DSA_ERR_TIMEOUT;
  if (st & 2u) return DSA_ERR_INDEX_RANGE;
  return DSA_OK;
}
uint64_t dsa_launch_count(void) { return g_launches; }

int dsa_debug_set_wait_limit(uint64_t limit_ns) {
  if (limit_ns > 2000000000ull) return DSA_ERR_INVALID_ARG;
  const uint64_t v = limit_ns == 0 ? 2000000000ull : limit_ns;
  indexer_set_wait_limit(v);
  attn_tc_set_wait_limit(v);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

int dsa_debug_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return DSA_ERR_INVALID_ARG;
  return launch_wait_timeout_probe(limit_ns, static_cast<cudaStream_t>(stream));
}

int dsa_index_scores(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                     const int32_t* ctx_len, int B, int T, int S_max, int H_I, int d_I, int pool,
                     int t_begin, int t_count, float* scores, int64_t ld, const dsa_paging* paging,
                     void* stream) {
  const int st = check_index_scores(q_idx, w, k_idx, ctx_len, B, T, S_max, H_I, d_I, pool,
                                    t_begin, t_count, scores, ld, paging);
  if (st != DSA_OK || B == 0 || t_count == 0) return st;
  return launch_index_scores(q_idx, w, k_idx, ctx_len, B, T, S_max, H_I, d_I, pool, t_begin,
                             t_count, scores, ld, page_map(paging), static_cast<cudaStream_t>(stream));
}

int dsa_topk(const float* scores, int64_t ld, const int32_t* ctx_len, int B, int T, int S_max,
             int pool, int t_begin, int t_count, int k, int32_t* idx, void* stream) {
  const int st = check_topk(scores, ld, ctx_len, B, T, S_max, pool, t_begin, t_count, k, idx);
  if (st != DSA_OK || B == 0 || t_count == 0) return st;
  return launch_topk(scores, ld, ctx_len, B, T, S_max, pool, t_begin, t_count, k, idx,
                     static_cast<cudaStream_t>(stream));
}

size_t dsa_sparse_attn_workspace_size(int B, int T, int Hq, int d_v, int k) {
  if (B <= 0 || T <= 0 || Hq <= 0 || d_v <= 0 || k <= 0) return 0;
  return attn_workspace_bytes(B, T, Hq, d_v, k);
}

int dsa_sparse_attn(const uint16_t* q, const uint16_t* kv, const uint16_t* v, int64_t kv_row_stride,
                    int64_t kv_batch_stride, int64_t v_row_stride, int64_t v_batch_stride, int S_kv,
                    const int32_t* idx, int B, int T, int Hq, int d_qk, int d_v, int k,
                    float sm_scale, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                    const dsa_paging* paging, void* stream) {
  const int st = check_sparse_attn(q, kv, v, kv_row_stride, kv_batch_stride, v_row_stride,
                                   v_batch_stride, S_kv, idx, B, T, Hq, d_qk, d_v, k, out, ws, ws_bytes, paging);
  if (st != DSA_OK || B == 0 || T == 0) return st;
  return launch_sparse_attn(q, kv, v, kv_row_stride, kv_batch_stride, v_row_stride, v_batch_stride,
                            S_kv, idx, B, T, Hq, d_qk, d_v, k, sm_scale, out, lse, ws, page_map(paging),
                            static_cast<cudaStream_t>(stream));
}

int dsa_index_pool(const uint8_t* k_idx, int B, int S_max, int d_I, int pool, uint8_t* k_pool,
                   const dsa_paging* paging, void* stream) {
  if (B < 0 || S_max < 0 || d_I <= 0) return DSA_ERR_INVALID_ARG;
  if (pool == 1 || !pool_ok(pool) || (S_max % pool) || (d_I % 16)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (const int st = check_paging(paging, S_max)) return st;
  if (B == 0 || S_max == 0) return DSA_OK;
  if (!k_idx || !k_pool) return DSA_ERR_INVALID_ARG;
  if (!aligned16(k_idx) || !aligned16(k_pool)) return DSA_ERR_MISALIGNED;
  return launch_index_pool(k_idx, B, S_max, d_I, pool, k_pool, page_map(paging), static_cast<cudaStream_t>(stream));
}

int dsa_index_pool_tail(const uint8_t* k_idx, const int32_t* ctx_len, int B, int T, int S_max, int d_I, int pool,
                        uint8_t* k_pool, const dsa_paging* paging, void* stream) {
  if (B < 0 || T < 1 || S_max < 0 || d_I <= 0) return DSA_ERR_INVALID_ARG;
  if (pool == 1 || !pool_ok(pool) || (S_max % pool) || (d_I % 16)) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (const int st = check_paging(paging, S_max)) return st;
  if (B == 0 || S_max == 0) return DSA_OK;
  if (!k_idx || !ctx_len || !k_pool) return DSA_ERR_INVALID_ARG;
  if (!aligned16(k_idx) || !aligned16(k_pool)) return DSA_ERR_MISALIGNED;
  return launch_index_pool_tail(k_idx, ctx_len, B, T, S_max, d_I, pool, k_pool, page_map(paging),
                                static_cast<cudaStream_t>(stream));
}

size_t dsa_group_workspace_size(const dsa_group_args* a, int t_chunk) {
  if (!a || t_chunk < 1) return 0;
  const GroupWs g = group_ws(a);
  const int tc = std::min(t_chunk, a->T);
  return g.fixed_bytes + select_ws((int64_t)a->B * tc, g.S_eff, g.fused).total();
}

size_t dsa_index_select_workspace_size(int B, int t_chunk, int S_max, int pool) {
  if (B <= 0 || t_chunk < 1 || S_max < 1 || pool < 1) return 0;
  return select_ws((int64_t)B * t_chunk, S_max, select_fused_ok(S_max, PageMap{nullptr, 0, 0, 0}, 1)).total();
}

int dsa_index_select(const uint8_t* q_idx, const float* w, const uint8_t* k_idx, const int32_t* ctx_len, int B,
                     int T, int S_max, int H_I, int d_I, int pool, int t_begin, int t_count, int k, int32_t* idx,
                     void* ws, size_t ws_bytes, const dsa_paging* paging, void* stream) {
  int st = check_index_scores(q_idx, w, k_idx, ctx_len, B, T, S_max, H_I, d_I, pool, t_begin, t_count,
                              reinterpret_cast<const float*>(16), (int64_t)round_up((size_t)S_max, 4), paging);
  if (st != DSA_OK) return st;
  if (k < 1 || k > 2048) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || t_count == 0) return DSA_OK;
  if (!idx) return DSA_ERR_INVALID_ARG;
  const PageMap key_pm = page_map(paging);
  const bool fused = select_fused_ok(S_max, key_pm, 1);
  const int t_chunk = select_chunk(ws_bytes, B, t_count, S_max, fused);
  if (t_chunk < 1) return DSA_ERR_WORKSPACE_TOO_SMALL;
  if (!ws) return DSA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return DSA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int t0 = t_begin; t0 < t_begin + t_count; t0 += t_chunk) {
    const int tc = std::min(t_chunk, t_begin + t_count - t0);
    st = run_select(q_idx, w, k_idx, ctx_len, B, T, S_max, H_I, d_I, pool, t0, tc, k, idx, static_cast<uint8_t*>(ws),
                    fused, key_pm, s);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

int dsa_group_forward(const dsa_group_args* a, void* ws, size_t ws_bytes, void* stream) {
  int st = check_group(a);
  if (st != DSA_OK) return st;
  if (a->B == 0) return DSA_OK;
  const GroupWs g = group_ws(a);
  const int t_chunk = ws_bytes < g.fixed_bytes ? 0 : select_chunk(ws_bytes - g.fixed_bytes, a->B, a->T, g.S_eff, g.fused);
  if (t_chunk < 1) return DSA_ERR_WORKSPACE_TOO_SMALL;
  if (!ws) return DSA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return DSA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* k_pool = base;
  void* attn_ws = base + g.pool_bytes;
  uint8_t* sel_ws = base + g.fixed_bytes;

  const PageMap pm = page_map(&a->paging);
  const uint8_t* keys = a->k_idx;
  PageMap key_pm = pm;   // the indexer reads the paged keys, or the (contiguous) pooled ones
  if (a->pool > 1) {
    if (a->k_pooled) {   // the caller keeps the pooled cache current (dsa_index_pool_tail)
      keys = a->k_pooled;
    } else {
      st = launch_index_pool(a->k_idx, a->B, a->S_max, a->d_I, a->pool, k_pool, pm, s);
      if (st != DSA_OK) return st;
      keys = k_pool;
    }
    key_pm = PageMap{nullptr, 0, 0, 0};
  }
  // IndexShare: one indexer + one top-k over every query, in chunks that fit the workspace
  for (int t0 = 0; t0 < a->T; t0 += t_chunk) {
    const int tc = std::min(t_chunk, a->T - t0);
    st = run_select(a->q_idx, a->w, keys, a->ctx_len, a->B, a->T, g.S_eff, a->H_I, a->d_I, a->pool, t0, tc, a->topk,
                    a->idx, sel_ws, g.fused, key_pm, s);
    if (st != DSA_OK) return st;
  }
  // every layer of the group reads the same selection
  for (int l = 0; l < a->group_size; ++l) {
    const uint16_t* v = a->v ? a->v[l] : nullptr;
    float* lse = a->lse ? a->lse[l] : nullptr;
    st = launch_sparse_attn(a->q[l], a->kv[l], v, a->kv_row_stride, a->kv_batch_stride,
                            a->v_row_stride, a->v_batch_stride, a->S_max, a->idx, a->B, a->T, a->Hq, a->d_qk,
                            a->d_v, a->topk * a->pool, a->sm_scale, a->out[l], lse, attn_ws, pm, s);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

// ---- context parallelism (keys sharded over ranks; the exchange itself is the caller's)

int dsa_gather_selected(const float* scores, int64_t ld, const int32_t* idx, int B, int T, int t_begin, int t_count,
                        int k, int32_t id_offset, float* cand_score, int32_t* cand_id, void* stream) {
  if (B < 0 || T < 1 || t_begin < 0 || t_count < 0 || t_begin + t_count > T || k < 1 || k > 2048 || ld < 1 ||
      id_offset < 0)
    return DSA_ERR_INVALID_ARG;
  if (B == 0 || t_count == 0) return DSA_OK;
  if (!scores || !idx || !cand_score || !cand_id) return DSA_ERR_INVALID_ARG;
  return dsa::launch_gather_selected(scores, ld, idx, B, T, t_begin, t_count, k, id_offset, cand_score, cand_id,
                                     static_cast<cudaStream_t>(stream));
}

int dsa_topk_merge(const float* cand_score, const int32_t* cand_id, int n_parts, int64_t part_stride, int kc,
                   const int32_t* ctx_len, int B, int T, int S_total, int t_begin, int t_count, int k, int32_t* idx,
                   void* stream) {
  if (B < 0 || T < 1 || S_total < 1 || t_begin < 0 || t_count < 0 || t_begin + t_count > T || n_parts < 1 || kc < 1)
    return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > 2048 || kc < k || (int64_t)n_parts * kc > dsa::kMergeMaxCand) return DSA_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || t_count == 0) return DSA_OK;
  if (part_stride < (int64_t)B * t_count * kc) return DSA_ERR_INVALID_ARG;
  if (!cand_score || !cand_id || !ctx_len || !idx) return DSA_ERR_INVALID_ARG;
  return dsa::launch_topk_merge(cand_score, cand_id, n_parts, part_stride, kc, ctx_len, B, T, S_total, t_begin,
                                t_count, k, idx, static_cast<cudaStream_t>(stream));
}

int dsa_idx_localize(const int32_t* idx, int64_t n, int32_t s0, int32_t s_len, int32_t* out, void* stream) {
  if (n < 0 || s0 < 0 || s_len < 0) return DSA_ERR_INVALID_ARG;
  if (n == 0) return DSA_OK;
  if (!idx || !out) return DSA_ERR_INVALID_ARG;
  return dsa::launch_idx_localize(idx, n, s0, s_len, out, static_cast<cudaStream_t>(stream));
}

int dsa_attn_combine(const uint16_t* part_o, const float* part_lse, int n_parts, int64_t rows, int d_v, uint16_t* out,
                     float* lse, void* stream) {
  if (n_parts < 1 || n_parts > 16 || rows < 0 || d_v < 2 || (d_v & 1)) return DSA_ERR_INVALID_ARG;
  if (rows == 0) return DSA_OK;
  if (!part_o || !part_lse || !out) return DSA_ERR_INVALID_ARG;
  if (!dsa::aligned16(part_o) || !dsa::aligned16(out)) return DSA_ERR_MISALIGNED;
  return dsa::launch_attn_combine(part_o, true, part_lse, n_parts, rows, d_v, out, lse,
                                  static_cast<cudaStream_t>(stream));
}

}  // extern "C"
