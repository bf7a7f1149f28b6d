// Stage 2 of DeepSeek Sparse Attention, fine selection ("GLM 5.2: How Four Co-Designed
// Mechanisms Beat Raw Scale", section "DeepSeek Sparse Attention"): keep the top-k keys of
// every query's indexer-score row.
//
// One CTA per row.  Radix select on order-preserving 32-bit keys (larger float -> larger
// unsigned key), three digit passes (11 + 11 + 10 bits) with shared-memory histograms, each
// restricted to the keys that share the digits fixed so far, stopping as soon as the pivot
// bucket is taken whole.  When the first digit's pivot bucket fits (TK_CAP keys), one more
// pass over the row takes every key above it as a winner and copies the bucket (key, id) to
// shared memory; the other digits and the ties are then resolved on the copy, so a row is
// read twice instead of up to five times.  Otherwise the digits run over the row and a last
// pass emits the winners.  Either way the winners are every key above the pivot prefix plus
// the lowest-indexed keys equal to it (the same tie rule as a sort by (score desc, index asc)).  The winners are sorted ascending in shared memory (bitonic)
// so the attention gathers walk the KV cache in address order, and written out, expanded
// to token ids when the scores were over IndexPool blocks.
#include "common.cuh"
#include "kernels.h"

#include <climits>

namespace dsa {
namespace {

constexpr int TK_THREADS = 1024;
constexpr int TK_KMAX = 2048;
constexpr int TK_BINS = 2048;
constexpr int TK_CAP = 8192;   // candidate buffer (keys, ids, tie ids) in dynamic shared memory
constexpr int TK_DYN_SMEM = 3 * TK_CAP * 4;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan of one int per thread across the block (blockDim.x == TK_THREADS).
__device__ __forceinline__ int block_excl_scan(int v, int* warp_buf, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_buf[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = warp_buf[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_buf[lane] = s;
  }
  __syncthreads();
  const int excl = x - v + (wid > 0 ? warp_buf[wid - 1] : 0);
  *total = warp_buf[31];
  __syncthreads();
  return excl;
}

// Calls fn(i, score) for every i in [0, n), 16-byte loads where the row allows.  Each thread
// issues TK_UNROLL loads before it consumes any, so a pass over a long row is not a chain of
// one-load round trips to L2.
constexpr int TK_UNROLL = 4;
template <typename F>
__device__ __forceinline__ void for_each_score(const float* __restrict__ row, int n, F&& fn) {
  const int n4 = n >> 2;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  for (int v0 = threadIdx.x; v0 < n4; v0 += TK_UNROLL * TK_THREADS) {
    float4 f[TK_UNROLL];
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) {
      const int v = v0 + u * TK_THREADS;
      if (v < n4) f[u] = __ldcs(r4 + v);
    }
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) {
      const int v = v0 + u * TK_THREADS;
      if (v < n4) {
        fn(4 * v + 0, f[u].x);
        fn(4 * v + 1, f[u].y);
        fn(4 * v + 2, f[u].z);
        fn(4 * v + 3, f[u].w);
      }
    }
  }
  for (int i = 4 * n4 + threadIdx.x; i < n; i += TK_THREADS) fn(i, __ldcs(row + i));
}

__device__ __forceinline__ void write_expanded(int32_t* __restrict__ out, int i, int s, int pool,
                                               int pos) {
  if (pool == 1) {
    out[i] = s;
    return;
  }
  for (int r = 0; r < pool; ++r) {
    const int tok = pool * s + r;
    out[i * pool + r] = (s >= 0 && tok <= pos) ? tok : -1;
  }
}

// Ascending bitonic sort of sel[0..n) in shared memory (n <= TK_KMAX), padded to a power of two.
__device__ __forceinline__ void sort_ascending(int* sel, int n) {
  int P = 1;
  while (P < n) P <<= 1;
  for (int i = n + threadIdx.x; i < P; i += TK_THREADS) sel[i] = INT_MAX;
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (P >> 1); i += TK_THREADS) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const int a = sel[lo], c = sel[hi];
        if ((a > c) == asc) { sel[lo] = c; sel[hi] = a; }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(TK_THREADS, 1)
topk_rows_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ ctx_len,
                 int T, int S_max, int pool, int t_begin, int t_count, int k,
                 int32_t* __restrict__ idx_out, const int* __restrict__ row_flag) {
  __shared__ uint32_t hist[TK_BINS];
  __shared__ int sel[TK_KMAX];
  __shared__ int warp_buf[32];
  __shared__ int sh_bin, sh_above, sh_cnt, sh_ngt, sh_neq;

  const int tid = threadIdx.x;
  const int row_id = blockIdx.x;
  if (row_flag != nullptr && row_flag[row_id] == 0) return;   // only the flagged rows (repair pass)
  const int b = row_id / t_count;
  const int t = t_begin + row_id % t_count;
  const int pos = ctx_len[b] - T + t;
  const int n_valid = pos < 0 ? 0 : min(S_max, pos / pool + 1);
  int32_t* out = idx_out + ((int64_t)b * T + t) * (int64_t)k * pool;

  if (n_valid <= k) {  // every visible key is selected
    for (int i = tid; i < k; i += TK_THREADS) write_expanded(out, i, i < n_valid ? i : -1, pool, pos);
    return;
  }
  const float* row = scores + (int64_t)row_id * ld;
  extern __shared__ uint32_t cand_smem[];
  uint32_t* ck = cand_smem;                                            // candidate keys
  int* ci = reinterpret_cast<int*>(cand_smem + TK_CAP);                 // their row indices
  int* tie = reinterpret_cast<int*>(cand_smem + 2 * TK_CAP);            // ids tied at the pivot

  // ---- radix select of the k-th largest key
  uint32_t prefix = 0, mask = 0;
  int kk = k;          // winners still to find among keys matching `prefix` under `mask`
  int eq_count = 0;    // keys matching the final prefix
  const int shifts[3] = {21, 10, 0};
  // one digit pass over the keys matching prefix/mask (from the row, or from the candidates)
  auto digit_pass = [&](int shift, bool from_cand, int ncand) {
    for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0u;
    __syncthreads();
    if (from_cand) {
      for (int j = tid; j < ncand; j += TK_THREADS) {
        const uint32_t key = ck[j];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (TK_BINS - 1)], 1u);
      }
    } else {
      for_each_score(row, n_valid, [&](int, float f) {
        const uint32_t key = order_key(f);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (TK_BINS - 1)], 1u);
      });
    }
    __syncthreads();
    // thread tid owns bins hb and hb-1, scanned from the top bin down
    const int hb = TK_BINS - 1 - 2 * tid;
    const int h0 = (int)hist[hb], h1 = (int)hist[hb - 1];
    int total;
    const int excl = block_excl_scan(h0 + h1, warp_buf, &total);
    if (excl < kk && kk <= excl + h0) {
      sh_bin = hb; sh_above = excl; sh_cnt = h0;
    } else if (excl + h0 < kk && kk <= excl + h0 + h1) {
      sh_bin = hb - 1; sh_above = excl + h0; sh_cnt = h1;
    }
    __syncthreads();
    kk -= sh_above;
    prefix |= (uint32_t)sh_bin << shift;
    mask |= (uint32_t)(TK_BINS - 1) << shift;
    eq_count = sh_cnt;
  };

  digit_pass(shifts[0], false, 0);
  const int n_gt_1 = k - kk;   // keys above the first pivot digit: all winners
  if (eq_count != kk && eq_count <= TK_CAP) {
    // ---- the pivot bucket fits in shared memory: one more pass over the row takes the keys
    //      above it as winners and copies the bucket; the rest works on the copy
    if (tid == 0) { sh_ngt = 0; sh_neq = 0; }
    __syncthreads();
    for_each_score(row, n_valid, [&](int i, float f) {
      const uint32_t key = order_key(f);
      const uint32_t m = key & mask;
      if (m > prefix) {
        sel[atomicAdd(&sh_ngt, 1)] = i;
      } else if (m == prefix) {
        const int j = atomicAdd(&sh_neq, 1);
        ck[j] = key;
        ci[j] = i;
      }
    });
    __syncthreads();
    const int ncand = sh_neq;   // == eq_count
    for (int p = 1; p < 3 && eq_count != kk; ++p) digit_pass(shifts[p], true, ncand);
    // winners among the candidates: above the final prefix, then the ties (all, or the kk
    // lowest ids)
    const bool take_all_eq = (eq_count == kk);
    if (tid == 0) { sh_ngt = n_gt_1; sh_neq = 0; }
    __syncthreads();
    for (int j = tid; j < ncand; j += TK_THREADS) {
      const uint32_t m = ck[j] & mask;
      if (m > prefix) {
        sel[atomicAdd(&sh_ngt, 1)] = ci[j];
      } else if (m == prefix) {
        tie[atomicAdd(&sh_neq, 1)] = ci[j];
      }
    }
    __syncthreads();
    const int n_gt = sh_ngt, nties = sh_neq;   // n_gt == k - kk
    if (!take_all_eq) sort_ascending(tie, nties);   // the lowest ids win
    __syncthreads();
    for (int j = tid; j < kk; j += TK_THREADS) sel[n_gt + j] = tie[j];
    __syncthreads();
  } else {
    // ---- the pivot bucket is taken whole, or too large to copy: digit passes over the row
    for (int p = 1; p < 3 && eq_count != kk; ++p) digit_pass(shifts[p], false, 0);

    // ---- emit winners: all keys above the prefix, then kk of the keys equal to it
    if (tid == 0) { sh_ngt = 0; sh_neq = 0; }
    __syncthreads();
    const int n_gt = k - kk;
    const bool take_all_eq = (eq_count == kk);
    for_each_score(row, n_valid, [&](int i, float f) {
      const uint32_t m = order_key(f) & mask;
      if (m > prefix) {
        sel[atomicAdd(&sh_ngt, 1)] = i;
      } else if (take_all_eq && m == prefix) {
        sel[n_gt + atomicAdd(&sh_neq, 1)] = i;
      }
    });
    if (!take_all_eq) {
      // exact ties at the k-th key: the lowest indices win (ordered block compaction)
      int base = 0;
      for (int c0 = 0; c0 < n_valid && base < kk; c0 += TK_THREADS) {
        const int i = c0 + tid;
        const int eq = (i < n_valid) && ((order_key(row[i]) & mask) == prefix);
        int total;
        const int r = block_excl_scan(eq, warp_buf, &total);
        if (eq && base + r < kk) sel[n_gt + base + r] = i;
        base += total;
      }
    }
    __syncthreads();
  }

  // ---- ascending bitonic sort of the k winners
  sort_ascending(sel, k);
  for (int i = tid; i < k; i += TK_THREADS) write_expanded(out, i, sel[i], pool, pos);
}


__device__ __forceinline__ float from_order_key(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Threshold of the fused selection (one CTA per query row): the r-th largest of the row's
// visible sampled scores -- the scores of every `stride`-th key row -- by three digit passes
// over the samples; -inf when every visible key fits the candidate buffer (cap) anyway.
__global__ void __launch_bounds__(TK_THREADS, 1)
sample_threshold_kernel(const float* __restrict__ samples, int64_t lds, const int32_t* __restrict__ ctx_len, int T,
                        int S_eff, int pool, int stride, int t_begin, int t_count, int r, int cap,
                        float* __restrict__ tau) {
  __shared__ uint32_t hist[TK_BINS];
  __shared__ int warp_buf[32];
  __shared__ int sh_bin, sh_above;
  const int tid = threadIdx.x;
  const int row_id = blockIdx.x;
  const int b = row_id / t_count;
  const int t = t_begin + row_id % t_count;
  const int pos = ctx_len[b] - T + t;
  const int n_valid = pos < 0 ? 0 : min(S_eff, pos / pool + 1);
  if (n_valid <= cap) {
    if (tid == 0) tau[row_id] = -INFINITY;
    return;
  }
  const int n_s = min((S_eff + stride - 1) / stride, pos / (pool * stride) + 1);   // >= cap / stride >= r
  const float* srow = samples + (int64_t)row_id * lds;
  uint32_t prefix = 0, mask = 0;
  int kk = r;
  const int shifts[3] = {21, 10, 0};
  for (int p = 0; p < 3; ++p) {
    const int shift = shifts[p];
    for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n_s; i += TK_THREADS) {
      const uint32_t key = order_key(__ldg(srow + i));
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (TK_BINS - 1)], 1u);
    }
    __syncthreads();
    const int hb = TK_BINS - 1 - 2 * tid;
    const int h0 = (int)hist[hb], h1 = (int)hist[hb - 1];
    int total;
    const int excl = block_excl_scan(h0 + h1, warp_buf, &total);
    if (excl < kk && kk <= excl + h0) {
      sh_bin = hb; sh_above = excl;
    } else if (excl + h0 < kk && kk <= excl + h0 + h1) {
      sh_bin = hb - 1; sh_above = excl + h0;
    }
    __syncthreads();
    kk -= sh_above;
    prefix |= (uint32_t)sh_bin << shift;
    mask |= (uint32_t)(TK_BINS - 1) << shift;
    __syncthreads();
  }
  if (tid == 0) tau[row_id] = from_order_key(prefix);   // the r-th largest sample exactly
}

// Exact top-k of one row from its candidates (score, key id): the fused indexer appended every
// visible key scoring at least the row's threshold.  When there are at least k candidates the
// k best keys of the row are all among them (ties at the k-th score included), so the result is
// the full row's selection; otherwise, or when the buffer overflowed, the row is flagged for
// the repair pass (full score row + topk_rows_kernel).
__global__ void __launch_bounds__(TK_THREADS, 1)
topk_cand_kernel(const float2* __restrict__ cand, const int* __restrict__ cnt, int cap,
                 const int32_t* __restrict__ ctx_len, int T, int S_max, int pool, int t_begin, int t_count, int k,
                 int32_t* __restrict__ idx_out, int* __restrict__ fail) {
  __shared__ uint32_t hist[TK_BINS];
  __shared__ int sel[TK_KMAX];
  __shared__ int warp_buf[32];
  __shared__ int sh_bin, sh_above, sh_cnt, sh_ngt, sh_neq;
  const int tid = threadIdx.x;
  const int row_id = blockIdx.x;
  const int b = row_id / t_count;
  const int t = t_begin + row_id % t_count;
  const int pos = ctx_len[b] - T + t;
  const int n_valid = pos < 0 ? 0 : min(S_max, pos / pool + 1);
  int32_t* out = idx_out + ((int64_t)b * T + t) * (int64_t)k * pool;
  if (n_valid <= k) {  // every visible key is selected
    if (tid == 0) fail[row_id] = 0;
    for (int i = tid; i < k; i += TK_THREADS) write_expanded(out, i, i < n_valid ? i : -1, pool, pos);
    return;
  }
  const int ncand = cnt[row_id];
  if (ncand < k || ncand > cap) {
    if (tid == 0) fail[row_id] = 1;
    return;
  }
  if (tid == 0) fail[row_id] = 0;
  extern __shared__ uint32_t cand_smem[];
  uint32_t* ck = cand_smem;
  int* ci = reinterpret_cast<int*>(cand_smem + TK_CAP);
  int* tie = reinterpret_cast<int*>(cand_smem + 2 * TK_CAP);
  const float2* crow = cand + (int64_t)row_id * cap;
  for (int j = tid; j < ncand; j += TK_THREADS) {
    const float2 c = __ldcs(crow + j);
    ck[j] = order_key(c.x);
    ci[j] = __float_as_int(c.y);
  }
  __syncthreads();
  uint32_t prefix = 0, mask = 0;
  int kk = k, eq_count = ncand;
  const int shifts[3] = {21, 10, 0};
  for (int p = 0; p < 3 && eq_count != kk; ++p) {
    const int shift = shifts[p];
    for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0u;
    __syncthreads();
    for (int j = tid; j < ncand; j += TK_THREADS) {
      const uint32_t key = ck[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (TK_BINS - 1)], 1u);
    }
    __syncthreads();
    const int hb = TK_BINS - 1 - 2 * tid;
    const int h0 = (int)hist[hb], h1 = (int)hist[hb - 1];
    int total;
    const int excl = block_excl_scan(h0 + h1, warp_buf, &total);
    if (excl < kk && kk <= excl + h0) {
      sh_bin = hb; sh_above = excl; sh_cnt = h0;
    } else if (excl + h0 < kk && kk <= excl + h0 + h1) {
      sh_bin = hb - 1; sh_above = excl + h0; sh_cnt = h1;
    }
    __syncthreads();
    kk -= sh_above;
    prefix |= (uint32_t)sh_bin << shift;
    mask |= (uint32_t)(TK_BINS - 1) << shift;
    eq_count = sh_cnt;
    __syncthreads();
  }
  // winners: every candidate above the prefix, then the ties at it (all, or the kk lowest ids)
  const bool take_all_eq = (eq_count == kk);
  if (tid == 0) { sh_ngt = 0; sh_neq = 0; }
  __syncthreads();
  for (int j = tid; j < ncand; j += TK_THREADS) {
    const uint32_t m = ck[j] & mask;
    if (m > prefix) {
      sel[atomicAdd(&sh_ngt, 1)] = ci[j];
    } else if (m == prefix) {
      tie[atomicAdd(&sh_neq, 1)] = ci[j];
    }
  }
  __syncthreads();
  const int n_gt = sh_ngt, nties = sh_neq;   // n_gt == k - kk
  if (!take_all_eq) sort_ascending(tie, nties);   // the lowest ids win
  __syncthreads();
  for (int j = tid; j < kk; j += TK_THREADS) sel[n_gt + j] = tie[j];
  __syncthreads();
  sort_ascending(sel, k);
  for (int i = tid; i < k; i += TK_THREADS) write_expanded(out, i, sel[i], pool, pos);
}

}  // namespace

int launch_topk(const float* scores, int64_t ld, const int32_t* ctx_len, int B, int T, int S_max,
                int pool, int t_begin, int t_count, int k, int32_t* idx, cudaStream_t stream, const int* row_flag) {
  if (B * t_count == 0) return DSA_OK;
  const int rows = B * t_count;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TK_DYN_SMEM);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  topk_rows_kernel<<<rows, TK_THREADS, TK_DYN_SMEM, stream>>>(scores, ld, ctx_len, T, S_max, pool, t_begin, t_count,
                                                               k, idx, row_flag);
  return check_launch();
}

int launch_sample_threshold(const float* samples, int64_t lds, const int32_t* ctx_len, int B, int T, int S_eff,
                            int pool, int stride, int t_begin, int t_count, int r, int cap, float* tau,
                            cudaStream_t stream) {
  if (B * t_count == 0) return DSA_OK;
  sample_threshold_kernel<<<B * t_count, TK_THREADS, 0, stream>>>(samples, lds, ctx_len, T, S_eff, pool, stride,
                                                                  t_begin, t_count, r, cap, tau);
  return check_launch();
}

int launch_topk_cand(const float2* cand, const int* cnt, int cap, const int32_t* ctx_len, int B, int T, int S_max,
                     int pool, int t_begin, int t_count, int k, int32_t* idx, int* fail, cudaStream_t stream) {
  if (B * t_count == 0) return DSA_OK;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaFuncSetAttribute(topk_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TK_DYN_SMEM);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  topk_cand_kernel<<<B * t_count, TK_THREADS, TK_DYN_SMEM, stream>>>(cand, cnt, cap, ctx_len, T, S_max, pool,
                                                                     t_begin, t_count, k, idx, fail);
  return check_launch();
}

}  // namespace dsa
