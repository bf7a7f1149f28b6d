// Stage 2 of DeepSeek Sparse Attention, fine selection ("GLM 5.2: How Four Co-Designed
// Mechanisms Beat Raw Scale", section "DeepSeek Sparse Attention"): keep the top-k keys of
// every query's indexer-score row.
//
// One CTA per row.  Radix select on order-preserving 32-bit keys (larger float -> larger
// unsigned key), three digit passes (11 + 11 + 10 bits) with shared-memory histograms, each
// pass restricted to the keys that share the digits fixed so far, stopping as soon as the
// pivot bucket is taken whole.  Then one pass emits the winners: every key above the pivot
// prefix, plus the lowest-indexed keys equal to it (the same tie rule as a sort by
// (score desc, index asc)).  The winners are sorted ascending in shared memory (bitonic)
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
                 int32_t* __restrict__ idx_out) {
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
    for (int i = tid; i < k; i += TK_THREADS) write_expanded(out, i, i < n_valid ? i : -1, pool, pos);
    return;
  }
  const float* row = scores + (int64_t)row_id * ld;

  // ---- radix select of the k-th largest key
  uint32_t prefix = 0, mask = 0;
  int kk = k;          // winners still to find among keys matching `prefix` under `mask`
  int eq_count = 0;    // keys matching the final prefix
  const int shifts[3] = {21, 10, 0};
  for (int p = 0; p < 3; ++p) {
    const int shift = shifts[p];
    for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0u;
    __syncthreads();
    for_each_score(row, n_valid, [&](int, float f) {
      const uint32_t key = order_key(f);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (TK_BINS - 1)], 1u);
    });
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
    if (eq_count == kk) break;  // the whole pivot bucket is selected (block-uniform)
  }

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

  // ---- ascending bitonic sort of the k winners
  sort_ascending(sel, k);
  for (int i = tid; i < k; i += TK_THREADS) write_expanded(out, i, sel[i], pool, pos);
}

// ---- few long rows (decode): a cluster of TK_CL CTAs per row, each over a 1/TK_CL slice
constexpr int TK_CL = 4;

__device__ __forceinline__ uint32_t cl_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// A 32-bit word of CTA `rank`'s shared memory at the address of `p` in this CTA.
__device__ __forceinline__ uint32_t ld_cluster_u32(const void* p, uint32_t rank) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  uint32_t r, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(a), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];\n" : "=r"(v) : "r"(r) : "memory");
  return v;
}

// The selection of topk_rows_kernel with the row split over the TK_CL CTAs of a cluster:
// each pass sums the CTAs' histograms through distributed shared memory (every CTA derives
// the same pivot), and the winners come out in index order because CTA c's slice holds lower
// indices than CTA c+1's: each CTA takes its keys above the pivot prefix plus its share of
// the lowest-indexed ties, sorts them, and writes them after the lower CTAs' winners.
__global__ void __cluster_dims__(TK_CL, 1, 1) __launch_bounds__(TK_THREADS, 1)
topk_rows_cluster_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ ctx_len,
                         int T, int S_max, int pool, int t_begin, int t_count, int k,
                         int32_t* __restrict__ idx_out) {
  __shared__ uint32_t hist[TK_BINS];
  __shared__ int sel[TK_KMAX];
  __shared__ int warp_buf[32];
  __shared__ int sh_bin, sh_above, sh_cnt, sh_ngt, sh_neq;
  __shared__ int sh_counts[2];   // this CTA's keys above the prefix / equal to it

  const int tid = threadIdx.x;
  const uint32_t rank = cl_rank();
  const int row_id = blockIdx.x / TK_CL;
  const int b = row_id / t_count;
  const int t = t_begin + row_id % t_count;
  const int pos = ctx_len[b] - T + t;
  const int n_valid = pos < 0 ? 0 : min(S_max, pos / pool + 1);
  int32_t* out = idx_out + ((int64_t)b * T + t) * (int64_t)k * pool;

  if (n_valid <= k) {  // every visible key is selected (the same for the whole cluster)
    for (int i = (int)rank * TK_THREADS + tid; i < k; i += TK_CL * TK_THREADS)
      write_expanded(out, i, i < n_valid ? i : -1, pool, pos);
    return;
  }
  // this CTA's slice [lo, lo + len), 4-aligned so the 16-byte loads stay aligned
  const int per = ((n_valid + TK_CL - 1) / TK_CL + 3) & ~3;
  const int lo = min(n_valid, (int)rank * per);
  const int len = min(n_valid, lo + per) - lo;
  const float* row = scores + (int64_t)row_id * ld + lo;

  uint32_t prefix = 0, mask = 0;
  int kk = k;
  int eq_count = 0;
  const int shifts[3] = {21, 10, 0};
  for (int p = 0; p < 3; ++p) {
    const int shift = shifts[p];
    for (int i = tid; i < TK_BINS; i += TK_THREADS) hist[i] = 0u;
    __syncthreads();
    for_each_score(row, len, [&](int, float f) {
      const uint32_t key = order_key(f);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (TK_BINS - 1)], 1u);
    });
    cl_sync();   // every CTA's histogram is complete
    const int hb = TK_BINS - 1 - 2 * tid;
    int h0 = 0, h1 = 0;
#pragma unroll
    for (int r = 0; r < TK_CL; ++r) {
      h0 += (int)ld_cluster_u32(&hist[hb], (uint32_t)r);
      h1 += (int)ld_cluster_u32(&hist[hb - 1], (uint32_t)r);
    }
    cl_sync();   // every CTA has read every histogram before any is cleared again
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
    if (eq_count == kk) break;  // the same merged histogram in every CTA: cluster-uniform
  }

  // ---- this CTA's counts above / equal to the prefix, shared with the cluster
  if (tid == 0) { sh_ngt = 0; sh_neq = 0; }
  __syncthreads();
  for_each_score(row, len, [&](int, float f) {
    const uint32_t m = order_key(f) & mask;
    if (m > prefix) atomicAdd(&sh_ngt, 1);
    else if (m == prefix) atomicAdd(&sh_neq, 1);
  });
  __syncthreads();
  if (tid == 0) { sh_counts[0] = sh_ngt; sh_counts[1] = sh_neq; }
  cl_sync();
  // the lowest-indexed kk ties win: CTA c takes ties after those of the lower CTAs
  int out_off = 0, eq_before = 0;
  for (int r = 0; r < (int)rank; ++r) {
    const int gt_r = (int)ld_cluster_u32(&sh_counts[0], (uint32_t)r);
    const int eq_r = (int)ld_cluster_u32(&sh_counts[1], (uint32_t)r);
    out_off += gt_r + min(eq_r, max(0, kk - eq_before));
    eq_before += eq_r;
  }
  const int my_gt = sh_counts[0];
  const int my_eq_take = min(sh_counts[1], max(0, kk - eq_before));
  cl_sync();   // the counts have been read before any CTA may leave

  // ---- collect this CTA's winners (row indices), sort, write after the lower CTAs' winners
  if (tid == 0) sh_ngt = 0;
  __syncthreads();
  for_each_score(row, len, [&](int i, float f) {
    if ((order_key(f) & mask) > prefix) sel[atomicAdd(&sh_ngt, 1)] = lo + i;
  });
  {
    int base = 0;   // ordered compaction of the slice's first my_eq_take ties
    for (int c0 = 0; c0 < len && base < my_eq_take; c0 += TK_THREADS) {
      const int i = c0 + tid;
      const int eq = (i < len) && ((order_key(row[i]) & mask) == prefix);
      int total;
      const int r = block_excl_scan(eq, warp_buf, &total);
      if (eq && base + r < my_eq_take) sel[my_gt + base + r] = lo + i;
      base += total;
    }
  }
  __syncthreads();
  const int mine = my_gt + my_eq_take;
  sort_ascending(sel, mine);
  for (int i = tid; i < mine; i += TK_THREADS) write_expanded(out, out_off + i, sel[i], pool, pos);
}

}  // namespace

int launch_topk(const float* scores, int64_t ld, const int32_t* ctx_len, int B, int T, int S_max,
                int pool, int t_begin, int t_count, int k, int32_t* idx, cudaStream_t stream) {
  if (B * t_count == 0) return DSA_OK;
  const int rows = B * t_count;
  if (rows * TK_CL <= num_sms() && S_max / pool >= TK_CL * 4 * TK_THREADS) {
    // few long rows (decode): a cluster per row, the whole grid in one wave
    topk_rows_cluster_kernel<<<rows * TK_CL, TK_THREADS, 0, stream>>>(scores, ld, ctx_len, T, S_max, pool, t_begin,
                                                                      t_count, k, idx);
    return check_launch();
  }
  topk_rows_kernel<<<rows, TK_THREADS, 0, stream>>>(scores, ld, ctx_len, T, S_max, pool, t_begin, t_count, k, idx);
  return check_launch();
}

}  // namespace dsa
