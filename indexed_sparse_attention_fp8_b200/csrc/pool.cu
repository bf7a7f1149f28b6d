// IndexPool ("GLM-5.3-Flash hybrid sparse-linear attention with IndexPool", section "What
// changed"): four consecutive indexer keys pooled into one key, so the indexer scores a
// quarter as many rows.  The pooled key is the fp32 mean ((k0 + k1) + (k2 + k3)) * 0.25 of
// the decoded e4m3 keys, requantised to e4m3 round-to-nearest-even with saturation.  Factors
// P = 2 and 8 take the same mean (a balanced pairwise fp32 sum times 1/P); P <= 8 e4m3
// values sum exactly in fp32, so the requantisation is the only rounding.
//
// HBM-bound streaming: each thread reads one 16-byte slice (16 dims) of the P source rows
// and writes one 16-byte slice of the pooled row.
#include "common.cuh"
#include "kernels.h"

namespace dsa {

// Status word of the pool kernel (bit 1: a page id out of range); read through
// dsa_device_status().
__device__ unsigned int g_pool_status;

namespace {

__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));   // e4m3 -> f16 is exact
}

// Pools group g (global over the B sequences: groups_per_seq per sequence) at 16-byte slice
// sl: the P source rows' slices are read, and the pooled slice is written to k_pool.
template <int P>
__device__ __forceinline__ void pool_group(const uint4* __restrict__ k_idx, int64_t g, int groups_per_seq, int slices,
                                           int sl, uint4* __restrict__ k_pool, const PageMap& pm) {
  // first source row of the group: contiguous, or in the page of its sequence that holds it
  // (a page holds whole groups: its size is a multiple of P); a bad page id reads as zeros
  int64_t row0 = P * g;
  bool ok = true;
  if (pm.bt != nullptr) {
    const int b = (int)(g / groups_per_seq);
    const int r = paged_row(pm, b, P * (int)(g % groups_per_seq));
    if (r < 0) {
      atomicOr(&g_pool_status, 2u);
      ok = false;
    }
    row0 = r;
  }
  uint4 src[P];
#pragma unroll
  for (int r = 0; r < P; ++r) src[r] = ok ? __ldcs(k_idx + (row0 + r) * slices + sl) : make_uint4(0, 0, 0, 0);
  uint32_t outw[4];
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    uint32_t packed = 0;
#pragma unroll
    for (int hpair = 0; hpair < 2; ++hpair) {
      float2 v[P];
#pragma unroll
      for (int r = 0; r < P; ++r) {
        const uint32_t word = (&src[r].x)[wd];
        v[r] = e4m3x2_to_float2(static_cast<uint16_t>(word >> (16 * hpair)));
      }
      // balanced pairwise sum: (k0 + k1), (k2 + k3), ... then the pair sums, and so on
#pragma unroll
      for (int n = P; n > 1; n >>= 1) {
#pragma unroll
        for (int i = 0; i < n / 2; ++i) v[i] = make_float2(v[2 * i].x + v[2 * i + 1].x, v[2 * i].y + v[2 * i + 1].y);
      }
      float2 m;
      m.x = v[0].x * (1.0f / P);
      m.y = v[0].y * (1.0f / P);
      const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(m, __NV_SATFINITE, __NV_E4M3);
      packed |= static_cast<uint32_t>(q) << (16 * hpair);
    }
    outw[wd] = packed;
  }
  k_pool[g * slices + sl] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
}

// Every group of every sequence: one thread per (group, slice).
template <int P>
__global__ void __launch_bounds__(256)
index_pool_kernel(const uint4* __restrict__ k_idx, int64_t n_groups, int groups_per_seq, int slices,
                  uint4* __restrict__ k_pool, PageMap pm) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= n_groups * slices) return;
  pool_group<P>(k_idx, gid / slices, groups_per_seq, slices, (int)(gid % slices), k_pool, pm);
}

// The groups holding rows ctx_len[b]-T .. ctx_len[b]-1 of each sequence b (at most `window`
// groups per sequence; rows outside [0, S_max) ignored): one thread per (b, group, slice).
template <int P>
__global__ void __launch_bounds__(256)
index_pool_tail_kernel(const uint4* __restrict__ k_idx, const int32_t* __restrict__ ctx_len, int B, int T,
                       int groups_per_seq, int window, int slices, uint4* __restrict__ k_pool, PageMap pm) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (int64_t)B * window * slices) return;
  const int sl = (int)(gid % slices);
  const int j = (int)((gid / slices) % window);
  const int b = (int)(gid / ((int64_t)slices * window));
  const int S_max = groups_per_seq * P;
  const int ctx = __ldg(ctx_len + b);
  const int lo = max(ctx - T, 0), hi = min(ctx, S_max);   // appended rows [ctx - T, ctx) in the cache
  if (hi <= lo) return;
  const int g = lo / P + j;
  if (g > (hi - 1) / P) return;
  pool_group<P>(k_idx, (int64_t)b * groups_per_seq + g, groups_per_seq, slices, sl, k_pool, pm);
}

}  // namespace

int launch_index_pool(const uint8_t* k_idx, int B, int S_max, int d_I, int pool, uint8_t* k_pool,
                      const PageMap& pm, cudaStream_t stream) {
  const int slices = d_I / 16;
  const int64_t n_groups = (int64_t)B * (S_max / pool);
  const int64_t n = n_groups * slices;
  if (n == 0) return DSA_OK;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  const uint4* src = reinterpret_cast<const uint4*>(k_idx);
  uint4* dst = reinterpret_cast<uint4*>(k_pool);
  switch (pool) {
    case 2: index_pool_kernel<2><<<(unsigned)blocks, threads, 0, stream>>>(src, n_groups, S_max / 2, slices, dst, pm); break;
    case 4: index_pool_kernel<4><<<(unsigned)blocks, threads, 0, stream>>>(src, n_groups, S_max / 4, slices, dst, pm); break;
    case 8: index_pool_kernel<8><<<(unsigned)blocks, threads, 0, stream>>>(src, n_groups, S_max / 8, slices, dst, pm); break;
    default: return DSA_ERR_UNSUPPORTED_SHAPE;
  }
  return check_launch();
}

int launch_index_pool_tail(const uint8_t* k_idx, const int32_t* ctx_len, int B, int T, int S_max, int d_I, int pool,
                           uint8_t* k_pool, const PageMap& pm, cudaStream_t stream) {
  const int slices = d_I / 16;
  const int window = (T - 1) / pool + 2;   // groups a run of T rows can touch
  const int64_t n = (int64_t)B * window * slices;
  if (n == 0) return DSA_OK;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  const uint4* src = reinterpret_cast<const uint4*>(k_idx);
  uint4* dst = reinterpret_cast<uint4*>(k_pool);
  switch (pool) {
    case 2: index_pool_tail_kernel<2><<<(unsigned)blocks, threads, 0, stream>>>(src, ctx_len, B, T, S_max / 2, window, slices, dst, pm); break;
    case 4: index_pool_tail_kernel<4><<<(unsigned)blocks, threads, 0, stream>>>(src, ctx_len, B, T, S_max / 4, window, slices, dst, pm); break;
    case 8: index_pool_tail_kernel<8><<<(unsigned)blocks, threads, 0, stream>>>(src, ctx_len, B, T, S_max / 8, window, slices, dst, pm); break;
    default: return DSA_ERR_UNSUPPORTED_SHAPE;
  }
  return check_launch();
}

unsigned int pool_take_status() {
  unsigned int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_pool_status, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_pool_status, &zero, sizeof(zero));
  return v;
}

}  // namespace dsa
