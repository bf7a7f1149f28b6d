// IndexPool ("GLM-5.3-Flash hybrid sparse-linear attention with IndexPool", section "What
// changed"): four consecutive indexer keys pooled into one key, so the indexer scores a
// quarter as many rows.  The pooled key is the fp32 mean ((k0 + k1) + (k2 + k3)) * 0.25 of
// the decoded e4m3 keys, requantised to e4m3 round-to-nearest-even with saturation.
//
// HBM-bound streaming: each thread reads one 16-byte slice (16 dims) of the 4 source rows
// and writes one 16-byte slice of the pooled row.
#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace {

__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));   // e4m3 -> f16 is exact
}

__global__ void __launch_bounds__(256)
index_pool_kernel(const uint4* __restrict__ k_idx, int64_t n_groups, int slices,
                  uint4* __restrict__ k_pool) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= n_groups * slices) return;
  const int64_t g = gid / slices;
  const int sl = (int)(gid % slices);
  uint4 src[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) src[r] = __ldcs(k_idx + (4 * g + r) * slices + sl);
  uint32_t outw[4];
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    uint32_t packed = 0;
#pragma unroll
    for (int hpair = 0; hpair < 2; ++hpair) {
      float2 v[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint32_t word = (&src[r].x)[wd];
        v[r] = e4m3x2_to_float2(static_cast<uint16_t>(word >> (16 * hpair)));
      }
      float2 m;
      m.x = ((v[0].x + v[1].x) + (v[2].x + v[3].x)) * 0.25f;
      m.y = ((v[0].y + v[1].y) + (v[2].y + v[3].y)) * 0.25f;
      const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(m, __NV_SATFINITE, __NV_E4M3);
      packed |= static_cast<uint32_t>(q) << (16 * hpair);
    }
    outw[wd] = packed;
  }
  k_pool[gid] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
}

}  // namespace

int launch_index_pool(const uint8_t* k_idx, int B, int S_max, int d_I, uint8_t* k_pool,
                      cudaStream_t stream) {
  const int slices = d_I / 16;
  const int64_t n_groups = (int64_t)B * (S_max / 4);
  const int64_t n = n_groups * slices;
  if (n == 0) return DSA_OK;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  index_pool_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
      reinterpret_cast<const uint4*>(k_idx), n_groups, slices, reinterpret_cast<uint4*>(k_pool));
  return check_launch();
}

}  // namespace dsa
