// Lightning indexer, CUDA-core reference kernel (Stage 1 of "DeepSeek Sparse Attention",
// "GLM 5.2: How Four Co-Designed Mechanisms Beat Raw Scale"):
//   I[t,s] = sum_j w[t,j] * max(0, q_idx[t,j,:] . k_idx[s,:])
// One thread per key, one CTA per (128-key tile, query).  The query's e4m3 heads are decoded
// to fp32 in shared memory; each thread streams its key row, decodes it and accumulates the
// H_I dot products in fp32 (e4m3 products are exact in fp32).
#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace {

constexpr int SIMT_TILE = 128;

__device__ __forceinline__ void decode16(uint4 raw, float* f) {
  const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw hr =
          __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(wds[i] >> (16 * h)), __NV_E4M3);
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      f[4 * i + 2 * h] = v.x;
      f[4 * i + 2 * h + 1] = v.y;
    }
  }
}

template <int H, int D>
__global__ void __launch_bounds__(SIMT_TILE)
index_scores_simt_kernel(const uint8_t* __restrict__ q_idx, const float* __restrict__ w,
                         const uint8_t* __restrict__ k_idx, const int32_t* __restrict__ ctx_len,
                         int T, int S_max, int pool, int t_begin, int t_count,
                         float* __restrict__ scores, int64_t ld) {
  __shared__ float qf[H][D];
  __shared__ float wf[H];
  const int b = blockIdx.z, tq = blockIdx.x, t = t_begin + tq;
  const int pos = ctx_len[b] - T + t;
  const int n_valid = pos < 0 ? 0 : min(S_max, pos / pool + 1);
  const int tile0 = blockIdx.y * SIMT_TILE;
  if (tile0 >= n_valid) return;  // block-uniform: tiles past the last visible key are skipped

  const uint8_t* qrow = q_idx + (((int64_t)b * T + t) * H) * D;
  for (int i = threadIdx.x; i < H * D / 16; i += SIMT_TILE) {
    float f[16];
    decode16(reinterpret_cast<const uint4*>(qrow)[i], f);
#pragma unroll
    for (int e = 0; e < 16; ++e) (&qf[0][0])[16 * i + e] = f[e];
  }
  for (int j = threadIdx.x; j < H; j += SIMT_TILE) wf[j] = w[((int64_t)b * T + t) * H + j];
  __syncthreads();

  const int s = tile0 + threadIdx.x;
  if (s >= S_max) return;
  float* out = scores + ((int64_t)b * t_count + tq) * ld;
  if (s >= n_valid) {
    out[s] = -INFINITY;
    return;
  }
  const uint4* krow = reinterpret_cast<const uint4*>(k_idx + ((int64_t)b * S_max + s) * D);
  float dot[H];
#pragma unroll
  for (int j = 0; j < H; ++j) dot[j] = 0.f;
#pragma unroll
  for (int c = 0; c < D / 16; ++c) {
    float kf[16];
    decode16(__ldg(krow + c), kf);
#pragma unroll
    for (int j = 0; j < H; ++j) {
#pragma unroll
      for (int e = 0; e < 16; ++e) dot[j] = fmaf(qf[j][16 * c + e], kf[e], dot[j]);
    }
  }
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < H; ++j) acc = fmaf(wf[j], fmaxf(dot[j], 0.f), acc);
  out[s] = acc;
}

}  // namespace

int launch_index_scores(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                        const int32_t* ctx_len, int B, int T, int S_max, int H_I, int d_I, int pool,
                        int t_begin, int t_count, float* scores, int64_t ld, cudaStream_t stream) {
  if (B == 0 || t_count == 0 || S_max == 0) return DSA_OK;
  dim3 grid(t_count, (S_max + SIMT_TILE - 1) / SIMT_TILE, B);
  if (H_I == 64 && d_I == 128) {
    index_scores_simt_kernel<64, 128><<<grid, SIMT_TILE, 0, stream>>>(
        q_idx, w, k_idx, ctx_len, T, S_max, pool, t_begin, t_count, scores, ld);
  } else if (H_I == 4 && d_I == 64) {
    index_scores_simt_kernel<4, 64><<<grid, SIMT_TILE, 0, stream>>>(
        q_idx, w, k_idx, ctx_len, T, S_max, pool, t_begin, t_count, scores, ld);
  } else {
    return DSA_ERR_UNSUPPORTED_SHAPE;
  }
  return check_launch();
}

}  // namespace dsa
