// Context parallelism (keys sharded over ranks): the two small kernels around the exchange.
// Each rank selects from its own contiguous key shard [s0, s0 + s_len) with the ordinary indexer
// and top-k; gather_selected_kernel turns those local selections into (score, global id)
// candidates for the exchange, and after the merge idx_localize_kernel maps the group's global
// selection back onto the rank's shard so its attention reads only keys it holds.
#include "common.cuh"
#include "kernels.h"

#include <cmath>

namespace dsa {
namespace {

__device__ unsigned int g_cp_status;   // bit 1: an id at or beyond its score row's width

// One thread per selected slot: rows (b, t_begin + r) of the [B, T, k] id array.  An id past
// the score row's ld entries is skipped like a -1 and flagged, so nothing outside the score
// rows is read.
__global__ void gather_selected_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ idx,
                                       int T, int t_begin, int t_count, int k, int id_offset,
                                       float* __restrict__ cand_score, int32_t* __restrict__ cand_id, int64_t n) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const int64_t row = e / k;          // (b, r) over B * t_count rows
  const int j = (int)(e % k);
  const int64_t b = row / t_count, r = row % t_count;
  int id = __ldg(idx + (b * T + t_begin + r) * k + j);
  if (id >= ld) {
    atomicOr(&g_cp_status, 2u);
    id = -1;
  }
  cand_id[e] = id < 0 ? -1 : id + id_offset;
  cand_score[e] = id < 0 ? -INFINITY : __ldg(scores + row * ld + id);
}

__global__ void idx_localize_kernel(const int32_t* __restrict__ idx, int64_t n, int s0, int s_len,
                                    int32_t* __restrict__ out) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const int id = __ldg(idx + e);
  out[e] = (id >= s0 && id - s0 < s_len) ? id - s0 : -1;
}

}  // namespace

int launch_gather_selected(const float* scores, int64_t ld, const int32_t* idx, int B, int T, int t_begin,
                           int t_count, int k, int id_offset, float* cand_score, int32_t* cand_id, cudaStream_t stream) {
  const int64_t n = (int64_t)B * t_count * k;
  if (n == 0) return DSA_OK;
  gather_selected_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(scores, ld, idx, T, t_begin, t_count, k,
                                                                          id_offset, cand_score, cand_id, n);
  return check_launch();
}

unsigned int cp_take_status() {
  unsigned int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_cp_status, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_cp_status, &zero, sizeof(zero));
  return v;
}

int launch_idx_localize(const int32_t* idx, int64_t n, int s0, int s_len, int32_t* out, cudaStream_t stream) {
  if (n == 0) return DSA_OK;
  idx_localize_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(idx, n, s0, s_len, out);
  return check_launch();
}

}  // namespace dsa
