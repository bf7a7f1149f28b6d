// Sparse attention without a caller workspace: the split-key partials live in a fixed scratch
// array that this file owns, so the call allocates no device memory at any point.
//
// Who needs it: code that can neither allocate device memory nor hand the library a workspace
// buffer -- for instance an operator plugged into a runtime that owns all device memory and
// gives its operators no scratch, or a serving loop that must not call cudaMalloc once it is
// running (an allocation there can synchronise the device, or fail once the memory pool has
// claimed the GPU).  Such callers still pass their own inputs and outputs.
//
// Costs and limits, in plain terms:
//   * every GPU that loads the library keeps kScratchBytes (16 MiB) reserved until the process
//     exits, whether or not this entry point is ever called;
//   * all calls on a device share the one array, so two calls whose kernels overlap on that
//     device (different streams, or a second host thread) race on it: serialise them;
//   * a problem whose default key split would need more partials than the array holds runs at
//     the largest split count whose partials fit (one split needs no scratch at all), so no
//     problem is turned away for its size; it only spreads over fewer CTAs.
#include <atomic>

#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace {

// 16 MiB.  At 128 heads x 512 dv the partials take 2 x 128 x 513 x 4 B = 525 KB per query and
// split, so 31 decode queries fit at two splits and 15 at four.
constexpr size_t kScratchBytes = size_t(16) << 20;

// The scratch itself.  Host code must not use this name as a pointer: on the host it is only a
// stand-in for the symbol, so its device address is fetched with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up on the first call for
// that device (with the device current) and cached; nullptr on failure (error recorded).  Two
// threads making their first call at once both look it up and store the same address.  A
// cudaDeviceReset() of a device invalidates its cached address: do not call this entry point
// on a device after resetting it in the same process.
void* scratch_on_current_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidDevice);
    return nullptr;
  }
  void* p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      return nullptr;
    }
    g_scratch_ptr[dev].store(p, std::memory_order_relaxed);
  }
  return p;
}

}  // namespace
}  // namespace dsa

extern "C" {

size_t dsa_noalloc_scratch_bytes(void) { return dsa::kScratchBytes; }

int dsa_sparse_attn_noalloc(const uint16_t* q, const uint16_t* kv, const uint16_t* v, int64_t kv_row_stride,
                            int64_t kv_batch_stride, int64_t v_row_stride, int64_t v_batch_stride, int S_kv,
                            const int32_t* idx, int B, int T, int Hq, int d_qk, int d_v, int k, float sm_scale,
                            uint16_t* out, float* lse, const dsa_paging* paging, void* stream) {
  // The same argument and shape checks as dsa_sparse_attn come first (with the workspace
  // requirement waived), so a bad call reports the same status it would there.
  int st = dsa::check_sparse_attn(q, kv, v, kv_row_stride, kv_batch_stride, v_row_stride, v_batch_stride, S_kv,
                                  idx, B, T, Hq, d_qk, d_v, k, out, reinterpret_cast<const void*>(256),
                                  ~size_t(0), paging);
  if (st != DSA_OK || B == 0 || T == 0) return st;
  // The default key split, halved until its partials fit the scratch (one split needs none).
  int splits = dsa::attn_num_splits(B, T, Hq, k);
  while (splits > 1 && dsa::attn_workspace_bytes(B, T, Hq, d_v, k, splits) > dsa::kScratchBytes) splits /= 2;
  const size_t need = dsa::attn_workspace_bytes(B, T, Hq, d_v, k, splits);
  void* scratch = nullptr;
  if (need > 0) {
    scratch = dsa::scratch_on_current_device();
    if (scratch == nullptr) return DSA_ERR_CUDA;
  }
  // Every partial the split kernels write is written before it is read, so nothing in the
  // shared scratch has to start at zero and the previous call's contents are harmless.
  return dsa::launch_sparse_attn(q, kv, v, kv_row_stride, kv_batch_stride, v_row_stride, v_batch_stride, S_kv, idx,
                                 B, T, Hq, d_qk, d_v, k, sm_scale, out, lse, scratch, dsa::page_map(paging),
                                 static_cast<cudaStream_t>(stream), splits);
}

}  // extern "C"
