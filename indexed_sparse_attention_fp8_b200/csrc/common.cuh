// Shared plumbing of the DSA library: status codes, launch accounting, small device helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// Records the CUDA error of a failed launch for dsa_last_cuda_error() (thread-local).
void set_cuda_error(cudaError_t e);
// Counts a kernel launch enqueued by the library (thread-local running counter).
void count_launch();

// Checks the launch that was just enqueued; returns DSA_ERR_CUDA on failure.
inline int check_launch() {
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms();  // SM count of the current device (cached per device)

// Page map of a paged cache (dsa_paging in dsa.h); bt == nullptr means the cache is contiguous
// per sequence.  Passed to kernels by value.
struct PageMap {
  const int32_t* bt;   // device [B, pps] page ids
  int shift;           // log2(page_size)
  int pps;             // pages per sequence
  int num_pages;       // pages in the pool
};

inline PageMap page_map(const dsa_paging* p) {
  PageMap m{nullptr, 0, 0, 0};
  if (p != nullptr && p->block_table != nullptr) {
    m.bt = p->block_table;
    while ((1 << m.shift) < p->page_size) ++m.shift;
    m.pps = p->pages_per_seq;
    m.num_pages = p->num_pages;
  }
  return m;
}

// Physical row of logical row s of sequence b in a paged pool, or -1 when the page id in the
// block table lies outside [0, num_pages).
__device__ __forceinline__ int paged_row(const PageMap& m, int b, int s) {
  const int page = __ldg(m.bt + (int64_t)b * m.pps + (s >> m.shift));
  return (page >= 0 && page < m.num_pages) ? (page << m.shift) | (s & ((1 << m.shift) - 1)) : -1;
}

// ---------------------------------------------------------------- device helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; src_bytes < 16 zero-fills the rest (0 = all zeros).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

}  // namespace dsa
