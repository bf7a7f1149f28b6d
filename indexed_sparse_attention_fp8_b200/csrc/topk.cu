// Stage 2 of DeepSeek Sparse Attention, fine selection ("GLM 5.2: How Four Co-Designed
// Mechanisms Beat Raw Scale", section "DeepSeek Sparse Attention"): keep the top-k keys of
// every query's indexer-score row.
//
// Keys are compared as order-preserving 32-bit integers (larger float -> larger unsigned key).
// topk_select_kernel serves one row with one CTA, or with a cluster of up to 8 CTAs when there
// are too few rows to fill the GPU (decode), each CTA taking a contiguous part of the row:
//   1. Threshold.  Blocks of 16 consecutive scores, one block every `sstride` keys (at most 8192
//      samples), go to the first CTA's shared memory; it finds the sample ranked r from the top,
//      r chosen so that about 1.5 k keys of the row are expected at or above it, and keeps the
//      top 22 bits of its key as the row's threshold tau (a lower bound of that sample).
//   2. Candidates.  One pass over the row appends every key >= tau, with its index, to the
//      CTA's candidate buffer: one warp ballot and prefix sum per 16 scores a lane loads, and one
//      shared-memory atomic per warp.
//   3. Selection.  The first CTA collects the cluster's candidates (distributed shared memory).
//      With at least k of them every key that a full sort would keep is among them (ties at the
//      k-th score included), so radix digit passes (11 + 11 + 10 bits) over the candidates find
//      the k-th key exactly; the winners are every candidate above it plus the lowest-indexed
//      candidates equal to it (the tie rule of a sort by (score desc, index asc)).
//   Rows whose threshold gave fewer than k or more than TS_CAP candidates (heavy ties, a
//   misleading sample) take the full-row path: digit passes over the row itself, copying the
//   pivot bucket to shared memory when it fits.  Either way the result is exact.
// The winners are written in ascending order (placed by a bucket scan, write_sorted) so the
// attention gathers walk the KV cache in address order, expanded to token ids when the scores
// were over IndexPool blocks.  The pass over a row runs behind TMA bulk prefetches into L2.
#include "common.cuh"
#include "kernels.h"

#include <climits>

namespace dsa {
namespace {

__device__ unsigned int g_merge_status;   // bit 1: a merge row whose candidates were out of range or too few

constexpr int TK_THREADS = 1024;     // the fused selection's kernels
constexpr int TK_KMAX = 2048;
constexpr int TK_BINS = 2048;
constexpr int TK_CAP = 8192;         // candidate buffer of the fused selection (keys, ids, tie ids)
constexpr int TK_DYN_SMEM = 3 * TK_CAP * 4;

constexpr int TS_THREADS = 512;      // topk_select_kernel
constexpr int TS_CAP = 4096;         // candidates of a row (and of each CTA of a row's cluster)
constexpr int TS_SBLK = 16;          // sampled scores come in blocks of 16 consecutive keys
constexpr int TS_NBLK = 512;         // at most 512 blocks: 8192 samples
constexpr int TS_MAX_CLUSTER = 8;
constexpr int TS_UNROLL = 8;         // float4 loads in flight per thread in a pass over a row
constexpr int TS_PREFETCH = 2;       // iterations of that pass (64 KB each) asked into L2 ahead
constexpr int TS_DYN_SMEM = 3 * TS_CAP * 4;   // keys, ids, tie ids; the samples reuse keys + ids
static_assert(TS_SBLK * TS_NBLK * 4 <= 2 * TS_CAP * 4, "samples fit the candidate key and id buffers");

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan of one int per thread across the block (blockDim.x == NT).
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* warp_buf, int* total) {
  constexpr int NW = NT / 32;
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
    int s = lane < NW ? warp_buf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NW) warp_buf[lane] = s;
  }
  __syncthreads();
  const int excl = x - v + (wid > 0 ? warp_buf[wid - 1] : 0);
  *total = warp_buf[NW - 1];
  __syncthreads();
  return excl;
}

// The bin holding the kk-th largest counted key (1 <= kk <= keys counted): each thread owns
// TK_BINS / NT adjacent bins, taken from the top bin down.  Writes {bin, keys above it, keys
// in it} to piv; every thread may read piv on return.
template <int NT>
__device__ __forceinline__ void pivot_bin(const uint32_t* hist, int kk, int* warp_buf, int* piv) {
  constexpr int BPT = TK_BINS / NT;
  const int top = TK_BINS - 1 - BPT * (int)threadIdx.x;
  int h[BPT], sum = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    h[i] = (int)hist[top - i];
    sum += h[i];
  }
  int total;
  int acc = block_excl_scan<NT>(sum, warp_buf, &total);
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    if (acc < kk && kk <= acc + h[i]) {
      piv[0] = top - i;
      piv[1] = acc;
      piv[2] = h[i];
    }
    acc += h[i];
  }
  __syncthreads();
}

// A slot in a shared list for every lane with `take` (-1 for the others): one atomic per warp.
// Called by whole warps.
__device__ __forceinline__ int warp_slot(int* counter, bool take) {
  const unsigned bal = __ballot_sync(0xffffffffu, take);
  if (bal == 0u) return -1;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(bal) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(counter, __popc(bal));
  base = __shfl_sync(0xffffffffu, base, leader);
  return take ? base + __popc(bal & ((1u << lane) - 1u)) : -1;
}

// One radix digit pass over keys[0, n) in shared memory: histogram of the `width`-bit digit at
// `shift` of the keys matching prefix under mask.
template <int NT>
__device__ __forceinline__ void digit_pass_smem(const uint32_t* keys, int n, uint32_t prefix, uint32_t mask,
                                                int shift, int width, uint32_t* hist) {
  for (int i = threadIdx.x; i < TK_BINS; i += NT) hist[i] = 0u;
  __syncthreads();
  const uint32_t dmask = (1u << width) - 1u;
  for (int j = threadIdx.x; j < n; j += NT) {
    const uint32_t key = keys[j];
    if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
  }
  __syncthreads();
}

// Calls fn(i, score) for every i in [0, n), 16-byte loads where the row allows.  Each thread
// issues TK_UNROLL loads before it consumes any, so a pass over a long row is not a chain of
// one-load round trips to L2.
constexpr int TK_UNROLL = 4;
template <int NT, typename F>
__device__ __forceinline__ void for_each_score(const float* __restrict__ row, int n, F&& fn) {
  const int n4 = n >> 2;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  for (int v0 = threadIdx.x; v0 < n4; v0 += TK_UNROLL * NT) {
    float4 f[TK_UNROLL];
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) {
      const int v = v0 + u * NT;
      if (v < n4) f[u] = __ldcs(r4 + v);
    }
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) {
      const int v = v0 + u * NT;
      if (v < n4) {
        fn(4 * v + 0, f[u].x);
        fn(4 * v + 1, f[u].y);
        fn(4 * v + 2, f[u].z);
        fn(4 * v + 3, f[u].w);
      }
    }
  }
  for (int i = 4 * n4 + threadIdx.x; i < n; i += NT) fn(i, __ldcs(row + i));
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

// Ascending bitonic sort of sel[0..n) in shared memory, padded to a power of two (the buffer
// holds that many).
template <int NT>
__device__ __forceinline__ void sort_ascending(int* sel, int n) {
  int P = 1;
  while (P < n) P <<= 1;
  for (int i = n + threadIdx.x; i < P; i += NT) sel[i] = INT_MAX;
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (P >> 1); i += NT) {
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

// Writes the k winners sel[0, k) -- distinct ids in [0, n_valid) -- to out in ascending order
// (expanded to token ids under IndexPool): the ids are bucketed by their place in [0, n_valid)
// (TK_BINS buckets of about n_valid / TK_BINS ids), the buckets laid out in order by a scan of
// their counts, and each id written after the ids of its own bucket that are smaller.
template <int NT>
__device__ __forceinline__ void write_sorted(const int* sel, int k, int n_valid, uint32_t* hist, int* tmp,
                                             int* warp_buf, int32_t* __restrict__ out, int pool, int pos) {
  // bucket of an id: floor(id * TK_BINS / n_valid) in float, non-decreasing in id (a bucket
  // order consistent with the id order is all the placement needs), clamped to the last bin
  const float scale = (float)TK_BINS / (float)n_valid;
  auto bucket = [&](int id) { return min(TK_BINS - 1, (int)((float)id * scale)); };
  for (int i = threadIdx.x; i < TK_BINS; i += NT) hist[i] = 0u;
  __syncthreads();
  for (int j = threadIdx.x; j < k; j += NT) atomicAdd(&hist[bucket(sel[j])], 1u);
  __syncthreads();
  constexpr int BPT = TK_BINS / NT;   // thread t scans bins BPT*t .. BPT*t+BPT-1
  uint32_t h[BPT];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    h[i] = hist[BPT * threadIdx.x + i];
    sum += (int)h[i];
  }
  int total;
  uint32_t acc = (uint32_t)block_excl_scan<NT>(sum, warp_buf, &total);
#pragma unroll
  for (int i = 0; i < BPT; ++i) {
    hist[BPT * threadIdx.x + i] = acc;   // first slot of the bucket
    acc += h[i];
  }
  __syncthreads();
  for (int j = threadIdx.x; j < k; j += NT) {
    const int id = sel[j];
    tmp[atomicAdd(&hist[bucket(id)], 1u)] = id;
  }
  __syncthreads();
  for (int j = threadIdx.x; j < k; j += NT) {   // bucket b now spans [hist[b-1], hist[b])
    const int id = tmp[j];
    const int b = bucket(id);
    const int s = b > 0 ? (int)hist[b - 1] : 0, e = (int)hist[b];
    int rank = 0;
    for (int x = s; x < e; ++x) rank += tmp[x] < id;
    write_expanded(out, s + rank, id, pool, pos);
  }
}

// Asks the TMA unit to bring row[a, b) (a a multiple of 4 floats) into L2, in pieces of up to
// 16 KB issued by the lanes of one warp.
__device__ __forceinline__ void prefetch_l2(const float* row, int a, int b, int lane) {
  const int n = ((b - a) >> 2) << 4;   // whole 16-byte pieces
  const char* p = reinterpret_cast<const char*>(row + a);
  for (int off = lane * 16384; off < n; off += 32 * 16384) {
    const int sz = min(16384, n - off);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p + off), "r"(sz) : "memory");
  }
}

// ---- cluster (distributed shared memory) helpers
__device__ __forceinline__ uint32_t cta_rank_in_cluster() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_addr(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
// (No memory clobber: the cluster barrier before these loads orders them, and leaving the
// compiler free to issue several before the first use keeps more of them in flight.)
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}
// Every thread of every CTA of the cluster: shared-memory writes before it are visible to the
// cluster after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Appends the keys of row[lo, hi) at or above the threshold to (ck, ci), counting them in *cnt
// (entries past TS_CAP are counted, not stored).  lo is a multiple of 4.  Called by the whole
// block.  The threshold is compared as a float, tau_f being the float whose order key is
// key_tau: the scores f >= tau_f are every non-NaN key >= key_tau, plus -0 when tau_f is +0 (the
// two compare equal), so they stay an upward-closed set in key order, which is what the exact
// selection on the candidates needs.  key_tau at or below -inf's key takes every key; a key_tau
// above +inf's (a NaN float) takes none, and the row then goes the full-row way.
template <int NT>
__device__ __forceinline__ void append_candidates(const float* __restrict__ row, int lo, int hi, uint32_t key_tau,
                                                  uint32_t* ck, int* ci, int* cnt) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int n4 = (hi - lo) >> 2;
  const float4* r4 = reinterpret_cast<const float4*>(row + lo);
  const bool take_all = key_tau <= order_key(-INFINITY);
  const float tau_f = take_all ? -INFINITY : __uint_as_float((key_tau & 0x80000000u) ? (key_tau & 0x7FFFFFFFu) : ~key_tau);
  auto pass = [&](float f) { return take_all || f >= tau_f; };
  constexpr int STEP = TS_UNROLL * NT;   // float4s per iteration
  for (int base = 0; base < n4; base += STEP) {   // the same trip count in every thread
    // keep the L2 prefetch TS_PREFETCH iterations ahead of the loads (the first ones were
    // asked for at the kernel's start)
    if (tid < 32) {
      const int a = base + TS_PREFETCH * STEP;
      if (a < n4) prefetch_l2(row, lo + 4 * a, lo + 4 * min(n4, a + STEP), lane);
    }
    float4 f[TS_UNROLL];
#pragma unroll
    for (int u = 0; u < TS_UNROLL; ++u) {
      const int v = base + u * NT + tid;
      f[u] = v < n4 ? __ldcs(r4 + v) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    int c = 0;
#pragma unroll
    for (int u = 0; u < TS_UNROLL; ++u) {
      if (base + u * NT + tid < n4)
        c += (int)pass(f[u].x) + (int)pass(f[u].y) + (int)pass(f[u].z) + (int)pass(f[u].w);
    }
    int x = c;   // inclusive prefix of the lanes' counts
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const int wtot = __shfl_sync(0xffffffffu, x, 31);
    if (wtot == 0) continue;   // the same in every lane
    int wbase = 0;
    if (lane == 31) wbase = atomicAdd(cnt, wtot);
    int slot = __shfl_sync(0xffffffffu, wbase, 31) + x - c;
    if (c == 0) continue;
#pragma unroll
    for (int u = 0; u < TS_UNROLL; ++u) {
      const int v = base + u * NT + tid;
      if (v >= n4) continue;
      const float e4[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (pass(e4[e])) {
          if (slot < TS_CAP) {
            ck[slot] = order_key(e4[e]);
            ci[slot] = lo + 4 * v + e;
          }
          ++slot;
        }
      }
    }
  }
  if (tid < 32) {   // the last (hi - lo) % 4 keys: warp 0
    const int i = lo + 4 * n4 + lane;
    const float f = i < hi ? __ldcs(row + i) : 0.f;
    const int slot = warp_slot(cnt, i < hi && pass(f));
    if (slot >= 0 && slot < TS_CAP) {
      ck[slot] = order_key(f);
      ci[slot] = i;
    }
  }
}

// The exact top-k of a row from its candidates (ck, ci)[0, ncand), k <= ncand <= TS_CAP, which
// hold every key of the row at or above the k-th key: winners into sel[0, k) (any order).
template <int NT>
__device__ __forceinline__ void select_from_candidates(const uint32_t* ck, const int* ci, int ncand, int k,
                                                       uint32_t* hist, int* sel, int* tie, int* warp_buf, int* piv,
                                                       int* counters) {
  // The candidates share every key bit above the highest one where two of them differ, so the
  // digits start there and spread the candidates over the histogram's bins.
  if (threadIdx.x == 0) { counters[0] = 0; counters[1] = -1; }
  __syncthreads();
  {
    uint32_t o = 0u, a = 0xFFFFFFFFu;
    for (int j = threadIdx.x; j < ncand; j += NT) {
      o |= ck[j];
      a &= ck[j];
    }
    o = __reduce_or_sync(0xffffffffu, o);
    a = __reduce_and_sync(0xffffffffu, a);
    if ((threadIdx.x & 31) == 0) {
      atomicOr(reinterpret_cast<unsigned*>(&counters[0]), o);
      atomicAnd(reinterpret_cast<unsigned*>(&counters[1]), a);
    }
  }
  __syncthreads();
  const uint32_t any = (uint32_t)counters[0], all = (uint32_t)counters[1];
  __syncthreads();
  const uint32_t diff = any ^ all;
  int shift = diff == 0u ? 0 : 32 - __clz(diff);    // bits [shift, 32) are common to all
  uint32_t mask = shift >= 32 ? 0u : ~((1u << shift) - 1u);
  if (diff == 0u) mask = 0xFFFFFFFFu;
  uint32_t prefix = all & mask;
  int kk = k, eq_count = ncand;
  while (eq_count != kk && shift > 0) {
    const int width = shift < 11 ? shift : 11;
    shift -= width;
    digit_pass_smem<NT>(ck, ncand, prefix, mask, shift, width, hist);
    pivot_bin<NT>(hist, kk, warp_buf, piv);
    kk -= piv[1];
    prefix |= (uint32_t)piv[0] << shift;
    mask |= ((1u << width) - 1u) << shift;
    eq_count = piv[2];
  }
  // every candidate above the prefix wins; of those equal to it, all or the kk lowest ids
  const bool take_all_eq = (eq_count == kk);
  if (threadIdx.x == 0) { counters[0] = 0; counters[1] = 0; }
  __syncthreads();
  for (int j0 = 0; j0 < ncand; j0 += NT) {
    const int j = j0 + (int)threadIdx.x;
    const uint32_t m = j < ncand ? (ck[j] & mask) : 0u;
    const int id = j < ncand ? ci[j] : 0;
    const int s_gt = warp_slot(&counters[0], j < ncand && m > prefix);
    if (s_gt >= 0) sel[s_gt] = id;
    const int s_eq = warp_slot(&counters[1], j < ncand && m == prefix);
    if (s_eq >= 0) tie[s_eq] = id;
  }
  __syncthreads();
  const int n_gt = counters[0], nties = counters[1];   // n_gt == k - kk
  if (!take_all_eq) sort_ascending<NT>(tie, nties);   // the lowest ids win
  __syncthreads();
  for (int j = threadIdx.x; j < kk; j += NT) sel[n_gt + j] = tie[j];
  __syncthreads();
}

// The full-row path: the exact top-k of row[0, n_valid) by digit passes over the row itself
// (the pivot bucket copied to shared memory when it fits).  Winners into sel[0, k).
template <int NT>
__device__ __forceinline__ void select_full_row(const float* __restrict__ row, int n_valid, int k, uint32_t* hist,
                                                int* sel, uint32_t* ck, int* ci, int* tie, int* warp_buf, int* piv,
                                                int* counters) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, mask = 0;
  int kk = k;          // winners still to find among keys matching `prefix` under `mask`
  int eq_count = 0;    // keys matching the final prefix
  const int shifts[3] = {21, 10, 0};
  auto digit_pass_row = [&](int shift) {
    for (int i = tid; i < TK_BINS; i += NT) hist[i] = 0u;
    __syncthreads();
    for_each_score<NT>(row, n_valid, [&](int, float f) {
      const uint32_t key = order_key(f);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (TK_BINS - 1)], 1u);
    });
    __syncthreads();
    pivot_bin<NT>(hist, kk, warp_buf, piv);
    kk -= piv[1];
    prefix |= (uint32_t)piv[0] << shift;
    mask |= (uint32_t)(TK_BINS - 1) << shift;
    eq_count = piv[2];
  };
  digit_pass_row(shifts[0]);
  if (eq_count != kk && eq_count <= TS_CAP) {
    // the pivot bucket fits in shared memory: one more pass over the row takes the keys above
    // it as winners and copies the bucket; the rest works on the copy
    const int n_gt_1 = k - kk;
    if (tid == 0) { counters[0] = 0; counters[1] = 0; }
    __syncthreads();
    for_each_score<NT>(row, n_valid, [&](int i, float f) {
      const uint32_t key = order_key(f);
      const uint32_t m = key & mask;
      if (m > prefix) {
        sel[atomicAdd(&counters[0], 1)] = i;
      } else if (m == prefix) {
        const int j = atomicAdd(&counters[1], 1);
        ck[j] = key;
        ci[j] = i;
      }
    });
    __syncthreads();
    const int ncand = counters[1];   // == eq_count
    __syncthreads();
    // the bucket's kk best, by the candidate selection, after the n_gt_1 winners found so far
    select_from_candidates<NT>(ck, ci, ncand, kk, hist, sel + n_gt_1, tie, warp_buf, piv, counters);
    return;
  }
  // the pivot bucket is taken whole, or too large to copy: digit passes over the row
  for (int p = 1; p < 3 && eq_count != kk; ++p) digit_pass_row(shifts[p]);
  // winners: all keys above the prefix, then kk of the keys equal to it
  if (tid == 0) { counters[0] = 0; counters[1] = 0; }
  __syncthreads();
  const int n_gt = k - kk;
  const bool take_all_eq = (eq_count == kk);
  for_each_score<NT>(row, n_valid, [&](int i, float f) {
    const uint32_t m = order_key(f) & mask;
    if (m > prefix) {
      sel[atomicAdd(&counters[0], 1)] = i;
    } else if (take_all_eq && m == prefix) {
      sel[n_gt + atomicAdd(&counters[1], 1)] = i;
    }
  });
  if (!take_all_eq) {
    // exact ties at the k-th key: the lowest indices win (ordered block compaction)
    int base = 0;
    for (int c0 = 0; c0 < n_valid && base < kk; c0 += NT) {
      const int i = c0 + tid;
      const int eq = (i < n_valid) && ((order_key(row[i]) & mask) == prefix);
      int total;
      const int r = block_excl_scan<NT>(eq, warp_buf, &total);
      if (eq && base + r < kk) sel[n_gt + base + r] = i;
      base += total;
    }
  }
  __syncthreads();
}

// One row per cluster of `csize` CTAs (csize = 1: one CTA; 2, 4 or 8: launched as a cluster).
__global__ void __launch_bounds__(TS_THREADS, 2)
topk_select_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ ctx_len,
                   int T, int S_max, int pool, int t_begin, int t_count, int k,
                   int32_t* __restrict__ idx_out, const int* __restrict__ row_flag, int csize) {
  constexpr int NT = TS_THREADS;
  __shared__ uint32_t hist[TK_BINS];
  __shared__ int sel[TK_KMAX];
  __shared__ int warp_buf[32];
  __shared__ int piv[3];
  __shared__ int counters[2];
  __shared__ int sh_cnt;                       // candidates this CTA found
  __shared__ uint32_t sh_tau;                  // the row's threshold (sent by the first CTA)
  __shared__ int sh_off[TS_MAX_CLUSTER + 1];   // first CTA: where each CTA's candidates go
  extern __shared__ uint32_t cand_smem[];
  uint32_t* ck = cand_smem;                                   // candidate keys
  int* ci = reinterpret_cast<int*>(cand_smem + TS_CAP);        // their row indices
  int* tie = reinterpret_cast<int*>(cand_smem + 2 * TS_CAP);   // ids tied at the pivot
  uint32_t* samp = cand_smem;                                  // the samples (before the candidates)

  const int tid = threadIdx.x;
  const int crank = csize > 1 ? (int)cta_rank_in_cluster() : 0;
  const int row_id = blockIdx.x / csize;
  // Every CTA of a cluster serves the same row, so all of them leave here together or none.
  if (row_flag != nullptr && row_flag[row_id] == 0) return;   // only the flagged rows (repair pass)
  const int b = row_id / t_count;
  const int t = t_begin + row_id % t_count;
  const int pos = ctx_len[b] - T + t;
  const int n_valid = pos < 0 ? 0 : min(S_max, pos / pool + 1);
  int32_t* out = idx_out + ((int64_t)b * T + t) * (int64_t)k * pool;
  if (n_valid <= k) {  // every visible key is selected
    if (crank == 0)
      for (int i = tid; i < k; i += NT) write_expanded(out, i, i < n_valid ? i : -1, pool, pos);
    return;
  }
  const float* row = scores + (int64_t)row_id * ld;
  const int part = ((n_valid + csize - 1) / csize + 15) & ~15;   // this CTA's keys: [lo, hi)
  const int lo = min(n_valid, crank * part), hi = min(n_valid, lo + part);
  // the first iterations of the pass over this part come into L2 while the threshold is found
  if (tid < 32) prefetch_l2(row, lo, min(hi, lo + 4 * TS_PREFETCH * TS_UNROLL * NT), tid);

  // ---- 1. threshold (every key is a candidate when the row fits the buffer)
  uint32_t key_tau = 0u;
  if (n_valid > TS_CAP) {
    const int sstride = TS_SBLK * ((n_valid + TS_SBLK * TS_NBLK - 1) / (TS_SBLK * TS_NBLK));
    const int nblk = (n_valid + sstride - 1) / sstride;
    // block q (keys q*sstride .. +15, zeros past the row's end) is loaded by the CTA whose part
    // holds its first key, into the first CTA's sample buffer
    const uint32_t samp0 = smem_u32(samp);
    const uint32_t dst = csize > 1 ? cluster_addr(samp0, 0) : samp0;
    const int q_lo = (lo + sstride - 1) / sstride, q_hi = (hi + sstride - 1) / sstride;
    static_assert(4 * TS_NBLK <= 4 * NT, "a thread loads at most four 16-byte pieces of samples");
    float4 f[4];   // every load in flight before the first store
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = 4 * q_lo + tid + u * NT;
      const int p = (v >> 2) * sstride + (v & 3) * 4;
      f[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (v < 4 * q_hi) {
        if (p + 3 < n_valid) {
          f[u] = __ldcs(reinterpret_cast<const float4*>(row + p));
        } else {
          if (p + 0 < n_valid) f[u].x = __ldcs(row + p + 0);
          if (p + 1 < n_valid) f[u].y = __ldcs(row + p + 1);
          if (p + 2 < n_valid) f[u].z = __ldcs(row + p + 2);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = 4 * q_lo + tid + u * NT;
      const int p = (v >> 2) * sstride + (v & 3) * 4;
      if (v < 4 * q_hi)   // keys past the row's end become 0, below every score's key
        st_cluster_v4(dst + 16u * v, p + 0 < n_valid ? order_key(f[u].x) : 0u, p + 1 < n_valid ? order_key(f[u].y) : 0u,
                      p + 2 < n_valid ? order_key(f[u].z) : 0u, p + 3 < n_valid ? order_key(f[u].w) : 0u);
    }
    if (csize > 1) cluster_sync_all(); else __syncthreads();
    if (crank == 0) {
      // the sample ranked r from the top, r for about 1.5 k candidates; its top 22 bits
      const int ns = (nblk - 1) * TS_SBLK + min(TS_SBLK, n_valid - (nblk - 1) * sstride);
      const int target = 3 * k / 2;
      const int r = max(1, min(ns, (int)(((int64_t)target * ns + n_valid - 1) / n_valid)));
      uint32_t prefix = 0u, mask = 0u;
      int kk = r;
      for (int p = 0; p < 2; ++p) {
        const int shift = p == 0 ? 21 : 10;
        digit_pass_smem<NT>(samp, nblk * TS_SBLK, prefix, mask, shift, 11, hist);
        pivot_bin<NT>(hist, kk, warp_buf, piv);
        kk -= piv[1];
        prefix |= (uint32_t)piv[0] << shift;
        mask |= (uint32_t)(TK_BINS - 1) << shift;
      }
      key_tau = prefix;
      if (csize > 1 && tid < csize) st_cluster_u32(cluster_addr(smem_u32(&sh_tau), (uint32_t)tid), key_tau);
    }
    if (csize > 1) {
      cluster_sync_all();   // the threshold is delivered; the sample buffer is free again
      key_tau = sh_tau;
    } else {
      __syncthreads();
    }
  }

  // ---- 2. candidates of this CTA's part
  if (tid == 0) sh_cnt = 0;
  __syncthreads();
  append_candidates<NT>(row, lo, hi, key_tau, ck, ci, &sh_cnt);
  __syncthreads();

  // ---- 3. the first CTA collects the cluster's candidates
  int ncand = sh_cnt;
  bool ok = false;
  if (csize > 1) {
    cluster_sync_all();   // every CTA's candidates and count are final
    if (crank == 0) {
      if (tid == 0) {
        int tot = 0;
        for (int c = 0; c < csize; ++c) {
          const int n = c == 0 ? sh_cnt : (int)ld_cluster_u32(cluster_addr(smem_u32(&sh_cnt), (uint32_t)c));
          sh_off[c] = n;   // the counts, then turned into offsets below
          tot += n;
        }
        int acc = 0;
        for (int c = 0; c < csize; ++c) {
          const int n = sh_off[c];
          sh_off[c] = acc;
          acc += n;
        }
        sh_off[csize] = acc;
      }
      __syncthreads();
      ncand = sh_off[csize];
      ok = ncand >= k && ncand <= TS_CAP;   // then no CTA's count passed TS_CAP either
      if (ok) {
        for (int c = 1; c < csize; ++c) {
          const int o = sh_off[c], n = sh_off[c + 1] - o;
          const uint32_t rk = cluster_addr(smem_u32(ck), (uint32_t)c);
          const uint32_t ri = cluster_addr(smem_u32(ci), (uint32_t)c);
          for (int j0 = 0; j0 < n; j0 += 4 * NT) {
            uint32_t kv[4], iv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = j0 + u * NT + tid;
              if (j < n) {
                kv[u] = ld_cluster_u32(rk + 4u * j);
                iv[u] = ld_cluster_u32(ri + 4u * j);
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = j0 + u * NT + tid;
              if (j < n) {
                ck[o + j] = kv[u];
                ci[o + j] = (int)iv[u];
              }
            }
          }
        }
      }
    }
    cluster_sync_all();   // the other CTAs' buffers are no longer read
    if (crank != 0) return;
  } else {
    ok = ncand >= k && ncand <= TS_CAP;
  }
  __syncthreads();

  if (ok) {
    select_from_candidates<NT>(ck, ci, ncand, k, hist, sel, tie, warp_buf, piv, counters);
  } else {
    select_full_row<NT>(row, n_valid, k, hist, sel, ck, ci, tie, warp_buf, piv, counters);
  }

  // ---- the k winners in ascending order
  write_sorted<NT>(sel, k, n_valid, hist, tie, warp_buf, out, pool, pos);
}

// Merge of per-shard selections (context parallelism): row r of part p holds that shard's
// selected keys as (score, global key id), ids ascending, -1 padding.  The exact top-k of the
// union: every key a full sort over the whole row keeps is in its shard's selection (a shard
// has at most k of them, and its own top-k keeps its lowest-indexed ties, which are the
// lowest global ids), so the candidate selection over the union gives the same ids.
__global__ void __launch_bounds__(TS_THREADS, 1)
topk_merge_kernel(const float* __restrict__ cand_score, const int32_t* __restrict__ cand_id, int n_parts,
                  int64_t part_stride, int kc, const int32_t* __restrict__ ctx_len, int T, int S_total, int t_begin,
                  int t_count, int k, int32_t* __restrict__ idx_out) {
  constexpr int NT = TS_THREADS;
  __shared__ uint32_t hist[TK_BINS];
  __shared__ int sel[TK_KMAX];
  __shared__ int warp_buf[32];
  __shared__ int piv[3];
  __shared__ int counters[2];
  __shared__ int sh_cnt;
  extern __shared__ uint32_t cand_smem[];
  const int cap = n_parts * kc;
  uint32_t* ck = cand_smem;
  int* ci = reinterpret_cast<int*>(cand_smem + cap);
  int* tie = reinterpret_cast<int*>(cand_smem + 2 * cap);
  const int tid = threadIdx.x;
  const int row_id = blockIdx.x;
  const int b = row_id / t_count;
  const int t = t_begin + row_id % t_count;
  const int pos = ctx_len[b] - T + t;
  const int n_valid = pos < 0 ? 0 : min(S_total, pos + 1);
  int32_t* out = idx_out + ((int64_t)b * T + t) * (int64_t)k;
  if (n_valid <= k) {
    for (int i = tid; i < k; i += NT) out[i] = i < n_valid ? i : -1;
    return;
  }
  if (tid == 0) sh_cnt = 0;
  __syncthreads();
  for (int e0 = 0; e0 < cap; e0 += NT) {   // the same trip count in every lane of a warp
    const int e = e0 + tid;
    const int p = e / kc, j = e % kc;
    int id = -1;
    float f = 0.f;
    if (e < cap) {
      const int64_t at = (int64_t)p * part_stride + (int64_t)row_id * kc + j;
      id = __ldg(cand_id + at);
      f = __ldg(cand_score + at);
      if (id >= n_valid) {   // not a key this row sees: skipped (the ordered write needs ids < n_valid)
        atomicOr(&g_merge_status, 2u);
        id = -1;
      }
    }
    const int slot = warp_slot(&sh_cnt, id >= 0);
    if (slot >= 0) {
      ck[slot] = order_key(f);
      ci[slot] = id;
    }
  }
  __syncthreads();
  const int ncand = sh_cnt;   // >= k: each shard kept min(k, its visible keys)
  __syncthreads();
  if (ncand < k) {   // only when the candidates are not shard selections of this row: no result
    if (tid == 0) atomicOr(&g_merge_status, 2u);
    for (int i = tid; i < k; i += NT) out[i] = -1;
    return;
  }
  select_from_candidates<NT>(ck, ci, ncand, k, hist, sel, tie, warp_buf, piv, counters);
  write_sorted<NT>(sel, k, n_valid, hist, tie, warp_buf, out, 1, pos);
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
    const int excl = block_excl_scan<TK_THREADS>(h0 + h1, warp_buf, &total);
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
// the repair pass (full score row + topk_select_kernel).
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
    const int excl = block_excl_scan<TK_THREADS>(h0 + h1, warp_buf, &total);
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
  if (!take_all_eq) sort_ascending<TK_THREADS>(tie, nties);   // the lowest ids win
  __syncthreads();
  for (int j = tid; j < kk; j += TK_THREADS) sel[n_gt + j] = tie[j];
  __syncthreads();
  sort_ascending<TK_THREADS>(sel, k);
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
    cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TS_DYN_SMEM);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  // Few rows (decode): a cluster of CTAs per row, as many as fill two CTAs per SM, each taking
  // at least 8192 keys of the row.
  int csize = 1;
  const int slots = 2 * num_sms();
  while (csize < TS_MAX_CLUSTER && rows * csize * 2 <= slots && S_max / (csize * 2) >= 8192) csize *= 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * csize));
  cfg.blockDim = dim3(TS_THREADS);
  cfg.dynamicSmemBytes = TS_DYN_SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, topk_select_kernel, scores, ld, ctx_len, T, S_max, pool, t_begin,
                                           t_count, k, idx, row_flag, csize);
  if (e != cudaSuccess) {
    count_launch();
    set_cuda_error(e);
    return DSA_ERR_CUDA;
  }
  return check_launch();
}

unsigned int merge_take_status() {
  unsigned int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_merge_status, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_merge_status, &zero, sizeof(zero));
  return v;
}

int launch_topk_merge(const float* cand_score, const int32_t* cand_id, int n_parts, int64_t part_stride, int kc,
                      const int32_t* ctx_len, int B, int T, int S_total, int t_begin, int t_count, int k, int32_t* idx,
                      cudaStream_t stream) {
  if (B * t_count == 0) return DSA_OK;
  const int cap = n_parts * kc;
  int cap2 = 1;
  while (cap2 < cap) cap2 <<= 1;   // the tie list is sorted in a power-of-two buffer
  const int smem = (2 * cap + cap2) * 4;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 3 * kMergeMaxCand * 4);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  topk_merge_kernel<<<B * t_count, TS_THREADS, smem, stream>>>(cand_score, cand_id, n_parts, part_stride, kc, ctx_len,
                                                               T, S_total, t_begin, t_count, k, idx);
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
