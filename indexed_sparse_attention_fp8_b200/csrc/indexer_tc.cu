// Lightning indexer on the 5th-generation tensor cores (Stage 1 of "DeepSeek Sparse
// Attention", "GLM 5.2: How Four Co-Designed Mechanisms Beat Raw Scale"; FP8 per the
// twiscan.com IndexShare post):
//
//     I[t,s] = sum_j w[t,j] * max(0, q_idx[t,j,:] . k_idx[s,:])
//
// GEMM view: A = 128 keys x d_I (e4m3, K-major rows of the key cache), B = QB queries x H_I
// heads = N rows x d_I (e4m3, the q_idx rows of QB consecutive queries), D = A B^T in TMEM
// (128 lanes = keys, N fp32 columns = (query, head)).  Each TMEM lane holds every head of
// every query of the block for one key, so the weighted ReLU reduction over heads runs in
// one thread, and the per-head logits never leave the SM.
//
// Persistent kernel, one CTA per SM (two for the one-query decode shape), warp-specialised:
//   warp 0      TMA producer: key tiles (ring of C::NA stages), query blocks + head weights
//               (2 stages), all through mbarrier transaction counts
//   warp 1      TMEM owner and MMA issuer: d_I/32 tcgen05.mma (kind::f8f6f4, M=128, N) per
//               key tile into one of two TMEM accumulators
//   warps 2..9  epilogue: tcgen05.ld the accumulator, w * relu, sum over heads, causal mask,
//               coalesced fp32 stores of the score rows
// Work items are (sequence, block of QB queries, chunk of KC key tiles); key tiles past the
// causal frontier of the block's last query are never loaded or multiplied.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace dsa {
namespace {

using namespace tc;

constexpr int KTILE = 128;        // keys per tile (MMA M)
constexpr int KC = 32;            // key tiles per work item
constexpr int NUM_THREADS = 320;  // 10 warps

template <int H, int D, int QB>
struct IdxCfg {
  // Decode (one query per block, N = 64): only the 4 epilogue warps of one column half have work,
  // one per SM sub-partition, so two CTAs share each SM (4-stage key rings, 96 registers) and
  // twice the epilogue warps hide each other's TMEM-load and reduction latency.
  static constexpr int NA = QB == 1 ? 4 : 6;       // key-tile stages
  static constexpr int CTAS_PER_SM = QB == 1 ? 2 : 1;
  static constexpr int N = QB * H;                 // MMA N: (query, head) columns
  static constexpr int A_BYTES = KTILE * D;        // one key tile
  static constexpr int B_BYTES = N * D;            // one query block
  static constexpr int W_BYTES = QB * H * 4;       // head weights of the block
  static constexpr int HALVES = N >= 128 ? 2 : 1;  // epilogue column halves
  static constexpr int COLS = N / HALVES;          // columns per epilogue warp
  static constexpr int CHUNKS = COLS / 32;
  static constexpr int QPH = COLS / H > 0 ? COLS / H : 1;  // queries per epilogue warp
  static constexpr uint32_t TMEM_COLS = 2 * N <= 32 ? 32 : (2 * N <= 64 ? 64 : (2 * N <= 128 ? 128 : (2 * N <= 256 ? 256 : 512)));
  static constexpr uint32_t SBO = 8 * D;           // 8-row group stride of a swizzled tile
  static constexpr uint32_t LAYOUT = D == 128 ? kLayoutSw128 : kLayoutSw64;
  static constexpr uint32_t IDESC = instr_desc(128, N, 0);
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NA * A_BYTES;
  static constexpr int OFF_W = OFF_B + 2 * B_BYTES;
  static constexpr int OFF_BAR = OFF_W + 2 * W_BYTES;
  static constexpr int NBAR = 2 * NA + 9;           // + the MMA drain barrier
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // fused selection (64-head shape): per epilogue warp and query, a staging buffer of CB
  // candidates, so the global slots are reserved with one atomic per flush, not per tile
  static constexpr int CB = 64;
  static constexpr int OFF_CBUF = (OFF_MISC + 16 + 15) / 16 * 16;
  static constexpr int CBUF_BYTES = H == 64 ? 8 * QPH * CB * 8 : 0;
  static constexpr int SMEM = OFF_CBUF + CBUF_BYTES + 1024;  // + alignment slack
  static_assert(D == 128 || D == 64, "row = one swizzle atom");
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N");
  static_assert(COLS % 32 == 0 && (COLS % H == 0 || H % COLS == 0), "epilogue split");
  static_assert(H <= COLS, "a query's heads stay in one warp");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "tile alignment");
};

struct ItemGeom {
  int b, t0, nq, kt0, kt1;
};

// Decodes work item `it` and returns false when it holds no visible key tile, or (with a row
// filter) none of its queries is flagged.
__device__ __forceinline__ bool item_geom(int it, int QB, int nqb, int nkc, int T, int t_begin, int t_count,
                                          int S_max, int pool, const int32_t* __restrict__ ctx_len, ItemGeom& g,
                                          const int* __restrict__ row_flag) {
  const int kc = it % nkc;
  const int r = it / nkc;
  const int qb = r % nqb;
  g.b = r / nqb;
  g.t0 = t_begin + qb * QB;
  g.nq = min(QB, t_begin + t_count - g.t0);
  if (row_flag != nullptr) {
    bool any = false;
    for (int q = 0; q < g.nq; ++q) any |= __ldg(row_flag + (int64_t)g.b * t_count + (g.t0 - t_begin) + q) != 0;
    if (!any) return false;
  }
  const int pos_last = __ldg(ctx_len + g.b) - T + g.t0 + g.nq - 1;
  if (pos_last < 0) return false;
  const int n_valid = min(S_max, pos_last / pool + 1);
  const int ntiles = (n_valid + KTILE - 1) / KTILE;
  g.kt0 = kc * KC;
  g.kt1 = min(g.kt0 + KC, ntiles);
  return g.kt0 < g.kt1;
}

// Candidate append of the fused selection: every lane of the warp calls it for the same query
// (the lanes hold different keys); the keys that pass (visible, score >= the query's threshold)
// take consecutive slots of the query's candidate row with one atomic per warp.  Slots past the
// buffer are not written; the count keeps growing, so the top-k sees the overflow.
__device__ __forceinline__ void cand_append(bool pass, float val, int s, int* __restrict__ cnt_row,
                                            float2* __restrict__ cand_row, int cap) {
  const unsigned m = __ballot_sync(0xffffffffu, pass);
  if (m == 0u) return;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(m) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(cnt_row, __popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (pass) {
    const int slot = base + __popc(m & ((1u << lane) - 1u));
    if (slot < cap) cand_row[slot] = make_float2(val, __int_as_float(s));
  }
}

// CAND = false: the score rows are stored (masked entries -inf).  CAND = true (fused
// selection): nothing is stored but the candidates of each query, the visible keys whose score
// reaches tau[row]; `cnt` counts them per row.  row_flag (optional): only the work items
// holding a flagged query run.
template <int H, int D, int QB, bool CAND>
__global__ void __launch_bounds__(NUM_THREADS, IdxCfg<H, D, QB>::CTAS_PER_SM)
index_scores_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                       const float* __restrict__ w, const int32_t* __restrict__ ctx_len, int B, int T, int S_max,
                       int pool, int t_begin, int t_count, float* __restrict__ scores, int64_t ld, PageMap pm,
                       const float* __restrict__ tau, float2* __restrict__ cand, int* __restrict__ cnt, int cap,
                       const int* __restrict__ row_flag) {
  const uint64_t wlim = wait_limit();   // the bounded waits' time limit, read once
  using C = IdxCfg<H, D, QB>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - sraw);
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto a_full = [&](int s) { return bar0 + 8u * s; };
  auto a_empty = [&](int s) { return bar0 + 8u * (C::NA + s); };
  auto b_full = [&](int s) { return bar0 + 8u * (2 * C::NA + s); };
  auto b_empty = [&](int s) { return bar0 + 8u * (2 * C::NA + 2 + s); };
  auto acc_full = [&](int s) { return bar0 + 8u * (2 * C::NA + 4 + s); };
  auto acc_empty = [&](int s) { return bar0 + 8u * (2 * C::NA + 6 + s); };
  const uint32_t mma_drain = bar0 + 8u * (2 * C::NA + 8);   // completes when every issued MMA has
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + C::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sgen + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (t_count + QB - 1) / QB;
  const int nkc = ((S_max + KTILE - 1) / KTILE + KC - 1) / KC;
  const int items = B * nqb * nkc;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NA; ++i) {
      mbar_init(a_full(i), 1);
      mbar_init(a_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_full(i), 1);
      mbar_init(b_empty(i), 1 + 4 * C::HALVES);  // MMA commit + every epilogue warp
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), 4 * C::HALVES);
    }
    mbar_init(mma_drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_q);
    }
    uint32_t a_cnt = 0, b_cnt = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      ItemGeom g;
      if (!item_geom(it, QB, nqb, nkc, T, t_begin, t_count, S_max, pool, ctx_len, g, row_flag)) continue;
      const int bs = b_cnt & 1;
      if (!(ok = mbar_wait_warp(b_empty(bs), ((b_cnt >> 1) & 1) ^ 1, abort, wlim))) break;
      if (lane == 0) {
        const uint32_t wbytes = (uint32_t)(g.nq * H * 4);
        mbar_arrive_expect_tx(b_full(bs), C::B_BYTES + wbytes);
        tma_load_2d(sbase + C::OFF_B + bs * C::B_BYTES, &tmap_q, b_full(bs), 0, (g.b * T + g.t0) * H);
        bulk_load(sbase + C::OFF_W + bs * C::W_BYTES, w + ((int64_t)g.b * T + g.t0) * H, wbytes, b_full(bs));
      }
      ++b_cnt;
      for (int kt = g.kt0; kt < g.kt1; ++kt) {
        const int as = a_cnt % C::NA;
        if (!(ok = mbar_wait_warp(a_empty(as), ((a_cnt / C::NA) & 1) ^ 1, abort, wlim))) break;
        if (lane == 0) {
          // contiguous: row b*S_max + s of the cache; paged: the tile's page (a tile never
          // straddles one); a bad page id loads past the map's extent, which reads zeros
          int y = g.b * S_max + kt * KTILE;
          if (pm.bt != nullptr) {
            y = paged_row(pm, g.b, kt * KTILE);
            if (y < 0) {
              atomicOr(&g_status, 2u);
              y = pm.num_pages << pm.shift;
            }
          }
          mbar_arrive_expect_tx(a_full(as), C::A_BYTES);
          tma_load_2d(sbase + C::OFF_A + as * C::A_BYTES, &tmap_k, a_full(as), 0, y);
        }
        ++a_cnt;
      }
      __syncwarp();
    }
    // drain, whether this warp gave up or not: the copies it issued land before the CTA can leave
    // (after a normal run they landed long ago; after any role gave up some may be in flight)
    for (uint32_t i = (a_cnt > C::NA ? a_cnt - C::NA : 0); i < a_cnt; ++i)
      mbar_wait_bounded(a_full(i % C::NA), (i / C::NA) & 1, 100000000ull);
    for (uint32_t i = (b_cnt > 2 ? b_cnt - 2 : 0); i < b_cnt; ++i)
      mbar_wait_bounded(b_full(i & 1), (i >> 1) & 1, 100000000ull);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t a_cnt = 0, b_cnt = 0, acc_cnt = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      ItemGeom g;
      if (!item_geom(it, QB, nqb, nkc, T, t_begin, t_count, S_max, pool, ctx_len, g, row_flag)) continue;
      const int bs = b_cnt & 1;
      if (!(ok = mbar_wait_warp(b_full(bs), (b_cnt >> 1) & 1, abort, wlim))) break;
      const uint32_t b_addr = sbase + C::OFF_B + bs * C::B_BYTES;
      for (int kt = g.kt0; kt < g.kt1; ++kt) {
        const int as = a_cnt % C::NA;
        const int ab = acc_cnt & 1;
        if (!(ok = mbar_wait_warp(a_full(as), (a_cnt / C::NA) & 1, abort, wlim))) break;
        if (!(ok = mbar_wait_warp(acc_empty(ab), ((acc_cnt >> 1) & 1) ^ 1, abort, wlim))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_addr = sbase + C::OFF_A + as * C::A_BYTES;
          const uint32_t d_tmem = tmem_base + (uint32_t)(ab * C::N);
#pragma unroll
          for (int k = 0; k < D / 32; ++k) {
            mma_f8(d_tmem, smem_desc(a_addr + 32 * k, C::SBO, C::LAYOUT), smem_desc(b_addr + 32 * k, C::SBO, C::LAYOUT),
                   C::IDESC, k > 0 ? 1u : 0u);
          }
          mma_commit(a_empty(as));
          mma_commit(acc_full(ab));
        }
        __syncwarp();
        ++a_cnt;
        ++acc_cnt;
      }
      if (!ok) break;
      if (lane == 0) mma_commit(b_empty(bs));
      __syncwarp();
      ++b_cnt;
    }
    // every MMA this warp issued must have finished before the TMEM is freed: after a normal
    // run the consumers have waited for all of them already, but after any role gave up (here or
    // elsewhere, now or later) some may still run
    if (lane == 0) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait_bounded(mma_drain, 0, 100000000ull);
  } else {
    // ------------------------------------------------------------ epilogue (8 warps)
    const int quad = warp & 3;          // TMEM lanes 32*quad .. +31
    const int half = (warp - 2) >> 2;   // column half
    const int row = quad * 32 + lane;   // key within the tile
    uint32_t b_cnt = 0, acc_cnt = 0;
    bool ok = true;
    // warps beyond the accumulator's column halves take no part (the barriers count only
    // the active ones)
    for (int it = blockIdx.x; half < C::HALVES && it < items && ok; it += gridDim.x) {
      ItemGeom g;
      if (!item_geom(it, QB, nqb, nkc, T, t_begin, t_count, S_max, pool, ctx_len, g, row_flag)) continue;
      const int bs = b_cnt & 1;
      if (!(ok = mbar_wait_warp(b_full(bs), (b_cnt >> 1) & 1, abort, wlim))) break;
      const float* wsm = reinterpret_cast<const float*>(sgen + C::OFF_W + bs * C::W_BYTES) + half * C::COLS;
      const int ctx_b = __ldg(ctx_len + g.b);
      // H == 64: the 16x256b TMEM shape gives each thread 2 keys x 2 heads per 8-column group,
      // always the same two heads (columns 2(lane%4), +1 of every group), so this thread's head
      // weights live in registers for the whole work item: 8 packed pairs per query.
      uint64_t wr[H == 64 ? C::QPH : 1][8];
      if constexpr (H == 64) {
#pragma unroll
        for (int ql = 0; ql < C::QPH; ++ql)
#pragma unroll
          for (int gg = 0; gg < 8; ++gg)
            wr[ql][gg] = *reinterpret_cast<const uint64_t*>(wsm + ql * H + 8 * gg + 2 * (lane & 3));
      }
      if constexpr (H == 64) {
        // Each tile's accumulator slice comes to registers in STEPS loads, (query ql of this
        // warp, row half rh of its 32 TMEM lanes) each, double-buffered in one flat pipeline
        // across the tiles of the item: the next tile's first load is in flight while this
        // tile's last step is summed and its sums are reduced across the quad and stored.
        constexpr int STEPS = 2 * C::QPH;
        static_assert(STEPS % 2 == 0, "buffer parity follows the step");
        float v[2][32];
        auto issue = [&](int ab, int st, float (&dst)[32]) {
          tmem_ld_16x256b_x8(tmem_base + (uint32_t)(ab * C::N + half * C::COLS) +
                                 ((uint32_t)(quad * 32 + (st & 1) * 16) << 16) + (uint32_t)((st >> 1) * H),
                             dst);
        };
        // per query of this warp: its score row, its causal limit (last visible key row) and
        // whether it exists in this block; a store is then an add, a compare and a select
        float* qrow[C::QPH];
        int lim[C::QPH];
        bool qok[C::QPH];
        float qtau[C::QPH];
        int64_t qr[C::QPH];
#pragma unroll
        for (int ql = 0; ql < C::QPH; ++ql) {
          const int qq = half * C::QPH + ql;
          const int t = g.t0 + qq;
          qok[ql] = qq < g.nq;
          qr[ql] = (int64_t)g.b * t_count + (t - t_begin);
          qrow[ql] = scores + qr[ql] * ld;
          const int pos = ctx_b - T + t;
          lim[ql] = pos < 0 ? -1 : pos / pool;   // s * pool <= pos  <=>  s <= pos / pool
          if constexpr (CAND) qtau[ql] = qok[ql] ? __ldg(tau + qr[ql]) : INFINITY;
        }
        // fused selection: the warp's candidates of each query wait in shared memory (scnt of
        // them, a warp-uniform count) and go out in one flush: one atomic reserves their slots
        float2* cb = reinterpret_cast<float2*>(sgen + C::OFF_CBUF) + (warp - 2) * C::QPH * C::CB;
        int scnt[C::QPH];
#pragma unroll
        for (int ql = 0; ql < C::QPH; ++ql) scnt[ql] = 0;
        auto flush = [&](int ql) {
          __syncwarp();
          int base = 0;
          if (lane == 0 && scnt[ql] > 0) base = atomicAdd(cnt + qr[ql], scnt[ql]);
          base = __shfl_sync(0xffffffffu, base, 0);
          for (int i = lane; i < scnt[ql]; i += 32)
            if (base + i < cap) cand[qr[ql] * cap + base + i] = cb[ql * C::CB + i];
          __syncwarp();
          scnt[ql] = 0;
        };
        auto store = [&](int ql, int s, float val) {
          if constexpr (CAND) {
            const bool pass = qok[ql] && s < S_max && s <= lim[ql] && val >= qtau[ql];
            const unsigned m = __ballot_sync(0xffffffffu, pass);
            if (m != 0u) {
              if (pass) cb[ql * C::CB + scnt[ql] + __popc(m & ((1u << lane) - 1u))] = make_float2(val, __int_as_float(s));
              scnt[ql] += __popc(m);
              if (scnt[ql] > C::CB - 32) flush(ql);   // room for a full warp's worth stays
            }
          } else {
            if (qok[ql] && s < S_max) qrow[ql][s] = (s <= lim[ql]) ? val : -INFINITY;
          }
        };
        if (g.kt0 < g.kt1) {
          if (!(ok = mbar_wait_warp(acc_full(acc_cnt & 1), (acc_cnt >> 1) & 1, abort, wlim))) break;
          tc_fence_after();
          issue(acc_cnt & 1, 0, v[0]);
          tmem_ld_wait();
          launder(v[0]);
        }
        for (int kt = g.kt0; kt < g.kt1; ++kt) {
          const int ab = acc_cnt & 1;
          const bool more = kt + 1 < g.kt1;
          float red[2 * STEPS];  // per step: partial sums of key A (lane base + lane/4) and key B (+8)
#pragma unroll
          for (int st = 0; st < STEPS; ++st) {
            if (st + 1 < STEPS) {
              issue(ab, st + 1, v[(st + 1) & 1]);
            } else {
              // every load of this tile has completed: hand the accumulator back to the MMA
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(acc_empty(ab));
              if (more) {
                if (!(ok = mbar_wait_warp(acc_full(ab ^ 1), ((acc_cnt + 1) >> 1) & 1, abort, wlim))) break;
                tc_fence_after();
                issue(ab ^ 1, 0, v[0]);
              }
            }
            const float* vc = v[st & 1];
            const int ql = st >> 1;
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // key A even/odd groups, key B even/odd
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              const float* x = vc + 4 * r;
              acc[r & 1] = ffma2(wr[ql][r], pack2(fmaxf(x[0], 0.f), fmaxf(x[1], 0.f)), acc[r & 1]);
              acc[2 + (r & 1)] = ffma2(wr[ql][r], pack2(fmaxf(x[2], 0.f), fmaxf(x[3], 0.f)), acc[2 + (r & 1)]);
            }
            float xa0, xa1, xb0, xb1;
            unpack2(fadd2(acc[0], acc[1]), xa0, xa1);
            unpack2(fadd2(acc[2], acc[3]), xb0, xb1);
            red[2 * st] = xa0 + xa1;
            red[2 * st + 1] = xb0 + xb1;
            if (st + 1 < STEPS) {
              tmem_ld_wait();
              launder(v[(st + 1) & 1]);
            }
          }
          if (!ok) break;
          ++acc_cnt;
          // Sum over the 4 threads of a quad (each holds 16 of a query's 64 heads) as a
          // transposing reduction: after the xor-1 round a thread keeps the values of its key
          // (A on even lanes, B on odd), after the xor-2 round those of its row half.
          const int odd = lane & 1, bit1 = (lane >> 1) & 1;
          float k1[STEPS];
#pragma unroll
          for (int m = 0; m < STEPS; ++m) {
            const float mine = odd ? red[2 * m + 1] : red[2 * m];
            const float other = odd ? red[2 * m] : red[2 * m + 1];
            k1[m] = mine + __shfl_xor_sync(0xffffffffu, other, 1);
          }
#pragma unroll
          for (int n = 0; n < C::QPH; ++n) {
            const float mine = bit1 ? k1[2 * n + 1] : k1[2 * n];
            const float other = bit1 ? k1[2 * n] : k1[2 * n + 1];
            store(n, kt * KTILE + quad * 32 + bit1 * 16 + (lane >> 2) + 8 * odd,
                  mine + __shfl_xor_sync(0xffffffffu, other, 2));
          }
          if (more) {
            tmem_ld_wait();
            launder(v[0]);
          }
        }
        if constexpr (CAND) {
          if (ok) {
#pragma unroll
            for (int ql = 0; ql < C::QPH; ++ql) flush(ql);
          }
        }
      } else {
      for (int kt = g.kt0; kt < g.kt1; ++kt) {
        const int ab = acc_cnt & 1;
        if (!(ok = mbar_wait_warp(acc_full(ab), (acc_cnt >> 1) & 1, abort, wlim))) break;
        tc_fence_after();
        // finished sum of query ql (local to this warp) for key s -> masked store
        auto store = [&](int ql, int s, float val) {
          const int qq = half * C::QPH + ql;
          const int t = g.t0 + qq;
          const int pos = ctx_b - T + t;
          const int64_t qrow_id = (int64_t)g.b * t_count + (t - t_begin);
          if constexpr (CAND) {
            const bool live = qq < g.nq && s < S_max && s * pool <= pos;
            cand_append(live && val >= __ldg(tau + (live ? qrow_id : 0)), val, s, cnt + (live ? qrow_id : 0),
                        cand + (live ? qrow_id : 0) * cap, cap);
          } else {
            if (qq < g.nq && s < S_max) scores[qrow_id * ld + s] = (s * pool <= pos) ? val : -INFINITY;
          }
        };
        const uint32_t tcol = tmem_base + (uint32_t)(ab * C::N + half * C::COLS);
        {
          const uint32_t taddr = tcol + ((uint32_t)(quad * 32) << 16);
          const int s = kt * KTILE + row;
          // w * relu(x) over 4 columns into two packed accumulators
          auto quad4 = [&](const float* v, int col, uint64_t& a0, uint64_t& a1) {
            const float4 wv = *reinterpret_cast<const float4*>(wsm + col);
            a0 = ffma2(pack2(wv.x, wv.y), pack2(fmaxf(v[0], 0.f), fmaxf(v[1], 0.f)), a0);
            a1 = ffma2(pack2(wv.z, wv.w), pack2(fmaxf(v[2], 0.f), fmaxf(v[3], 0.f)), a1);
          };
          float v[2][32];
          tmem_ld32(taddr, v[0]);
          tmem_ld_wait();
          launder(v[0]);
          uint64_t a2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
          for (int c = 0; c < C::CHUNKS; ++c) {
            if (c + 1 < C::CHUNKS) tmem_ld32(taddr + 32 * (c + 1), v[(c + 1) & 1]);   // in flight during c
            const float* vc = v[c & 1];
            if constexpr (H >= 32) {
              // a query spans H/32 chunks: 4 packed partial sums, chains of H/16 FMAs
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                quad4(vc + i, 32 * c + i, a2[0], a2[1]);
                quad4(vc + i + 4, 32 * c + i + 4, a2[2], a2[3]);
              }
              if ((c + 1) % (H / 32) == 0) {
                float x0, x1, x2, x3, x4, x5, x6, x7;
                unpack2(a2[0], x0, x1); unpack2(a2[1], x2, x3); unpack2(a2[2], x4, x5); unpack2(a2[3], x6, x7);
                store(c / (H / 32), s, ((x0 + x1) + (x2 + x3)) + ((x4 + x5) + (x6 + x7)));
                a2[0] = a2[1] = a2[2] = a2[3] = 0ull;
              }
            } else {
              // 32/H whole queries per chunk
#pragma unroll
              for (int qc = 0; qc < 32 / H; ++qc) {
                uint64_t b0 = 0ull, b1 = 0ull;
#pragma unroll
                for (int i = 0; i < H; i += 4) quad4(vc + qc * H + i, 32 * c + qc * H + i, b0, b1);
                float x0, x1, x2, x3;
                unpack2(b0, x0, x1); unpack2(b1, x2, x3);
                store(c * (32 / H) + qc, s, (x0 + x1) + (x2 + x3));
              }
            }
            if (c + 1 < C::CHUNKS) {
              tmem_ld_wait();
              launder(v[(c + 1) & 1]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty(ab));
        }
        ++acc_cnt;
      }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(b_empty(bs));
      ++b_cnt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

// 2-D uint8 tensor map: `rows` rows of `row_bytes` spaced `row_stride` bytes apart (0 = dense),
// boxes of box_rows x row_bytes.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t row_bytes, uint32_t box_rows,
              uint64_t row_stride = 0) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_stride ? row_stride : row_bytes};
  cuuint32_t box[2] = {row_bytes, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int H, int D, int QB, bool CAND>
int launch_tc(const uint8_t* q_idx, const float* w, const uint8_t* k_idx, const int32_t* ctx_len, int B, int T,
              int S_max, int pool, int t_begin, int t_count, float* scores, int64_t ld, const PageMap& pm,
              const IndexerMode& md, cudaStream_t stream) {
  using C = IdxCfg<H, D, QB>;
  CUtensorMap mk, mq;
  // key rows: contiguous (every md.kstride-th row of the cache when sampling), or the page pool
  const uint64_t key_rows = pm.bt != nullptr ? ((uint64_t)pm.num_pages << pm.shift) : (uint64_t)B * S_max;
  if (!make_map(&mk, k_idx, key_rows, D, KTILE, (uint64_t)md.kstride * D)) return DSA_ERR_CUDA;
  if (!make_map(&mq, q_idx, (uint64_t)B * T * H, D, C::N)) return DSA_ERR_CUDA;
  auto kern = index_scores_tc_kernel<H, D, QB, CAND>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int nqb = (t_count + QB - 1) / QB;
  const int nkc = ((S_max + KTILE - 1) / KTILE + KC - 1) / KC;
  const int64_t items = (int64_t)B * nqb * nkc;
  const int grid = (int)std::min<int64_t>(items, (int64_t)C::CTAS_PER_SM * num_sms());
  kern<<<grid, NUM_THREADS, C::SMEM, stream>>>(mk, mq, w, ctx_len, B, T, S_max, pool, t_begin, t_count, scores, ld,
                                               pm, md.tau, md.cand, md.cnt, md.cap, md.row_flag);
  return check_launch();
}

template <bool CAND>
int launch_shape(const uint8_t* q_idx, const float* w, const uint8_t* k_idx, const int32_t* ctx_len, int B, int T,
                 int S_max, int H_I, int d_I, int pool, int t_begin, int t_count, float* scores, int64_t ld,
                 const PageMap& pm, const IndexerMode& md, cudaStream_t stream) {
  if (H_I == 64 && d_I == 128) {
    if (t_count < 4)  // decode-like: one query per block keeps the MMA N at the head count
      return launch_tc<64, 128, 1, CAND>(q_idx, w, k_idx, ctx_len, B, T, S_max, pool, t_begin, t_count, scores, ld,
                                         pm, md, stream);
    return launch_tc<64, 128, 4, CAND>(q_idx, w, k_idx, ctx_len, B, T, S_max, pool, t_begin, t_count, scores, ld, pm,
                                       md, stream);
  }
  if (H_I == 4 && d_I == 64)
    return launch_tc<4, 64, 64, CAND>(q_idx, w, k_idx, ctx_len, B, T, S_max, pool, t_begin, t_count, scores, ld, pm,
                                      md, stream);
  return DSA_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace

int launch_index_scores(const uint8_t* q_idx, const float* w, const uint8_t* k_idx, const int32_t* ctx_len, int B,
                        int T, int S_max, int H_I, int d_I, int pool, int t_begin, int t_count, float* scores,
                        int64_t ld, const PageMap& pm, cudaStream_t stream, const IndexerMode& md) {
  if (B == 0 || t_count == 0 || S_max == 0) return DSA_OK;
  if (md.cand != nullptr)
    return launch_shape<true>(q_idx, w, k_idx, ctx_len, B, T, S_max, H_I, d_I, pool, t_begin, t_count, scores, ld, pm,
                              md, stream);
  return launch_shape<false>(q_idx, w, k_idx, ctx_len, B, T, S_max, H_I, d_I, pool, t_begin, t_count, scores, ld, pm,
                             md, stream);
}

namespace {
// Test hook: one thread waits on an mbarrier that nothing ever arrives at, through the same
// bounded wait the tensor-core kernels use, so the time limit runs out and the device
// status word is set.  The kernel then returns normally; the context stays usable.
__global__ void wait_timeout_probe_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  abort_flag = 0;
  mbar_init(b, 1);
  fence_barrier_init();
  mbar_wait(b, 0, &abort_flag, limit_ns);
}
}  // namespace

int launch_wait_timeout_probe(uint64_t limit_ns, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 1, 0, stream>>>(limit_ns);
  return check_launch();
}

void indexer_set_wait_limit(uint64_t ns) {
  const unsigned long long v = ns;
  cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v));
}

// Reads and clears the indexer's device status word (bit 0: a bounded wait gave up).
unsigned int indexer_take_status() {
  unsigned int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
  return v;
}

}  // namespace dsa
