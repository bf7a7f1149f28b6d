// Sparse MLA attention on the 5th-generation tensor cores (Stage 2 of "DeepSeek Sparse
// Attention", "GLM 5.2: How Four Co-Designed Mechanisms Beat Raw Scale": full attention over
// the selected tokens only).  All 128 query heads of a token share one latent row per key:
// K = the 576-wide row, V = its first 512 columns.
//
// TMEM holds 128 lanes x 512 fp32 columns, exactly the size of O = 128 heads x 512 dv, so a
// query is served by a cluster of two CTAs.  CTA c (c = 0, 1):
//   * holds q[:, 288c .. 288c+287] in TMEM (the MMA's A operand, so no shared-memory
//     bandwidth goes to re-reading q) and computes the partial scores over those 288 columns
//     (18 x tcgen05.mma M128 N64 K16 per tile of 64 keys), then swaps its partial with the
//     partner through distributed shared memory; both add the two partials in the same
//     order, so both hold the same scores, softmax and P;
//   * accumulates O[:, 256c .. 256c+255] = P V in TMEM (4 x M128 N256 K16 per tile, P read
//     from TMEM, V read MN-major straight from the gathered rows);
//   * gathers only the row columns it needs: c = 0 columns 0..287, c = 1 columns 256..575.
// Per CTA: a 4-stage ring of 40 KB key tiles; TMEM 64 score + 144 q + 32 P + 256 output
// columns.
//
//   warps 0-3  softmax: thread = head.  First each thread stores its head's q columns into
//              TMEM.  Per tile j: (1) the partner's partial of tile j (sent a tile earlier)
//              + our own -> masked scores and their max; a relaxed remote arrive, ordered
//              after every read of the partner's rows by a data dependency, frees its buffer;
//              (2) our partial of tile j+1 from TMEM -> a local stage -> per warp, one 8 KB
//              bulk copy into the partner (completing that warp's barrier there), in flight
//              while (3) the running max moves only when a tile exceeds it by more than 2^8
//              (then O is rescaled in TMEM) and P = exp2(S - m) goes to TMEM as bf16 pairs.
//              At the end O / l is written out (or a split partial with its lse).
//   warps 4-6  gather: 16-byte cp.async of the selected rows into the 128-byte-swizzled
//              K-major layout the tensor core reads (also V's MN-major layout).
//   warp 7     TMEM owner and MMA issuer: S_0, S_1, then per tile S_{j+2} ahead of P_j.V_j.
// Persistent: one cluster per two SMs serves work items (query, key split) in turn, and every
// barrier phase counts tiles over all its items.  At an item boundary the next query's q
// (prefetched to L2 an item earlier) goes into TMEM before the previous query's O is read out,
// so the MMA computes the next query's first scores meanwhile, and the gather warps run
// straight on into the next query's rows.
// Every wait is bounded (tc_common.cuh); the two CTAs meet at cluster barriers only at start
// and end.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace dsa {
namespace {

using namespace tc;

constexpr int HQ = 128, DQK = 576, DV = 512, DVH = 256;
constexpr int NK = 64;                  // keys per tile
constexpr int NS = 4;                   // key-tile stages
constexpr int BLKS = 5;                 // 64-column blocks of a key row held per CTA
constexpr int K_BLK = NK * 128;         // 64 rows x 128 B
constexpr int KSTEPS = 18;              // 288 score columns / 16 per MMA
constexpr int KV_STAGE = BLKS * K_BLK;                 // 40960
constexpr int OFF_KV = 0;
constexpr int X_BYTES = HQ * NK * 4;                   // 32768: one tile of fp32 partial scores
constexpr int OFF_XS = OFF_KV + NS * KV_STAGE;         // own partial, staged for the bulk copy out
constexpr int OFF_X = OFF_XS + X_BYTES;                // partner's partial, copied in
constexpr int OFF_IDS = OFF_X + X_BYTES;
constexpr int OFF_BAR = OFF_IDS + NS * NK * 4 + 16 * NS;   // ids + an all-valid flag per stage
constexpr int NBARS = 3 * NS + 14;   // + the MMA drain barrier
constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;       // + alignment slack
constexpr int THREADS = 256;            // 8 warps: 2 per SM sub-partition, so up to 255 registers
constexpr int GATHER_THREADS = 96;
constexpr int MMA_WARP = 7;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S = 0;      // partial scores, NK columns
constexpr uint32_t COL_Q = 64;     // this CTA's 288 q columns as packed bf16 pairs: 144 columns
constexpr uint32_t COL_P = 224;    // P of one tile as packed bf16 pairs (the P.V MMA's A operand): 32 columns
constexpr uint32_t COL_O = 256;    // DVH output columns
constexpr float kRescaleLog2 = 8.0f;

static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert((OFF_KV % 1024) == 0 && (OFF_X % 128) == 0 && (OFF_XS % 128) == 0, "alignment");
static_assert(COL_S + NK <= COL_Q && COL_Q + 144 <= COL_P && COL_P + NK / 2 <= COL_O, "TMEM map");

constexpr uint32_t IDESC_S = instr_desc(128, NK, 1);                   // bf16, K-major A and B
constexpr uint32_t IDESC_PV = instr_desc(128, DVH, 1) | (1u << 16);    // A (P) from TMEM, B (V) MN-major

__device__ __forceinline__ uint64_t smem_desc_lbo(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1u << 46) | ((uint64_t)layout << 61);
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
      "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
      "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31]));
}
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]));
}
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}
// D[tmem] (+)= A[tmem] x B[smem desc]^T, bf16 inputs, fp32 accumulation (A read from TMEM:
// row m in lane m, element k of the row at column k/2, even k in the low half).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// 32-byte global store (one whole sector per lane); the address must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t a4,
                                             uint32_t a5, uint32_t a6, uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"l"(p), "r"(a0), "r"(a1), "r"(a2),
               "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ---- cluster (distributed shared memory) helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_cta(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Relaxed arrive on a barrier in the partner CTA: no cluster-scope fence.  `dep` is a value
// computed from every shared-memory load the arrive must follow, so those loads have returned
// their data (and can no longer observe a later write) before the arrive is issued.
__device__ __forceinline__ void mbar_arrive_cluster_after(uint32_t cluster_bar, float dep) {
  asm volatile("{\n\t.reg .f32 d;\n\tmov.f32 d, %1;\n\t"
               "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];\n\t}\n" ::"r"(cluster_bar), "f"(dep)
               : "memory");
}
// Non-blocking and potentially blocking checks of a local barrier that the partner CTA completes
// (cluster-scope acquire).
__device__ __forceinline__ bool mbar_test_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on a local barrier that the partner CTA completes (cluster-scope acquire).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort,
                                                  uint64_t limit) {
  if (limit < kImmediateNs) {
    if (mbar_test_wait_cluster(bar, parity)) return true;
    *abort = 1;
    atomicOr(&g_status, 1u);
    return false;
  }
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 31u) == 0u) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > limit) {
        *abort = 1;
        atomicOr(&g_status, 1u);
        return false;
      }
    }
  }
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// q[bt, head, 288*half .. +287] -> TMEM lane `head` (bf16 pairs packed per 32-bit column),
// then this warp's arrival on q_ready.  Out of line: it runs once per query, and inlined its
// registers would crowd the per-tile loop.
__device__ __noinline__ void attn_load_q(const __nv_bfloat16* __restrict__ q, int bt, int row, int half, uint32_t tmem,
                                         uint32_t lane_off, uint32_t q_ready, int lane) {
  // q[head, 288*half .. +287] -> TMEM lane `head`, bf16 pairs packed per 32-bit column
  const uint4* qsrc = reinterpret_cast<const uint4*>(q + ((int64_t)bt * HQ + row) * DQK + 288 * half);
  // two batches of loads (16 + 20 x 16 B; the rows were asked into L2 an item earlier, or at the
  // kernel start for a CTA's first item)
  {
    uint4 qa[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) qa[i] = __ldg(qsrc + i);
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) { w[4 * i] = qa[i].x; w[4 * i + 1] = qa[i].y; w[4 * i + 2] = qa[i].z; w[4 * i + 3] = qa[i].w; }
    tmem_st32u(tmem + lane_off + COL_Q, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) { w[4 * i] = qa[8 + i].x; w[4 * i + 1] = qa[8 + i].y; w[4 * i + 2] = qa[8 + i].z; w[4 * i + 3] = qa[8 + i].w; }
    tmem_st32u(tmem + lane_off + COL_Q + 32, w);
  }
  {
    uint4 qb[20];
#pragma unroll
    for (int i = 0; i < 20; ++i) qb[i] = __ldg(qsrc + 16 + i);
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) { w[4 * i] = qb[i].x; w[4 * i + 1] = qb[i].y; w[4 * i + 2] = qb[i].z; w[4 * i + 3] = qb[i].w; }
    tmem_st32u(tmem + lane_off + COL_Q + 64, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) { w[4 * i] = qb[8 + i].x; w[4 * i + 1] = qb[8 + i].y; w[4 * i + 2] = qb[8 + i].z; w[4 * i + 3] = qb[8 + i].w; }
    tmem_st32u(tmem + lane_off + COL_Q + 96, w);
    uint32_t w16[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) { w16[4 * i] = qb[16 + i].x; w16[4 * i + 1] = qb[16 + i].y; w16[4 * i + 2] = qb[16 + i].z; w16[4 * i + 3] = qb[16 + i].w; }
    tmem_st16u(tmem + lane_off + COL_Q + 128, w16);
  }
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(q_ready);
}

// Epilogue of one item: waits for its last P.V, then O / l (or the split partial and its lse)
// out of TMEM.  Out of line for the same reason as attn_load_q.
__device__ __noinline__ bool attn_epilogue(int bt, int sp, int ntiles, float m_fin, float l_fin, uint32_t g_last,
                                           bool good, int nbt, int row, int half, uint32_t tmem, uint32_t lane_off,
                                           uint32_t pv_done, volatile int* abort, __nv_bfloat16* __restrict__ out,
                                           float* __restrict__ lse, __nv_bfloat16* __restrict__ part_o,
                                           float* __restrict__ part_lse) {
  if (good && ntiles > 0) good = mbar_wait(pv_done, g_last & 1, abort, wait_limit());
  good = __all_sync(0xffffffffu, good);   // the TMEM reads below are warp-collective
  tc_fence_after();
  const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
  const float lse_r = l_fin > 0.f ? (m_fin + log2f(l_fin)) * 0.69314718055994531f : -INFINITY;
  const bool have_o = good && ntiles > 0;
  const int64_t orow = (int64_t)bt * HQ + row;
  // every row and column half starts a multiple of 32 B past the base: the base decides whether
  // the 32-byte stores can be used
  const bool wide = ((reinterpret_cast<uintptr_t>(part_o == nullptr ? (void*)out : (void*)part_o)) & 31u) == 0;
  if (part_o == nullptr) {
    __nv_bfloat16* dst = out + orow * DV + half * DVH;
#pragma unroll 1
    for (int c = 0; c < DVH; c += 32) {
      float o[32];
      if (have_o) {
        tmem_ld32(tmem + lane_off + COL_O + c, o);
        tmem_ld_wait();
        launder(o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      if (wide) {   // 32 B per store: each lane fills whole sectors of its row
#pragma unroll
        for (int i = 0; i < 32; i += 16)
          st_global_v8(dst + c + i, pack2_bf16(o[i] * inv, o[i + 1] * inv), pack2_bf16(o[i + 2] * inv, o[i + 3] * inv),
                       pack2_bf16(o[i + 4] * inv, o[i + 5] * inv), pack2_bf16(o[i + 6] * inv, o[i + 7] * inv),
                       pack2_bf16(o[i + 8] * inv, o[i + 9] * inv), pack2_bf16(o[i + 10] * inv, o[i + 11] * inv),
                       pack2_bf16(o[i + 12] * inv, o[i + 13] * inv), pack2_bf16(o[i + 14] * inv, o[i + 15] * inv));
      } else {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint4 v;
          v.x = pack2_bf16(o[i] * inv, o[i + 1] * inv);
          v.y = pack2_bf16(o[i + 2] * inv, o[i + 3] * inv);
          v.z = pack2_bf16(o[i + 4] * inv, o[i + 5] * inv);
          v.w = pack2_bf16(o[i + 6] * inv, o[i + 7] * inv);
          *reinterpret_cast<uint4*>(dst + c + i) = v;
        }
      }
    }
    if (lse != nullptr && half == 0) lse[orow] = lse_r;
  } else {
    const int64_t rows = (int64_t)nbt * HQ;
    __nv_bfloat16* dst = part_o + ((int64_t)sp * rows + orow) * DV + half * DVH;   // bf16 partial
#pragma unroll 1
    for (int c = 0; c < DVH; c += 32) {
      float o[32];
      if (have_o) {
        tmem_ld32(tmem + lane_off + COL_O + c, o);
        tmem_ld_wait();
        launder(o);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      if (wide) {
#pragma unroll
        for (int i = 0; i < 32; i += 16)
          st_global_v8(dst + c + i, pack2_bf16(o[i] * inv, o[i + 1] * inv), pack2_bf16(o[i + 2] * inv, o[i + 3] * inv),
                       pack2_bf16(o[i + 4] * inv, o[i + 5] * inv), pack2_bf16(o[i + 6] * inv, o[i + 7] * inv),
                       pack2_bf16(o[i + 8] * inv, o[i + 9] * inv), pack2_bf16(o[i + 10] * inv, o[i + 11] * inv),
                       pack2_bf16(o[i + 12] * inv, o[i + 13] * inv), pack2_bf16(o[i + 14] * inv, o[i + 15] * inv));
      } else {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint4 v;
          v.x = pack2_bf16(o[i] * inv, o[i + 1] * inv);
          v.y = pack2_bf16(o[i + 2] * inv, o[i + 3] * inv);
          v.z = pack2_bf16(o[i + 4] * inv, o[i + 5] * inv);
          v.w = pack2_bf16(o[i + 6] * inv, o[i + 7] * inv);
          *reinterpret_cast<uint4*>(dst + c + i) = v;
        }
      }
    }
    if (half == 0) part_lse[(int64_t)sp * rows + orow] = lse_r;
  }
  return good;
}

struct Item {
  int bt, sp, b, kbeg, kend, ntiles;
};

__global__ void __cluster_dims__(1, 2, 1) __launch_bounds__(THREADS, 1)
sparse_mla_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv, int64_t kv_rs,
                     int64_t kv_bs, int S_kv, const int32_t* __restrict__ idx, int T, int nbt, int items, int k,
                     int keys_per_split, float scale_log2, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                     __nv_bfloat16* __restrict__ part_o, float* __restrict__ part_lse, PageMap pm) {
  const uint64_t wlim = wait_limit();   // the bounded waits' time limit, read once
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - sraw);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto kv_full = [&](int s) { return bar0 + 8u * s; };
  auto kv_empty = [&](int s) { return bar0 + 8u * (NS + s); };
  auto ids_ready = [&](int s) { return bar0 + 8u * (2 * NS + s); };
  const uint32_t s_full = bar0 + 8u * (3 * NS);
  const uint32_t s_empty = bar0 + 8u * (3 * NS + 1);
  const uint32_t p_full = bar0 + 8u * (3 * NS + 2);
  const uint32_t pv_done = bar0 + 8u * (3 * NS + 3);
  const uint32_t q_ready = bar0 + 8u * (3 * NS + 4);
  // per softmax warp w (rows 32w..32w+31): the partner's rows landed / the partner read ours
  auto x_full = [&](int w) { return bar0 + 8u * (3 * NS + 5 + w); };
  auto x_free = [&](int w) { return bar0 + 8u * (3 * NS + 9 + w); };
  const uint32_t mma_drain = bar0 + 8u * (3 * NS + 13);   // completes when every issued MMA has
  volatile int* ids_s = reinterpret_cast<volatile int*>(sgen + OFF_IDS);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sgen + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a split-key launch's combine kernel (a programmatic dependent) may be scheduled from now on;
  // it waits for this grid's completion before it reads anything
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  if (threadIdx.x == 0 && (int)blockIdx.x < items)   // the first item's q: to L2 while the CTA sets up
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(q + (int64_t)((int)blockIdx.x % nbt) * HQ * DQK),
                 "r"((uint32_t)(HQ * DQK * 2))
                 : "memory");
  const int half = (int)cluster_rank();       // 0 or 1: score columns 288*half.., output columns 256*half..
  const uint32_t partner = (uint32_t)(half ^ 1);
  // Work item it = (query bt = it % nbt, key split sp = it / nbt); the cluster takes items
  // blockIdx.x, blockIdx.x + gridDim.x, ..  Every barrier phase below counts tiles (g) or
  // items with tiles, over all the items this CTA has served.
  auto geom = [&](int it) {
    Item I;
    I.bt = it % nbt;
    I.sp = it / nbt;
    I.b = I.bt / T;
    I.kbeg = I.sp * keys_per_split;
    I.kend = min(k, I.kbeg + keys_per_split);
    I.ntiles = I.kend > I.kbeg ? (I.kend - I.kbeg + NK - 1) / NK : 0;
    return I;
  };
  const int blk0 = half == 0 ? 0 : 4;             // first 64-column block held by this CTA
  const int ch_lo = half == 0 ? 0 : 32;           // gathered 16-byte chunks [ch_lo, ch_hi) of a row
  const int ch_hi = half == 0 ? 36 : 72;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(kv_full(s), GATHER_THREADS);
      mbar_init(kv_empty(s), 1);
      mbar_init(ids_ready(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    for (int w = 0; w < 4; ++w) {
      mbar_init(x_full(w), 1);   // one expect-tx arrival per use, plus the partner's 8 KB
      mbar_init(x_free(w), 1);   // the partner's warp w, once it has read our rows
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(q_ready, 4);
    mbar_init(mma_drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(sbase + OFF_MISC, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if (warp < 4 && lane == 0) mbar_arrive_expect_tx(x_full(warp), X_BYTES / 4);   // arm the first exchange
  cluster_sync();   // both CTAs' barriers exist (and are armed) before either signals the other
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 && warp < MMA_WARP) {
    // ------------------------------------------------------------ gather (cp.async)
    // Warp gw copies the first 32 16-byte chunks of rows gw, gw+3, .. (lane l chunk l, one
    // coalesced request per row), and the remaining 4 (CTA 0) or 8 (CTA 1) chunks of groups of
    // 8 or 4 rows in one request per group, so every request has all 32 lanes busy.  A tile's
    // ids come from one coalesced load per warp, issued a tile ahead, and reach the rows
    // through shuffles.
    const int gw = warp - 4;
    bool ok = true;
    uint32_t g = 0;   // tiles gathered so far
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
    const Item I = geom(it);
    // contiguous: rows of this sequence's cache; paged: rows of the shared page pool
    const __nv_bfloat16* kvb = pm.bt != nullptr ? kv : kv + (int64_t)I.b * kv_bs;
    const int32_t* irow = idx + (int64_t)I.bt * k;
    // The selected ids of a tile pass three steps a tile apart, so no load's latency stalls the
    // gather: tile j+2's ids are loaded, tile j+1's page ids looked up (paged caches), and tile
    // j's ids checked and turned into cache rows.  Ids at or beyond the cache's S_kv rows, and ids
    // whose page id is out of range, are skipped like a -1 (nothing outside the cache is read)
    // and flagged in the status word.
    auto raw_id = [&](int j, int r) -> int {
      const int p = I.kbeg + j * NK + r;
      return (j < I.ntiles && p < I.kend) ? __ldg(irow + p) : -1;
    };
    auto page_of = [&](int id) -> int {   // the page holding cache id `id` (paged caches)
      return (pm.bt != nullptr && id >= 0 && id < S_kv) ? __ldg(pm.bt + (int64_t)I.b * pm.pps + (id >> pm.shift)) : 0;
    };
    auto to_row = [&](int& id, int page) -> int {
      if (id < 0) return -1;
      if (id >= S_kv || (pm.bt != nullptr && (page < 0 || page >= pm.num_pages))) {
        atomicOr(&g_status, 2u);
        id = -1;
        return -1;
      }
      return pm.bt == nullptr ? id : (page << pm.shift) | (id & ((1 << pm.shift) - 1));
    };
    int ra0 = raw_id(0, lane), ra1 = raw_id(0, lane + 32);   // tile j
    int rb0 = raw_id(1, lane), rb1 = raw_id(1, lane + 32);   // tile j+1
    int pa0 = page_of(ra0), pa1 = page_of(ra1);              // tile j's pages
    for (int j = 0; j < I.ntiles; ++j, ++g) {
      const int st = g % NS;
      int id0 = ra0, id1 = ra1;
      const int row0 = to_row(id0, pa0), row1 = to_row(id1, pa1);
      ra0 = rb0;
      ra1 = rb1;
      pa0 = page_of(ra0);
      pa1 = page_of(ra1);
      rb0 = raw_id(j + 2, lane);
      rb1 = raw_id(j + 2, lane + 32);
      if (!(ok = mbar_wait_warp(kv_empty(st), ((g / NS) & 1) ^ 1, abort, wlim))) break;
      if (gw == 0) {
        ids_s[st * NK + lane] = id0;
        ids_s[st * NK + 32 + lane] = id1;
        const unsigned all_valid = __all_sync(0xffffffffu, id0 >= 0 && id1 >= 0);
        if (lane == 0) ids_s[NS * NK + 4 * st] = (int)all_valid;   // tile needs no masking
        __syncwarp();
        if (lane == 0) mbar_arrive(ids_ready(st));
      }
      const uint32_t stage = sbase + OFF_KV + st * KV_STAGE;
#pragma unroll 4
      for (int r = gw; r < NK; r += 3) {
        const int key = __shfl_sync(0xffffffffu, r < 32 ? id0 : id1, r & 31);
        const int crow = __shfl_sync(0xffffffffu, r < 32 ? row0 : row1, r & 31);
        const __nv_bfloat16* src = kvb + (int64_t)(key < 0 ? 0 : crow) * kv_rs;
        const int c = ch_lo + lane;
        const uint32_t dst = stage + ((c >> 3) - blk0) * K_BLK + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        cp_async16(dst, src + c * 8, key < 0 ? 0 : 16);
      }
      // the last rc = 4 (CTA 0) or 8 (CTA 1) chunks of 32/rc rows at a time: lane l takes row
      // r0 + l/rc, chunk ch_lo + 32 + l%rc
      const int rc_sh = half == 0 ? 2 : 3;
      const int rpg = 32 >> rc_sh;
      for (int grp = gw; grp < NK / rpg; grp += 3) {
        const int r0 = grp * rpg;
        const int r = r0 + (lane >> rc_sh);
        const int key = __shfl_sync(0xffffffffu, r0 < 32 ? id0 : id1, (r0 & 31) + (lane >> rc_sh));
        const int crow = __shfl_sync(0xffffffffu, r0 < 32 ? row0 : row1, (r0 & 31) + (lane >> rc_sh));
        const __nv_bfloat16* src = kvb + (int64_t)(key < 0 ? 0 : crow) * kv_rs;
        const int c = ch_lo + 32 + (lane & ((1 << rc_sh) - 1));
        const uint32_t dst = stage + ((c >> 3) - blk0) * K_BLK + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        cp_async16(dst, src + c * 8, key < 0 ? 0 : 16);
      }
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(kv_full(st)) : "memory");
    }
    }
    cp_async_wait<0>();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // Order: S_0, S_1, then for each tile j: S_{j+2} (as soon as the softmax has read S_{j+1})
    // ahead of P_j.V_j (once P_j is in TMEM), so the next tile's scores are always ready when
    // the softmax asks for them.  The key ring holds tiles j .. j+2 meanwhile.
    bool ok = true;
    const int ks0 = half * KSTEPS;
    auto issue_s = [&](uint32_t gg) -> bool {
      const int st = gg % NS;
      if (!mbar_wait_warp(kv_full(st), (gg / NS) & 1, abort, wlim)) return false;
      if (!mbar_wait_warp(s_empty, (gg & 1) ^ 1, abort, wlim)) return false;
      tc_fence_after();
      fence_proxy_async();
      if (lane == 0) {
        const uint32_t stage = sbase + OFF_KV + st * KV_STAGE;
#pragma unroll 2
        for (int i = 0; i < KSTEPS; ++i) {
          const int ks = ks0 + i;                      // global 16-column step 0..35
          const uint32_t blk = (uint32_t)((ks >> 2) - blk0);
          const uint32_t off = (uint32_t)(ks & 3) * 32u;   // 16 columns = 32 bytes inside the atom
          const uint64_t bd = smem_desc(stage + blk * K_BLK + off, 1024, kLayoutSw128);
          mma_bf16_ts(tmem + COL_S, tmem + COL_Q + 8u * i, bd, IDESC_S, i > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
      }
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](uint32_t gg, bool first) -> bool {
      if (!mbar_wait_warp(p_full, gg & 1, abort, wlim)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t stage = sbase + OFF_KV + (gg % NS) * KV_STAGE;
#pragma unroll
        for (int kk = 0; kk < NK / 16; ++kk) {
          // V columns 256*half .. +255 are the stage's blocks 0..3 for both CTAs; keys 16kk..
          const uint64_t bd = smem_desc_lbo(stage + kk * 2048, K_BLK, 1024, kLayoutSw128);
          mma_bf16_ts(tmem + COL_O, tmem + COL_P + 8u * kk, bd, IDESC_PV, (!first || kk > 0) ? 1u : 0u);
        }
        mma_commit(kv_empty(gg % NS));
        mma_commit(pv_done);
      }
      __syncwarp();
      return true;
    };
    uint32_t g = 0, nq = 0;   // tiles, and items with tiles, issued so far
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      const Item I = geom(it);
      if (I.ntiles == 0) continue;
      if (!(ok = mbar_wait_warp(q_ready, nq & 1, abort, wlim))) break;   // this item's q is in TMEM
      ++nq;
      ok = issue_s(g);
      if (ok && I.ntiles > 1) ok = issue_s(g + 1);
      for (int j = 0; j < I.ntiles && ok; ++j) {
        if (j + 2 < I.ntiles && !(ok = issue_s(g + j + 2))) break;
        ok = issue_pv(g + j, j == 0);
      }
      g += I.ntiles;
    }
    // every MMA this warp issued must have finished before the TMEM is freed: after a normal
    // run the consumers have waited for all of them already, but after any role gave up (here or
    // elsewhere, now or later) some may still run
    if (lane == 0) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait_bounded(mma_drain, 0, 100000000ull);
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0-3)
    const int row = warp * 32 + lane;  // head
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_use = -INFINITY, l_run = 0.f;
    bool ok = true;
    const uint32_t sw = (uint32_t)(row & 7);
    // S_jj from TMEM into sv, then this warp's 32 rows of it into the partner's exchange buffer
    // jj&1: staged locally, one 8 KB bulk copy that completes the partner's per-warp barrier.
    // Sent one tile ahead, so the copy is in flight while the current tile is finished.
    auto load_send = [&](uint32_t jj, float (&sv)[NK]) -> bool {
      if (!mbar_wait_warp(s_full, jj & 1, abort, wlim)) return false;
      tc_fence_after();
      tmem_ld32(tmem + lane_off + COL_S, *reinterpret_cast<float(*)[32]>(sv));
      tmem_ld32(tmem + lane_off + COL_S + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
      tmem_ld_wait();
      launder(*reinterpret_cast<float(*)[32]>(sv));   // no use of the scores before the wait
      launder(*reinterpret_cast<float(*)[32]>(sv + 32));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      if (lane == 0 && jj >= 1) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");  // stage free
      __syncwarp();
      const uint32_t xs_row = sbase + OFF_XS + row * 256;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};\n" ::"r"(xs_row + ((c ^ sw) << 4)), "f"(sv[4 * c]),
                     "f"(sv[4 * c + 1]), "f"(sv[4 * c + 2]), "f"(sv[4 * c + 3]));
      fence_proxy_async();
      __syncwarp();
      bool good = true;
      if (lane == 0) {
        // the partner's warp has read what we sent last (tile jj-1): it read it before sending
        // tile jj itself, so this wait is short
        good = mbar_wait_cluster(x_free(warp), (jj & 1) ^ 1, abort, wlim);
        if (good) {
          const uint32_t off = (uint32_t)(warp * 32 * 256);
          asm volatile(
              "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
              "cp.async.bulk.commit_group;\n"
              ::"r"(map_to_cta(sbase + OFF_X + off, partner)), "r"(sbase + OFF_XS + off),
                "r"((uint32_t)(X_BYTES / 4)), "r"(map_to_cta(x_full(warp), partner))
              : "memory");
        }
      }
      return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
    };
    // Tile jj, first half: the partner's partial + ours -> masked scores and their max.
    auto part1 = [&](uint32_t jj, float (&sv)[NK], float& mt) -> bool {
      const int st = jj % NS;
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(x_full(warp), jj & 1, abort, wlim))) return false;
      {
        // both CTAs add the partials in column order (0..287 first): the same scores in both
        const uint32_t xrow = sbase + OFF_X + row * 256;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float4 v;
          asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                       : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                       : "r"(xrow + ((c ^ sw) << 4)));
          sv[4 * c] = half == 0 ? sv[4 * c] + v.x : v.x + sv[4 * c];
          sv[4 * c + 1] = half == 0 ? sv[4 * c + 1] + v.y : v.y + sv[4 * c + 1];
          sv[4 * c + 2] = half == 0 ? sv[4 * c + 2] + v.z : v.z + sv[4 * c + 2];
          sv[4 * c + 3] = half == 0 ? sv[4 * c + 3] + v.w : v.w + sv[4 * c + 3];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(x_full(warp), X_BYTES / 4);   // arm the next exchange
      if (!mbar_wait_warp(ids_ready(st), (jj / NS) & 1, abort, wlim)) return false;
      {   // tile max in the log2 domain (scaled)
        const bool all_valid = ids_s[NS * NK + 4 * st] != 0;
        if (!all_valid) {
          const uint32_t ids_addr = sbase + OFF_IDS + st * NK * 4;
#pragma unroll
          for (int c = 0; c < NK / 4; ++c) {
            int4 id4;
            asm volatile("ld.shared.v4.s32 {%0,%1,%2,%3}, [%4];\n"
                         : "=r"(id4.x), "=r"(id4.y), "=r"(id4.z), "=r"(id4.w) : "r"(ids_addr + 16 * c));
            if (id4.x < 0) sv[4 * c] = -INFINITY;
            if (id4.y < 0) sv[4 * c + 1] = -INFINITY;
            if (id4.z < 0) sv[4 * c + 2] = -INFINITY;
            if (id4.w < 0) sv[4 * c + 3] = -INFINITY;
          }
        }
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int i = 0; i < NK; i += 4) {
          m0 = fmaxf(m0, sv[i]); m1 = fmaxf(m1, sv[i + 1]); m2 = fmaxf(m2, sv[i + 2]); m3 = fmaxf(m3, sv[i + 3]);
        }
        mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * scale_log2;   // scale > 0 commutes with max
      }
      // every value of the partner's rows has been read (mt depends on all of them, in every
      // lane of this warp): the partner's warp may copy in again
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_after(map_to_cta(x_free(warp), partner), mt);
      return true;
    };
    // Tile jj (the item's tile j), second half: running max, P_jj = exp2(s - m) into TMEM.
    auto part2 = [&](uint32_t jj, int j, float (&sv)[NK], float mt) -> bool {
      // P.V of tile jj-1 has finished: the P columns are free and O holds the item's tiles < j
      if (jj >= 1) {
        if (!mbar_wait_warp(pv_done, (jj - 1) & 1, abort, wlim)) return false;
        tc_fence_after();
      }
      // Lazy rescale, decided for the whole warp: the O round trip through TMEM is a
      // warp-collective operation.  Every lane then moves to max(m_use, mt) with its own
      // alpha (1 where its max did not move; O and l are still 0 where m_use was -inf).
      const bool want = mt > m_use + kRescaleLog2 || (m_use == -INFINITY && mt > -INFINITY);
      if (__any_sync(0xffffffffu, want)) {
        const float m_new = fmaxf(m_use, mt);
        const float alpha = (m_use == -INFINITY) ? 0.f : ex2(m_use - m_new);
        if (j >= 1) {   // O already holds earlier tiles of this item: rescale it
#pragma unroll 1
          for (int c = 0; c < DVH; c += 32) {
            float o[32];
            tmem_ld32(tmem + lane_off + COL_O + c, o);
            tmem_ld_wait();
            launder(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tmem + lane_off + COL_O + c, o);
          }
        }
        l_run *= alpha;
        m_use = m_new;
      }
      // ---- P = exp2(s - m_use) as bf16 pairs (even key in the low half) into this lane's
      //      32 P columns: the A operand of the P.V MMA
      {
        const bool live = m_use != -INFINITY;
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0v = live ? ex2(fmaf(sv[2 * i], scale_log2, -m_use)) : 0.f;
          const float p1v = live ? ex2(fmaf(sv[2 * i + 1], scale_log2, -m_use)) : 0.f;
          l_run += p0v + p1v;
          pk[i] = pack2_bf16(p0v, p1v);
        }
        tmem_st32u(tmem + lane_off + COL_P, pk);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      return true;
    };
    // Per item: the next item's q goes to L2 ahead of time; this item's q into TMEM (the S MMAs
    // of the previous item have all finished: its last S has been read); then the previous
    // item's O out of TMEM, while the MMA already computes this item's first scores; then the
    // tiles.  Per tile j: part1(j), then the next tile's scores go out (their copy overlaps
    // part2(j)), then part2(j).  Two score arrays alternate between the tiles.
    float sa[NK], sb[NK];
    uint32_t g = 0;   // tiles served so far
    int prev_it = -1;   // the item written out at the start of the next pass
    float prev_m = -INFINITY, prev_l = 0.f;
    // one pass more than there are items: the last pass only writes out the last item
    for (int it = blockIdx.x;; it += gridDim.x) {
      const bool real = it < items && ok;
      Item I{};
      if (real) I = geom(it);
      if (real && warp == 0 && lane == 0 && it + (int)gridDim.x < items) {
        const int bt_next = (it + (int)gridDim.x) % nbt;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(q + (int64_t)bt_next * HQ * DQK),
                     "r"((uint32_t)(HQ * DQK * 2))
                     : "memory");
      }
      if (I.ntiles > 0) attn_load_q(q, I.bt, row, half, tmem, lane_off, q_ready, lane);
      if (prev_it >= 0) {
        const Item P = geom(prev_it);
        ok = attn_epilogue(P.bt, P.sp, P.ntiles, prev_m, prev_l, g - 1, ok, nbt, row, half, tmem, lane_off, pv_done,
                           abort, out, lse, part_o, part_lse);
      }
      if (!real || !ok) break;
      m_use = -INFINITY;
      l_run = 0.f;
      if (I.ntiles > 0) {
        const uint32_t g0 = g;
        float mt = -INFINITY;
        ok = load_send(g0, sa);
        for (int j = 0; j < I.ntiles && ok; j += 2) {
          if (!(ok = part1(g0 + j, sa, mt))) break;
          if (j + 1 < I.ntiles && !(ok = load_send(g0 + j + 1, sb))) break;
          if (!(ok = part2(g0 + j, j, sa, mt))) break;
          if (j + 1 >= I.ntiles) break;
          if (!(ok = part1(g0 + j + 1, sb, mt))) break;
          if (j + 2 < I.ntiles && !(ok = load_send(g0 + j + 2, sa))) break;
          if (!(ok = part2(g0 + j + 1, j + 1, sb, mt))) break;
        }
        g += I.ntiles;
      }
      prev_it = it;
      prev_m = m_use;
      prev_l = l_run;
    }
  }

  if (warp < 4 && lane == 0) asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");   // own copies landed
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  cluster_sync();   // neither CTA leaves while the partner may still touch its shared memory
}

}  // namespace

int launch_sparse_mla_tc(const uint16_t* q, const uint16_t* kv, int64_t kv_rs, int64_t kv_bs, int S_kv,
                         const int32_t* idx, int B, int T, int k, float sm_scale, uint16_t* out, float* lse,
                         void* ws, int splits, const PageMap& pm, cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaFuncSetAttribute(sparse_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  if (splits <= 0) splits = attn_num_splits(B, T, HQ, k);
  int kps = (k + splits - 1) / splits;
  kps = (kps + NK - 1) / NK * NK;
  const int64_t rows = (int64_t)B * T * HQ;
  // split partials: O_s as bf16 (normalised, so within bf16's range), then lse_s as fp32
  __nv_bfloat16* part_o = nullptr;
  float* part_lse = nullptr;
  if (splits > 1) {
    part_o = reinterpret_cast<__nv_bfloat16*>(ws);
    part_lse = reinterpret_cast<float*>(part_o + (int64_t)splits * rows * DV);
  }
  // persistent: one cluster (CTA pair) per two SMs, each serving items (query, key split) in turn
  const int nbt = B * T;
  const int items = nbt * splits;
  const int nclu = std::max(1, std::min(items, num_sms() / 2));
  dim3 grid((unsigned)nclu, 2, 1);
  sparse_mla_tc_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(kv), kv_rs, kv_bs, S_kv, idx, T, nbt,
      items, k, kps, sm_scale * 1.4426950408889634f, reinterpret_cast<__nv_bfloat16*>(out), lse, part_o, part_lse, pm);
  int st = check_launch();
  if (st != DSA_OK || splits == 1) return st;
  return launch_attn_combine(part_o, true, part_lse, splits, rows, DV, out, lse, stream);
}

void attn_tc_set_wait_limit(uint64_t ns) {
  const unsigned long long v = ns;
  cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v));
}

unsigned int attn_tc_take_status() {
  unsigned int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
  return v;
}

}  // namespace dsa
