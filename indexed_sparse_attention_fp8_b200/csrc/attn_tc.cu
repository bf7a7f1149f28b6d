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
//   warps 0-7  softmax: warp w owns 16 heads, TMEM lanes 32*(w%4) + 16*(w/4) .. +15 (its
//              warp slot's lane quadrant, one half of it), read in the 16x256b shape: thread
//              i holds heads r0 = base + i/4 and r0 + 8 and, of every 8-key group of a tile,
//              the keys 2*(i%4), +1 -- 2 heads x 16 keys.  First warps w and w+4 store their
//              quadrant's q columns into TMEM (each half of them).  Per tile j: (1) the
//              partner's partial of tile j (sent a tile earlier) + our own -> masked scores,
//              their row maxima over the quad (2 shuffles); a relaxed remote arrive, ordered
//              after every read of the partner's values by a data dependency, frees its
//              buffer; (2) our partial of tile j+1 from TMEM -> a local stage -> per warp,
//              one 4 KB bulk copy into the partner (completing that warp's barrier there), in
//              flight while (3) the running max moves only when a tile exceeds it by more
//              than 2^8 (then the warp's O rows are rescaled in TMEM) and P = exp2(S - m)
//              goes to TMEM as bf16 pairs (16x128b shape, which puts each thread's key pairs
//              where the P.V MMA reads them).  At the end O / l is written out (or a split
//              partial with its lse).
//   warps 8-10 gather: 16-byte cp.async of the selected rows into the 128-byte-swizzled
//              K-major layout the tensor core reads (also V's MN-major layout).
//   warp 11    TMEM owner and MMA issuer: S_0, S_1, then per tile the first K-steps of S_{j+2},
//              then P_j.V_j interleaved with its other K-steps.
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
constexpr int S_EARLY = 9;              // K-steps of S_{j+2} issued before P_j.V_j is interleaved
constexpr int KV_STAGE = BLKS * K_BLK;                 // 40960
constexpr int OFF_KV = 0;
constexpr int SMW = 8;                  // softmax warps: 2 per SM sub-partition, 16 heads each
constexpr int XW_BYTES = 16 * NK * 4;   // 4096: one warp's 16 heads x 64 keys of fp32 partial scores
constexpr int X_BYTES = SMW * XW_BYTES;                // 32768: one tile of fp32 partial scores
constexpr int OFF_XS = OFF_KV + NS * KV_STAGE;         // own partial, staged for the bulk copy out
constexpr int OFF_X = OFF_XS + X_BYTES;                // partner's partial, copied in
constexpr int OFF_MASK = OFF_X + X_BYTES;              // per stage: the tile's 64-slot validity mask
constexpr int OFF_BAR = OFF_MASK + 8 * NS;
constexpr int NBARS = 3 * NS + 6 + 2 * SMW;            // .. + s_full, s_empty, p_full, pv_done, q_ready,
                                                       //    drain; x_full and x_free per softmax warp
constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;       // + alignment slack
// Five warpgroups: 0-1 softmax (warps 0-7), 2 the MMA warp (8) and gather warps 9-11, 3-4 gather
// warps 12-19.  A tile's gather is bound by how many rows are in flight at once, not by its bytes,
// so it takes many warps; they need few registers, and the softmax warps many: the kernel starts
// at REGS_LAUNCH per thread, warpgroup 2 drops to REGS_MID, 3-4 to REGS_LOW, and 0-1 rise to
// REGS_HIGH, within the registers the block was launched with.
constexpr int THREADS = 640;
constexpr int MMA_WARP = SMW;           // warp 8
constexpr int GATHER_WARP0 = SMW + 1;   // warps 9..19
constexpr int GATHER_WARPS = THREADS / 32 - GATHER_WARP0;
constexpr int GATHER_THREADS = GATHER_WARPS * 32;
constexpr int REGS_LAUNCH = 96, REGS_MID = 72, REGS_LOW = 48, REGS_HIGH = 152;
static_assert(THREADS == 5 * 128, "warpgroup roles");
static_assert(2 * 128 * REGS_HIGH + 128 * REGS_MID + 2 * 128 * REGS_LOW <= THREADS * REGS_LAUNCH, "register split");
static_assert(THREADS * REGS_LAUNCH <= 65536, "register file");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S = 0;      // partial scores, NK columns
constexpr uint32_t COL_Q = 64;     // this CTA's 288 q columns as packed bf16 pairs: 144 columns
constexpr uint32_t COL_P = 224;    // P of one tile as packed bf16 pairs (the P.V MMA's A operand): 32 columns
constexpr uint32_t COL_O = 256;    // DVH output columns
constexpr float kRescaleLog2 = 8.0f;

static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert((OFF_KV % 1024) == 0 && (OFF_X % 128) == 0 && (OFF_XS % 128) == 0 && (OFF_BAR % 8) == 0, "alignment");
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
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
// 16 lanes x 64 fp32 columns in the 16x256b shape (the register order of tmem_ld_16x256b_x8).
__device__ __forceinline__ void tmem_st_16x256b_x8(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
      "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
      "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31]));
}
// 16 lanes x 32 columns in the 16x128b shape: register 2r goes to lane base + i/4, register
// 2r+1 to lane base + 8 + i/4, both at column 4r + i%4 (thread i of the warp).
__device__ __forceinline__ void tmem_st_16x128b_x8(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}
__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]));
}
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
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (mbar_test_wait_cluster(bar, parity)) return true;
  const uint64_t limit = *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns);
  if (limit < kImmediateNs) {
    *abort = 1;
    atomicOr(&g_status, 1u);
    return false;
  }
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

// This CTA's q columns of the query into TMEM (bf16 pairs packed per 32-bit column), then this
// warp's arrival on q_ready.  Warps w and w+4 share the TMEM lane quadrant w%4: each writes all
// 32 of its heads (32x32b shape, thread = head), warp w the first 144 of the CTA's 288 q
// columns and warp w+4 the other 144.
__device__ __forceinline__ void attn_load_q(const __nv_bfloat16* __restrict__ q, int bt, int quad, int hh, int half,
                                         uint32_t tmem, uint32_t q_ready, int lane) {
  const int head = 32 * quad + lane;
  const uint4* qsrc = reinterpret_cast<const uint4*>(q + ((int64_t)bt * HQ + head) * DQK + 288 * half + 144 * hh);
  const uint32_t taddr = tmem + ((uint32_t)(32 * quad) << 16) + COL_Q + 72u * hh;
  uint4 qa[18];   // 144 bf16 = 288 bytes (prefetched to L2 an item earlier)
#pragma unroll
  for (int i = 0; i < 18; ++i) qa[i] = __ldg(qsrc + i);
  uint32_t w[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) { w[4 * i] = qa[i].x; w[4 * i + 1] = qa[i].y; w[4 * i + 2] = qa[i].z; w[4 * i + 3] = qa[i].w; }
  tmem_st32u(taddr, w);
#pragma unroll
  for (int i = 0; i < 8; ++i) { w[4 * i] = qa[8 + i].x; w[4 * i + 1] = qa[8 + i].y; w[4 * i + 2] = qa[8 + i].z; w[4 * i + 3] = qa[8 + i].w; }
  tmem_st32u(taddr + 32, w);
  uint32_t w8[8];
#pragma unroll
  for (int i = 0; i < 2; ++i) { w8[4 * i] = qa[16 + i].x; w8[4 * i + 1] = qa[16 + i].y; w8[4 * i + 2] = qa[16 + i].z; w8[4 * i + 3] = qa[16 + i].w; }
  tmem_st8u(taddr + 64, w8);
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(q_ready);
}

// Epilogue of one item for this warp's 16 heads: waits for its last P.V, finishes the row sums
// over the quad, then O / l (or the split partial and its lse) out of TMEM in the 16x256b shape:
// per 64-column chunk, thread i writes columns 8r + 2*(i%4), +1 of its two heads.
__device__ __forceinline__ bool attn_epilogue(int bt, int sp, int ntiles, float m0, float m1, float l0, float l1,
                                           uint32_t g_last, bool good, int nbt, int r0, int qi, int half,
                                           uint32_t tmem, uint32_t lane_off, uint32_t pv_done, volatile int* abort,
                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                                           float* __restrict__ part_o, float* __restrict__ part_lse) {
  if (good && ntiles > 0) good = mbar_wait(pv_done, g_last & 1, abort, kWaitLimitNs);
  good = __all_sync(0xffffffffu, good);   // the TMEM reads below are warp-collective
  tc_fence_after();
  // each thread summed 16 of every tile's 64 keys: the quad holds the whole row
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const float lse0 = l0 > 0.f ? (m0 + log2f(l0)) * 0.69314718055994531f : -INFINITY;
  const float lse1 = l1 > 0.f ? (m1 + log2f(l1)) * 0.69314718055994531f : -INFINITY;
  const bool have_o = good && ntiles > 0;
  const int64_t orow0 = (int64_t)bt * HQ + r0, orow1 = orow0 + 8;
  const int64_t rows = (int64_t)nbt * HQ;
#pragma unroll 1
  for (int c = 0; c < DVH; c += 64) {
    float o[32];
    if (have_o) {
      tmem_ld_16x256b_x8(tmem + lane_off + COL_O + c, o);
      tmem_ld_wait();
      launder(o);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0.f;
    }
    const int col = half * DVH + c + 2 * qi;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (part_o == nullptr) {
        *reinterpret_cast<uint32_t*>(out + orow0 * DV + col + 8 * r) = pack2_bf16(o[4 * r] * inv0, o[4 * r + 1] * inv0);
        *reinterpret_cast<uint32_t*>(out + orow1 * DV + col + 8 * r) =
            pack2_bf16(o[4 * r + 2] * inv1, o[4 * r + 3] * inv1);
      } else {
        float* p0 = part_o + ((int64_t)sp * rows + orow0) * DV + col + 8 * r;
        float* p1 = part_o + ((int64_t)sp * rows + orow1) * DV + col + 8 * r;
        *reinterpret_cast<float2*>(p0) = make_float2(o[4 * r] * inv0, o[4 * r + 1] * inv0);
        *reinterpret_cast<float2*>(p1) = make_float2(o[4 * r + 2] * inv1, o[4 * r + 3] * inv1);
      }
    }
  }
  if (half == 0 && qi == 0) {
    if (part_o == nullptr) {
      if (lse != nullptr) {
        lse[orow0] = lse0;
        lse[orow1] = lse1;
      }
    } else {
      part_lse[(int64_t)sp * rows + orow0] = lse0;
      part_lse[(int64_t)sp * rows + orow1] = lse1;
    }
  }
  return good;
}

struct Item {
  int bt, sp, b, kbeg, kend, ntiles;
};

__global__ void __cluster_dims__(1, 2, 1) __maxnreg__(REGS_LAUNCH)
sparse_mla_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv, int64_t kv_rs,
                     int64_t kv_bs, int S_kv, const int32_t* __restrict__ idx, int T, int nbt, int items, int k,
                     int keys_per_split, float scale_log2, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                     float* __restrict__ part_o, float* __restrict__ part_lse, PageMap pm) {
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
  const uint32_t mma_drain = bar0 + 8u * (3 * NS + 5);   // completes when every issued MMA has
  // per softmax warp w (its 16 heads): the partner's values landed / the partner read ours
  auto x_full = [&](int w) { return bar0 + 8u * (3 * NS + 6 + w); };
  auto x_free = [&](int w) { return bar0 + 8u * (3 * NS + 6 + SMW + w); };
  volatile uint64_t* vmask = reinterpret_cast<volatile uint64_t*>(sgen + OFF_MASK);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sgen + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    mbar_init(s_empty, SMW);
    for (int w = 0; w < SMW; ++w) {
      mbar_init(x_full(w), 1);   // one expect-tx arrival per use, plus the partner's 4 KB
      mbar_init(x_free(w), 1);   // the partner's warp w, once it has read our values
    }
    mbar_init(p_full, SMW);
    mbar_init(pv_done, 1);
    mbar_init(q_ready, SMW);
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
  if (warp < SMW && lane == 0) mbar_arrive_expect_tx(x_full(warp), XW_BYTES);   // arm the first exchange
  cluster_sync();   // both CTAs' barriers exist (and are armed) before either signals the other
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The register split opens each warpgroup's branch (warpgroup-uniform, taken before any role
  // can give up), so the compiler sizes each role's code for its own register budget.
  if (warp >= SMW) {
    auto gather_role = [&]() {
    // ------------------------------------------------------------ gather (cp.async)
    // Warp gw copies rows gw, gw+GATHER_WARPS, ..: lane l moves 16-byte chunks l, l+32 of its
    // column range, so each row is read with coalesced requests.  A tile's ids come from one
    // coalesced load per warp, issued a tile ahead, and reach the rows through shuffles.
    const int gw = warp - GATHER_WARP0;
    bool ok = true;
    uint32_t g = 0;   // tiles gathered so far
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
    const Item I = geom(it);
    // contiguous: rows of this sequence's cache; paged: rows of the shared page pool
    const __nv_bfloat16* kvb = pm.bt != nullptr ? kv : kv + (int64_t)I.b * kv_bs;
    const int32_t* irow = idx + (int64_t)I.bt * k;
    // Selected id of slot r of tile j (-1 when empty), and through `row` the cache row to read.
    // Ids at or beyond the cache's S_kv rows, and ids whose page id is out of range, are
    // skipped like a -1 (nothing outside the cache is read) and flagged in the status word.
    auto load_id = [&](int j, int r, int& row) -> int {
      const int p = I.kbeg + j * NK + r;
      int id = (j < I.ntiles && p < I.kend) ? __ldg(irow + p) : -1;
      if (id >= S_kv) {
        atomicOr(&g_status, 2u);
        id = -1;
      }
      row = id;
      if (id >= 0 && pm.bt != nullptr) {
        row = paged_row(pm, I.b, id);
        if (row < 0) {
          atomicOr(&g_status, 2u);
          id = -1;
        }
      }
      return id;
    };
    int row_next0, row_next1;
    int id_next0 = load_id(0, lane, row_next0), id_next1 = load_id(0, lane + 32, row_next1);
    for (int j = 0; j < I.ntiles; ++j, ++g) {
      const int st = g % NS;
      const int id0 = id_next0, id1 = id_next1;
      const int row0 = row_next0, row1 = row_next1;
      id_next0 = load_id(j + 1, lane, row_next0);
      id_next1 = load_id(j + 1, lane + 32, row_next1);
      if (!(ok = mbar_wait_warp(kv_empty(st), ((g / NS) & 1) ^ 1, abort, kWaitLimitNs))) break;
      if (gw == 0) {
        // the tile's validity mask: bit r set iff slot r holds a key (the softmax masks the rest)
        const uint64_t m = (uint64_t)__ballot_sync(0xffffffffu, id0 >= 0) |
                           ((uint64_t)__ballot_sync(0xffffffffu, id1 >= 0) << 32);
        if (lane == 0) {
          vmask[st] = m;
          mbar_arrive(ids_ready(st));
        }
      }
      const uint32_t stage = sbase + OFF_KV + st * KV_STAGE;
#pragma unroll 1
      for (int r = gw; r < NK; r += GATHER_WARPS) {
        const int key = __shfl_sync(0xffffffffu, r < 32 ? id0 : id1, r & 31);
        const int crow = __shfl_sync(0xffffffffu, r < 32 ? row0 : row1, r & 31);
        const __nv_bfloat16* src = kvb + (int64_t)(key < 0 ? 0 : crow) * kv_rs;
        const int nbytes = key < 0 ? 0 : 16;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = ch_lo + lane + 32 * cc;
          if (c < ch_hi) {
            const uint32_t dst = stage + ((c >> 3) - blk0) * K_BLK + r * 128 + (((c & 7) ^ (r & 7)) << 4);
            cp_async16(dst, src + c * 8, nbytes);
          }
        }
      }
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(kv_full(st)) : "memory");
    }
    }
    cp_async_wait<0>();
    };
    if (warp < 12) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(REGS_MID));
      if (warp >= GATHER_WARP0) {
        gather_role();
      } else {
    // ------------------------------------------------------------ MMA issuer (warp MMA_WARP)
    // Order: S_0, S_1, then for each tile j: the first S_EARLY K-steps of S_{j+2} (as soon as the
    // softmax has read S_{j+1}), then -- once P_j is in TMEM -- P_j.V_j interleaved with the other
    // K-steps of S_{j+2}.  The tensor pipe runs the 64-key score MMAs and the MN-major P.V MMAs
    // side by side when they alternate, and the early K-steps cover the softmax's second half, so
    // the next tile's scores are ready when the softmax asks for them.  The key ring holds tiles
    // j .. j+2 meanwhile.
    bool ok = true;
    const int ks0 = half * KSTEPS;
    // K-steps i0 .. i1-1 of S_gg (lane 0)
    auto s_steps = [&](uint32_t gg, int i0, int i1) {
      const uint32_t stage = sbase + OFF_KV + (gg % NS) * KV_STAGE;
      for (int i = i0; i < i1; ++i) {
        const int ks = ks0 + i;                      // global 16-column step 0..35
        const uint32_t blk = (uint32_t)((ks >> 2) - blk0);
        const uint32_t off = (uint32_t)(ks & 3) * 32u;   // 16 columns = 32 bytes inside the atom
        const uint64_t bd = smem_desc(stage + blk * K_BLK + off, 1024, kLayoutSw128);
        mma_bf16_ts(tmem + COL_S, tmem + COL_Q + 8u * i, bd, IDESC_S, i > 0 ? 1u : 0u);
      }
    };
    // keys 16kk .. 16kk+15 of P_gg.V_gg (lane 0); V columns 256*half .. +255 are the stage's
    // blocks 0..3 for both CTAs
    auto pv_step = [&](uint32_t gg, bool first, int kk) {
      const uint32_t stage = sbase + OFF_KV + (gg % NS) * KV_STAGE;
      const uint64_t bd = smem_desc_lbo(stage + kk * 2048, K_BLK, 1024, kLayoutSw128);
      mma_bf16_ts(tmem + COL_O, tmem + COL_P + 8u * kk, bd, IDESC_PV, (!first || kk > 0) ? 1u : 0u);
    };
    auto wait_s = [&](uint32_t gg) -> bool {
      if (!mbar_wait_warp(kv_full(gg % NS), (gg / NS) & 1, abort, kWaitLimitNs)) return false;
      if (!mbar_wait_warp(s_empty, (gg & 1) ^ 1, abort, kWaitLimitNs)) return false;
      tc_fence_after();
      fence_proxy_async();
      return true;
    };
    auto issue_s = [&](uint32_t gg) -> bool {
      if (!wait_s(gg)) return false;
      if (lane == 0) {
        s_steps(gg, 0, KSTEPS);
        mma_commit(s_full);
      }
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](uint32_t gg, bool first) -> bool {
      if (!mbar_wait_warp(p_full, gg & 1, abort, kWaitLimitNs)) return false;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < NK / 16; ++kk) pv_step(gg, first, kk);
        mma_commit(kv_empty(gg % NS));
        mma_commit(pv_done);
      }
      __syncwarp();
      return true;
    };
    auto issue_s_pv = [&](uint32_t gs, uint32_t gpv, bool first) -> bool {
      if (!wait_s(gs)) return false;
      if (lane == 0) s_steps(gs, 0, S_EARLY);
      __syncwarp();
      if (!mbar_wait_warp(p_full, gpv & 1, abort, kWaitLimitNs)) return false;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < NK / 16; ++kk) {
          s_steps(gs, S_EARLY + kk, S_EARLY + kk + 1);
          pv_step(gpv, first, kk);
        }
        mma_commit(kv_empty(gpv % NS));   // both complete once every MMA issued so far has
        mma_commit(pv_done);
        s_steps(gs, S_EARLY + NK / 16, KSTEPS);
        mma_commit(s_full);
      }
      __syncwarp();
      return true;
    };
    uint32_t g = 0, nq = 0;   // tiles, and items with tiles, issued so far
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      const Item I = geom(it);
      if (I.ntiles == 0) continue;
      if (!(ok = mbar_wait_warp(q_ready, nq & 1, abort, kWaitLimitNs))) break;   // this item's q is in TMEM
      ++nq;
      ok = issue_s(g);
      if (ok && I.ntiles > 1) ok = issue_s(g + 1);
      for (int j = 0; j < I.ntiles && ok; ++j)
        ok = j + 2 < I.ntiles ? issue_s_pv(g + j + 2, g + j, j == 0) : issue_pv(g + j, j == 0);
      g += I.ntiles;
    }
    // every MMA this warp issued must have finished before the TMEM is freed: after a normal
    // run the consumers have waited for all of them already, but after any role gave up (here or
    // elsewhere, now or later) some may still run
    if (lane == 0) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait_bounded(mma_drain, 0, 100000000ull);
      }
    } else {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(REGS_LOW));
      gather_role();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(REGS_HIGH));
    // ------------------------------------------------------------ softmax + epilogue (warps 0-7)
    const int quad = warp & 3, hh = warp >> 2;
    const int base = 32 * quad + 16 * hh;          // first TMEM lane (head) of this warp
    const int qi = lane & 3;                       // key pair 2*qi, +1 of every 8-key group
    const int r0 = base + (lane >> 2);             // this thread's heads: r0 and r0 + 8
    const uint32_t lane_off = (uint32_t)base << 16;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;
    // this thread's 128 bytes of the warp's 4 KB in the exchange buffers; 16-byte chunk c sits at
    // c ^ (lane & 7), which spreads a warp's stores and loads over all banks
    const uint32_t xoff = (uint32_t)(warp * XW_BYTES + lane * 128);
    const uint32_t xsw = (uint32_t)(lane & 7);
    // S_jj from TMEM into sv (16x256b: sv[4r+e] = head r0, key 8r+2qi+e; sv[4r+2+e] = head r0+8),
    // then this warp's values into the partner's exchange buffer: staged locally, one 4 KB bulk
    // copy that completes the partner's per-warp barrier.  Sent one tile ahead, so the copy is in
    // flight while the current tile is finished.
    auto load_send = [&](uint32_t jj, float (&sv)[32]) -> bool {
      if (!mbar_wait_warp(s_full, jj & 1, abort, kWaitLimitNs)) return false;
      tc_fence_after();
      tmem_ld_16x256b_x8(tmem + lane_off + COL_S, sv);
      tmem_ld_wait();
      launder(sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      if (lane == 0 && jj >= 1) asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");  // stage free
      __syncwarp();
      const uint32_t xs = sbase + OFF_XS + xoff;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};\n" ::"r"(xs + ((c ^ xsw) << 4)), "f"(sv[4 * c]),
                     "f"(sv[4 * c + 1]), "f"(sv[4 * c + 2]), "f"(sv[4 * c + 3]));
      fence_proxy_async();
      __syncwarp();
      bool good = true;
      if (lane == 0) {
        // the partner's warp has read what we sent last (tile jj-1): it read it before sending
        // tile jj itself, so this wait is short
        good = mbar_wait_cluster(x_free(warp), (jj & 1) ^ 1, abort);
        if (good) {
          const uint32_t off = (uint32_t)(warp * XW_BYTES);
          asm volatile(
              "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
              "cp.async.bulk.commit_group;\n"
              ::"r"(map_to_cta(sbase + OFF_X + off, partner)), "r"(sbase + OFF_XS + off), "r"((uint32_t)XW_BYTES),
                "r"(map_to_cta(x_full(warp), partner))
              : "memory");
        }
      }
      return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
    };
    // Tile jj, first half: the partner's partial + ours -> masked scores and the row maxima.
    auto part1 = [&](uint32_t jj, float (&sv)[32], float& mt0, float& mt1) -> bool {
      const int st = jj % NS;
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(x_full(warp), jj & 1, abort))) return false;
      {
        // both CTAs add the partials in column order (0..287 first): the same scores in both
        const uint32_t xr = sbase + OFF_X + xoff;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float4 v;
          asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                       : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                       : "r"(xr + ((c ^ xsw) << 4)));
          sv[4 * c] = half == 0 ? sv[4 * c] + v.x : v.x + sv[4 * c];
          sv[4 * c + 1] = half == 0 ? sv[4 * c + 1] + v.y : v.y + sv[4 * c + 1];
          sv[4 * c + 2] = half == 0 ? sv[4 * c + 2] + v.z : v.z + sv[4 * c + 2];
          sv[4 * c + 3] = half == 0 ? sv[4 * c + 3] + v.w : v.w + sv[4 * c + 3];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(x_full(warp), XW_BYTES);   // arm the next exchange
      if (!mbar_wait_warp(ids_ready(st), (jj / NS) & 1, abort, kWaitLimitNs)) return false;
      {
        const uint64_t vm = vmask[st];
        if (vm != ~0ull) {   // empty slots (-1 ids) score -inf
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const uint32_t bits = (uint32_t)(vm >> (8 * r + 2 * qi));
            if (!(bits & 1u)) { sv[4 * r] = -INFINITY; sv[4 * r + 2] = -INFINITY; }
            if (!(bits & 2u)) { sv[4 * r + 1] = -INFINITY; sv[4 * r + 3] = -INFINITY; }
          }
        }
        float a = -INFINITY, b = -INFINITY;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          a = fmaxf(a, fmaxf(sv[4 * r], sv[4 * r + 1]));
          b = fmaxf(b, fmaxf(sv[4 * r + 2], sv[4 * r + 3]));
        }
        // a row's 64 keys are spread over the 4 threads of a quad
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, 2));
        mt0 = a * scale_log2;   // in the log2 domain; scale > 0 commutes with max
        mt1 = b * scale_log2;
      }
      // every value of the partner's buffer has been read (each lane's maxima depend on its own
      // loads, and the shuffles and the syncwarp join the lanes): the partner may copy in again
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_after(map_to_cta(x_free(warp), partner), mt0 + mt1);
      return true;
    };
    // Tile jj (the item's tile j), second half: running maxima, P_jj = exp2(s - m) into TMEM.
    auto part2 = [&](uint32_t jj, int j, float (&sv)[32], float mt0, float mt1) -> bool {
      // P.V of tile jj-1 has finished: the P columns are free and O holds the item's tiles < j
      if (jj >= 1) {
        if (!mbar_wait_warp(pv_done, (jj - 1) & 1, abort, kWaitLimitNs)) return false;
        tc_fence_after();
      }
      // Lazy rescale, decided for the whole warp: the O round trip through TMEM is a
      // warp-collective operation.  Every row then moves to max(m, mt) with its own factor
      // (1 where its max did not move; O and l are still 0 where m was -inf).
      const bool want = mt0 > m0 + kRescaleLog2 || (m0 == -INFINITY && mt0 > -INFINITY) ||
                        mt1 > m1 + kRescaleLog2 || (m1 == -INFINITY && mt1 > -INFINITY);
      if (__any_sync(0xffffffffu, want)) {
        const float n0 = fmaxf(m0, mt0), n1 = fmaxf(m1, mt1);
        const float a0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - n0);
        const float a1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - n1);
        if (j >= 1) {   // O already holds earlier tiles of this item: rescale this warp's rows
#pragma unroll 1
          for (int c = 0; c < DVH; c += 64) {
            float o[32];
            tmem_ld_16x256b_x8(tmem + lane_off + COL_O + c, o);
            tmem_ld_wait();
            launder(o);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              o[4 * r] *= a0; o[4 * r + 1] *= a0; o[4 * r + 2] *= a1; o[4 * r + 3] *= a1;
            }
            tmem_st_16x256b_x8(tmem + lane_off + COL_O + c, o);
          }
        }
        l0 *= a0;
        l1 *= a1;
        m0 = n0;
        m1 = n1;
      }
      // ---- P = exp2(s - m) as bf16 pairs: key pair 8r+2qi, +1 of head r0 is P column 4r+qi,
      //      exactly where the 16x128b shape puts register 2r (register 2r+1: head r0+8)
      {
        const bool live0 = m0 != -INFINITY, live1 = m1 != -INFINITY;
        uint32_t pk[16];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float p00 = live0 ? ex2(fmaf(sv[4 * r], scale_log2, -m0)) : 0.f;
          const float p01 = live0 ? ex2(fmaf(sv[4 * r + 1], scale_log2, -m0)) : 0.f;
          const float p10 = live1 ? ex2(fmaf(sv[4 * r + 2], scale_log2, -m1)) : 0.f;
          const float p11 = live1 ? ex2(fmaf(sv[4 * r + 3], scale_log2, -m1)) : 0.f;
          l0 += p00 + p01;
          l1 += p10 + p11;
          pk[2 * r] = pack2_bf16(p00, p01);
          pk[2 * r + 1] = pack2_bf16(p10, p11);
        }
        tmem_st_16x128b_x8(tmem + lane_off + COL_P, pk);
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
    float sa[32], sb[32];
    uint32_t g = 0;   // tiles served so far
    int prev_it = -1;   // the item written out at the start of the next pass
    float prev_m0 = -INFINITY, prev_m1 = -INFINITY, prev_l0 = 0.f, prev_l1 = 0.f;
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
      if (I.ntiles > 0) attn_load_q(q, I.bt, quad, hh, half, tmem, q_ready, lane);
      if (prev_it >= 0) {
        const Item P = geom(prev_it);
        ok = attn_epilogue(P.bt, P.sp, P.ntiles, prev_m0, prev_m1, prev_l0, prev_l1, g - 1, ok, nbt, r0, qi, half,
                           tmem, lane_off, pv_done, abort, out, lse, part_o, part_lse);
      }
      if (!real || !ok) break;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      if (I.ntiles > 0) {
        const uint32_t g0 = g;
        float mt0 = -INFINITY, mt1 = -INFINITY;
        ok = load_send(g0, sa);
        for (int j = 0; j < I.ntiles && ok; j += 2) {
          if (!(ok = part1(g0 + j, sa, mt0, mt1))) break;
          if (j + 1 < I.ntiles && !(ok = load_send(g0 + j + 1, sb))) break;
          if (!(ok = part2(g0 + j, j, sa, mt0, mt1))) break;
          if (j + 1 >= I.ntiles) break;
          if (!(ok = part1(g0 + j + 1, sb, mt0, mt1))) break;
          if (j + 2 < I.ntiles && !(ok = load_send(g0 + j + 2, sa))) break;
          if (!(ok = part2(g0 + j + 1, j + 1, sb, mt0, mt1))) break;
        }
        g += I.ntiles;
      }
      prev_it = it;
      prev_m0 = m0;
      prev_m1 = m1;
      prev_l0 = l0;
      prev_l1 = l1;
    }
  }

  if (warp < SMW && lane == 0) asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");   // own copies landed
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
    // The warpgroups' register split draws on the registers the block is launched with: launch
    // only a build whose register count covers it (otherwise the rising warpgroups would wait).
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, sparse_mla_tc_kernel) != cudaSuccess || fa.numRegs < REGS_LAUNCH)
      return DSA_ERR_CUDA;
    cudaFuncSetAttribute(sparse_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  if (splits <= 0) splits = attn_num_splits(B, T, HQ, k);
  int kps = (k + splits - 1) / splits;
  kps = (kps + NK - 1) / NK * NK;
  const int64_t rows = (int64_t)B * T * HQ;
  float* part_o = nullptr;
  float* part_lse = nullptr;
  if (splits > 1) {
    part_o = reinterpret_cast<float*>(ws);
    part_lse = part_o + (int64_t)splits * rows * DV;
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
  return launch_attn_combine(part_o, part_lse, splits, rows, DV, out, lse, stream);
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
