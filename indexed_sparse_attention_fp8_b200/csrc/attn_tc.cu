// Sparse MLA attention on the 5th-generation tensor cores (Stage 2 of "DeepSeek Sparse
// Attention", "GLM 5.2: How Four Co-Designed Mechanisms Beat Raw Scale": full attention over
// the selected tokens only).  All 128 query heads of a token share one latent row per key:
// K = the 576-wide row, V = its first 512 columns.
//
// TMEM holds 128 lanes x 512 fp32 columns, exactly the size of O = 128 heads x 512 dv, so one
// CTA cannot keep O and the scores together.  Each query is therefore served by a pair of
// CTAs: both compute the full score tile S = q K^T (M = 128 heads), and CTA h accumulates
// O[:, 256h .. 256h+255].  Per CTA, TMEM = 2 x 32 score columns + 256 output columns.
//
//   warps 0-3  softmax: thread = head.  Loads its S row from TMEM, masks skipped ids, keeps a
//              running max that is only moved when a tile exceeds it by more than 2^8 (then O
//              is rescaled in TMEM), writes P = exp2(S - m) as bf16 to shared memory, and at
//              the end normalises O and writes the output (or a split partial).
//   warps 4-7  gather: 16-byte cp.async of the selected latent rows into a 2-stage ring laid
//              out as the tensor core's 128-byte-swizzled K-major tile (which is also V's
//              MN-major tile), plus q once.
//   warp 8     TMEM owner and MMA issuer: S_j = q K_j^T (36 x M128 N32 K16), then
//              O += P_{j-1} V_{j-1} (2 x M128 N256 K16, V read MN-major from the same rows).
// All waits are bounded (see tc_common.cuh).
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace dsa {
namespace {

using namespace tc;

constexpr int HQ = 128, DQK = 576, DV = 512, DVH = 256;
constexpr int NK = 32;                  // keys per tile (MMA N of the score product)
constexpr int KB = DQK / 64;            // 64-column blocks of a row (9)
constexpr int ROWCH = DQK / 8;          // 16-byte chunks per row (72)
constexpr int Q_BLK = HQ * 128;         // one 64-column block of q: 128 rows x 128 B
constexpr int K_BLK = NK * 128;         // one 64-column block of a key tile: 32 rows x 128 B
constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + KB * Q_BLK;          // 147456
constexpr int KV_STAGE = KB * K_BLK;                // 36864
constexpr int OFF_P = OFF_KV + 2 * KV_STAGE;        // 221184
constexpr int P_BYTES = HQ * NK * 2;                // 8192 (rows of 64 B, 64-byte swizzle)
constexpr int OFF_BAR = OFF_P + P_BYTES;            // 229376
constexpr int NBARS = 12;
constexpr int OFF_IDS = OFF_BAR + NBARS * 8;          // two stages of NK selected ids
constexpr int OFF_MISC = OFF_IDS + 2 * NK * 4;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;    // + alignment slack
constexpr int THREADS = 288;
constexpr int GATHER_THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_S = 0;      // two score buffers of NK columns
constexpr uint32_t COL_O = 256;    // DVH output columns
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kRescaleLog2 = 8.0f;   // move the running max only when it grows by > 2^8

static_assert(SMEM_BYTES <= 232448, "shared memory budget");

constexpr uint32_t IDESC_S = instr_desc(128, NK, 1);                   // bf16, K-major A and B
constexpr uint32_t IDESC_PV = instr_desc(128, DVH, 1) | (1u << 16);    // B (V) MN-major

// Descriptor with an explicit leading byte offset (MN-major operands).
__device__ __forceinline__ uint64_t smem_desc_lbo(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1u << 46) | ((uint64_t)layout << 61);
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
      "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
      "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31]));
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(THREADS, 1)
sparse_mla_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv, int64_t kv_rs,
                     int64_t kv_bs, const int32_t* __restrict__ idx, int T, int k, int keys_per_split,
                     float scale_log2, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                     float* __restrict__ part_o, float* __restrict__ part_lse) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - sraw);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto kv_full = [&](int s) { return bar0 + 8u * s; };
  auto kv_empty = [&](int s) { return bar0 + 8u * (2 + s); };
  auto s_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto s_empty = [&](int s) { return bar0 + 8u * (6 + s); };
  const uint32_t p_full = bar0 + 8u * 8;
  const uint32_t pv_done = bar0 + 8u * 9;
  auto ids_ready = [&](int s) { return bar0 + 8u * (10 + s); };
  volatile int* ids_s = reinterpret_cast<volatile int*>(sgen + OFF_IDS);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(sgen + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bt = blockIdx.x;
  const int half = blockIdx.y;
  const int sp = blockIdx.z;
  const int b = bt / T;
  const int kbeg = sp * keys_per_split;
  const int kend = min(k, kbeg + keys_per_split);
  const int ntiles = kend > kbeg ? (kend - kbeg + NK - 1) / NK : 0;
  const int32_t* irow = idx + (int64_t)bt * k;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(kv_full(s), GATHER_THREADS);
      mbar_init(kv_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(s_empty(s), 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(ids_ready(0), 1);
    mbar_init(ids_ready(1), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(sbase + OFF_MISC, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ gather (cp.async)
    // Warp gw copies rows gw, gw+4, ..: lane l moves 16-byte chunks l, l+32, l+64 of a row,
    // so each row is read with coalesced requests.  A tile's 32 ids come from one coalesced
    // load per warp, issued a tile ahead, and reach the rows through shuffles.
    const int gw = warp - 4;
    const __nv_bfloat16* qrow = q + (int64_t)bt * HQ * DQK;
    for (int r = gw; r < HQ; r += 4) {
      const __nv_bfloat16* src = qrow + (int64_t)r * DQK;
      for (int c = lane; c < ROWCH; c += 32) {
        const uint32_t dst = sbase + OFF_Q + (c >> 3) * Q_BLK + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        cp_async16(dst, src + c * 8, 16);
      }
    }
    const __nv_bfloat16* kvb = kv + (int64_t)b * kv_bs;
    auto load_id = [&](int j) -> int {
      const int p = kbeg + j * NK + lane;
      return (j < ntiles && p < kend) ? __ldg(irow + p) : -1;
    };
    int id_next = load_id(0);
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int st = j & 1;
      const int id_cur = id_next;
      id_next = load_id(j + 1);
      if (!(ok = mbar_wait(kv_empty(st), ((j >> 1) & 1) ^ 1, abort, kWaitLimitNs))) break;
      if (gw == 0) {   // publish the tile's ids for the softmax warps
        ids_s[st * NK + lane] = id_cur;
        __syncwarp();
        if (lane == 0) mbar_arrive(ids_ready(st));
      }
      const uint32_t stage = sbase + OFF_KV + st * KV_STAGE;
#pragma unroll
      for (int i = 0; i < NK / 4; ++i) {
        const int r = gw + 4 * i;
        const int key = __shfl_sync(0xffffffffu, id_cur, r);
        const __nv_bfloat16* src = kvb + (int64_t)(key < 0 ? 0 : key) * kv_rs;
        const int nbytes = key < 0 ? 0 : 16;
#pragma unroll
        for (int cc = 0; cc < 3; ++cc) {
          const int c = lane + 32 * cc;
          if (c < ROWCH) {
            const uint32_t dst = stage + (c >> 3) * K_BLK + r * 128 + (((c & 7) ^ (r & 7)) << 4);
            cp_async16(dst, src + c * 8, nbytes);
          }
        }
      }
      // one arrival per gather thread, triggered when all its copies so far (q too) have landed
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(kv_full(st)) : "memory");
    }
    cp_async_wait<0>();
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = true;
    auto issue_pv = [&](int jj) -> bool {
      if (!mbar_wait(p_full, jj & 1, abort, kWaitLimitNs)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t stage = sbase + OFF_KV + (jj & 1) * KV_STAGE;
#pragma unroll
        for (int kk = 0; kk < NK / 16; ++kk) {
          const uint64_t ad = smem_desc(sbase + OFF_P + kk * 32, 512, kLayoutSw64);
          // V = this half's 256 columns: blocks 4*half .. 4*half+3 of the rows, keys 16kk..16kk+15
          const uint64_t bd = smem_desc_lbo(stage + (4 * half) * K_BLK + kk * 2048, K_BLK, 1024, kLayoutSw128);
          mma_bf16(tmem + COL_O, ad, bd, IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(kv_empty(jj & 1));
        mma_commit(pv_done);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < ntiles && ok; ++j) {
      const int st = j & 1;
      if (!(ok = mbar_wait(kv_full(st), (j >> 1) & 1, abort, kWaitLimitNs))) break;
      if (!(ok = mbar_wait(s_empty(st), ((j >> 1) & 1) ^ 1, abort, kWaitLimitNs))) break;
      tc_fence_after();
      fence_proxy_async();
      if (lane == 0) {
        const uint32_t stage = sbase + OFF_KV + st * KV_STAGE;
#pragma unroll 4
        for (int ks = 0; ks < DQK / 16; ++ks) {
          const uint32_t off = (ks & 3) * 32;   // 16 columns = 32 bytes inside the swizzle atom
          const uint64_t ad = smem_desc(sbase + OFF_Q + (ks >> 2) * Q_BLK + off, 1024, kLayoutSw128);
          const uint64_t bd = smem_desc(stage + (ks >> 2) * K_BLK + off, 1024, kLayoutSw128);
          mma_bf16(tmem + COL_S + st * NK, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full(st));
      }
      __syncwarp();
      if (j >= 1) ok = issue_pv(j - 1);
    }
    if (ok && ntiles > 0) ok = issue_pv(ntiles - 1);
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0-3)
    const int row = warp * 32 + lane;  // head
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_use = -INFINITY, l_run = 0.f;
    bool ok = true;
    const uint32_t prow = sbase + OFF_P + row * 64;
    for (int j = 0; j < ntiles; ++j) {
      const int st = j & 1;
      if (!(ok = mbar_wait(s_full(st), (j >> 1) & 1, abort, kWaitLimitNs))) break;
      tc_fence_after();
      float s[32];
      tmem_ld32(tmem + lane_off + COL_S + st * NK, s);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty(st));
      // mask skipped ids (negative entries and the ragged end), scale to the log2 domain
      if (!(ok = mbar_wait(ids_ready(st), (j >> 1) & 1, abort, kWaitLimitNs))) break;
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        s[i] = ids_s[st * NK + i] >= 0 ? s[i] * scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[i]);
      }
      // P of the previous tile must have been consumed (and O be stable) before writing P
      if (j >= 1 && !(ok = mbar_wait(pv_done, (j - 1) & 1, abort, kWaitLimitNs))) break;
      tc_fence_after();
      if (mt > m_use + kRescaleLog2 || (m_use == -INFINITY && mt > -INFINITY)) {
        const float alpha = (m_use == -INFINITY) ? 0.f : exp2f(m_use - mt);
        if (j >= 1 && m_use != -INFINITY) {   // O already holds earlier tiles: rescale it
#pragma unroll 1
          for (int c = 0; c < DVH; c += 32) {
            float o[32];
            tmem_ld32(tmem + lane_off + COL_O + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tmem + lane_off + COL_O + c, o);
          }
          tmem_st_wait();
        }
        l_run *= alpha;
        m_use = mt;
      }
      // P = exp2(s - m_use) -> bf16, 64-byte-swizzled rows of 32 keys
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float p0v = m_use == -INFINITY ? 0.f : exp2f(s[i] - m_use);
        const float p1v = m_use == -INFINITY ? 0.f : exp2f(s[i + 1] - m_use);
        l_run += p0v + p1v;
        pk[i >> 1] = pack2_bf16(p0v, p1v);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t dst = prow + ((c ^ ((row >> 1) & 3)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(dst), "r"(pk[4 * c]), "r"(pk[4 * c + 1]),
                     "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3]));
      }
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ---- epilogue: wait for the last P.V, normalise, write
    if (ok && ntiles > 0) ok = mbar_wait(pv_done, (ntiles - 1) & 1, abort, kWaitLimitNs);
    tc_fence_after();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    const float lse_r = l_run > 0.f ? (m_use + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    const bool have_o = ok && ntiles > 0;
    const int64_t orow = (int64_t)bt * HQ + row;
    if (part_o == nullptr) {
      __nv_bfloat16* dst = out + orow * DV + half * DVH;
#pragma unroll 1
      for (int c = 0; c < DVH; c += 32) {
        float o[32];
        if (have_o) {
          tmem_ld32(tmem + lane_off + COL_O + c, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
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
      if (lse != nullptr && half == 0) lse[orow] = lse_r;
    } else {
      const int64_t rows = (int64_t)gridDim.x * HQ;
      float* dst = part_o + ((int64_t)sp * rows + orow) * DV + half * DVH;
#pragma unroll 1
      for (int c = 0; c < DVH; c += 32) {
        float o[32];
        if (have_o) {
          tmem_ld32(tmem + lane_off + COL_O + c, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(dst + c + i) = make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
      }
      if (half == 0) part_lse[(int64_t)sp * rows + orow] = lse_r;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

int launch_sparse_mla_tc(const uint16_t* q, const uint16_t* kv, int64_t kv_rs, int64_t kv_bs, const int32_t* idx,
                         int B, int T, int k, float sm_scale, uint16_t* out, float* lse, void* ws,
                         cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaFuncSetAttribute(sparse_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int splits = attn_num_splits(B, T, HQ, k);
  int kps = (k + splits - 1) / splits;
  kps = (kps + NK - 1) / NK * NK;
  const int64_t rows = (int64_t)B * T * HQ;
  float* part_o = nullptr;
  float* part_lse = nullptr;
  if (splits > 1) {
    part_o = reinterpret_cast<float*>(ws);
    part_lse = part_o + (int64_t)splits * rows * DV;
  }
  dim3 grid((unsigned)(B * T), 2, splits);
  sparse_mla_tc_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(kv), kv_rs, kv_bs, idx, T, k,
      kps, sm_scale * 1.4426950408889634f, reinterpret_cast<__nv_bfloat16*>(out), lse, part_o, part_lse);
  int st = check_launch();
  if (st != DSA_OK || splits == 1) return st;
  return launch_attn_combine(part_o, part_lse, splits, rows, DV, out, lse, stream);
}

unsigned int attn_tc_take_status() {
  unsigned int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
  return v;
}

}  // namespace dsa
