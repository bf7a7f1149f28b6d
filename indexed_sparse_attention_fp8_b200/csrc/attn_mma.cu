// Sparse MQA / MLA attention over the selected keys (Stage 2 of "DeepSeek Sparse Attention",
// "GLM 5.2: How Four Co-Designed Mechanisms Beat Raw Scale"; the "China's First Frontier
// Model?" page, section "The Time has Come": each token attends only to the indexer's
// candidates).  All query heads share one KV head; in the MLA form V is the first d_v
// columns of the latent K row, so one gathered row serves both products.
//
// One CTA per (query, group of HG heads, key split).  Warp (hw, vh): heads hw*16..+16; for
// S = q.K^T it owns key columns vh*KT/2..+KT/2 of each tile, for O += P.V it owns V columns
// vh*DVW..+DVW.  The selected rows are gathered with 16-byte cp.async into an XOR-swizzled
// shared-memory ring (chunk c of row r lives at c ^ (r & 7)), so ldmatrix reads are free of
// bank conflicts.  Online softmax in fp32 (exp2 domain), bf16 P staged in shared memory.
// With several key splits each CTA writes a normalised fp32 partial and its log-sum-exp,
// and a combine kernel merges them.
#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace {

constexpr int kTargetCtas = 296;  // 2 x 148 SMs

// Status word of this kernel (bit 1: a selected id at or beyond the cache length was skipped);
// read and cleared by the host through dsa_device_status().
__device__ unsigned int g_attn_mma_status;

// A selected id as the gathers use it: ids at or beyond the cache's S_kv rows are skipped like
// a -1 (nothing outside the cache is read) and flagged in the status word.
__device__ __forceinline__ int checked_id(int key, int S_kv) {
  if (key >= S_kv) {
    atomicOr(&g_attn_mma_status, 2u);
    return -1;
  }
  return key;
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Byte offset of 16-byte chunk c of row r in a swizzled tile whose rows have `chunks` chunks.
__device__ __forceinline__ uint32_t swz(int r, int c, int chunks) {
  return (uint32_t)(r * chunks + (c ^ (r & 7))) * 16u;
}
// P tile: rows of KT bf16 (4 chunks); chunk c of row r lives at c ^ ((r >> 1) & 3).
__device__ __forceinline__ uint32_t pswz(int r, int c) { return (uint32_t)(r * 4 + (c ^ ((r >> 1) & 3))) * 16u; }

template <int D_QK, int D_V, int HG, bool LATENT>
struct Cfg {
  static constexpr int KT = 32;
  static constexpr int NWH = HG / 16;
  static constexpr int NWV = 2;
  static constexpr int NWARPS = NWH * NWV;
  static constexpr int THREADS = NWARPS * 32;
  static constexpr int DVW = D_V / NWV;
  static constexpr int STAGES = 2;   // double-buffered: the smaller footprint fits six CTAs per SM (three stages: four), which pays more than the deeper ring
  static constexpr int QCH = D_QK / 8;  // 16-byte chunks per q/K row
  static constexpr int VCH = D_V / 8;
  static constexpr int Q_BYTES = HG * D_QK * 2;
  static constexpr int K_TILE = KT * D_QK * 2;
  static constexpr int V_TILE = LATENT ? 0 : KT * D_V * 2;
  static constexpr int P_BYTES = HG * KT * 2;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * K_TILE;
  // With separate V rows, P lives in the current stage's K tile, free once the tile's scores
  // are computed (every warp has passed the barrier after its score reads before P is
  // written, and the next copy into that stage follows the barrier that ends the tile's P.V);
  // the smaller footprint fits one more CTA per SM.  In the latent form K is also V: P gets its
  // own buffer.
  static constexpr bool P_IN_K = !LATENT && P_BYTES <= K_TILE;
  static constexpr int OFF_P = OFF_V + STAGES * V_TILE;
  static constexpr int OFF_IDX = OFF_P + (P_IN_K ? 0 : P_BYTES);
  static constexpr int OFF_RED = OFF_IDX + STAGES * KT * 4;
  static constexpr int SMEM = OFF_RED + 2 * NWV * HG * 4;
  static_assert(QCH % 8 == 0 && VCH % 8 == 0, "rows must be whole 128-byte swizzle groups");
  static_assert(KT == 32 && NWV == 2, "tile split assumed below");
};

template <int D_QK, int D_V, int HG, bool LATENT>
__global__ void __launch_bounds__(Cfg<D_QK, D_V, HG, LATENT>::THREADS, 1)
sparse_attn_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv,
                       const __nv_bfloat16* __restrict__ vv, int64_t kv_rs, int64_t kv_bs,
                       int64_t v_rs, int64_t v_bs, int S_kv, const int32_t* __restrict__ idx, int T, int Hq,
                       int k, int keys_per_split, float scale_log2, __nv_bfloat16* __restrict__ out,
                       float* __restrict__ lse, float* __restrict__ part_o,
                       float* __restrict__ part_lse, PageMap pm) {
  using C = Cfg<D_QK, D_V, HG, LATENT>;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  int* idx_s = reinterpret_cast<int*>(smem + C::OFF_IDX);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);  // [2][NWV][HG]: max, then sums

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hw = warp % C::NWH, vh = warp / C::NWH;
  const int g = lane >> 2, tig = lane & 3;
  const int bt = blockIdx.x;            // b*T + t
  const int b = bt / T;
  const int hg = blockIdx.y;
  const int sp = blockIdx.z;
  const int kbeg = sp * keys_per_split;
  const int kend = min(k, kbeg + keys_per_split);
  const int ntiles = kend > kbeg ? (kend - kbeg + C::KT - 1) / C::KT : 0;

  const __nv_bfloat16* qrow = q + ((int64_t)bt * Hq + hg * HG) * D_QK;
  // contiguous: this sequence's cache rows; paged: rows of the shared page pools
  const __nv_bfloat16* kvb = pm.bt != nullptr ? kv : kv + (int64_t)b * kv_bs;
  const __nv_bfloat16* vb = LATENT ? kvb : (pm.bt != nullptr ? vv : vv + (int64_t)b * v_bs);
  // cache row of a (checked) selected id: itself, or its page's row; -1 stays -1, and an id
  // whose page id is out of range becomes -1 and is flagged
  auto cache_row = [&](int key) -> int {
    if (key < 0 || pm.bt == nullptr) return key;
    const int r = paged_row(pm, b, key);
    if (r < 0) atomicOr(&g_attn_mma_status, 2u);
    return r;
  };
  const int32_t* irow = idx + (int64_t)bt * k;

  // ---- async loads: q once, then one tile of gathered rows per stage
  for (int i = tid; i < HG * C::QCH; i += C::THREADS) {
    const int r = i / C::QCH, c = i % C::QCH;
    cp_async16(sbase + swz(r, c, C::QCH), qrow + (int64_t)r * D_QK + c * 8, 16);
  }
  // A tile's selected ids are all loaded (and their page rows looked up) before the first of
  // its row copies is issued: each copy is an asm statement the compiler keeps in order with
  // the loads around it, so loading each id right before its copy would put one memory round
  // trip per row into every tile.
  constexpr int NK_IT = (C::KT * C::QCH + C::THREADS - 1) / C::THREADS;
  constexpr int NV_IT = LATENT ? 1 : (C::KT * C::VCH + C::THREADS - 1) / C::THREADS;
  auto load_tile = [&](int tile, int stage) {
    const int p0 = kbeg + tile * C::KT;
    int krow[NK_IT], vrow[NV_IT];
#pragma unroll
    for (int u = 0; u < NK_IT; ++u) {
      const int i = tid + u * C::THREADS;
      const int p = p0 + i / C::QCH;
      krow[u] = (i < C::KT * C::QCH && p < kend) ? __ldg(irow + p) : -1;
    }
    if constexpr (!LATENT) {
#pragma unroll
      for (int u = 0; u < NV_IT; ++u) {
        const int i = tid + u * C::THREADS;
        const int p = p0 + i / C::VCH;
        vrow[u] = (i < C::KT * C::VCH && p < kend) ? __ldg(irow + p) : -1;
      }
    }
#pragma unroll
    for (int u = 0; u < NK_IT; ++u) krow[u] = cache_row(checked_id(krow[u], S_kv));
    if constexpr (!LATENT) {
#pragma unroll
      for (int u = 0; u < NV_IT; ++u) vrow[u] = cache_row(vrow[u] >= S_kv ? -1 : vrow[u]);   // flagged once above
    }
#pragma unroll
    for (int u = 0; u < NK_IT; ++u) {
      const int i = tid + u * C::THREADS;
      if (i < C::KT * C::QCH) {
        const int r = i / C::QCH, c = i % C::QCH;
        const int key = krow[u];
        const __nv_bfloat16* src = kvb + (int64_t)(key < 0 ? 0 : key) * kv_rs + c * 8;
        cp_async16(sbase + C::OFF_K + stage * C::K_TILE + swz(r, c, C::QCH), src, key < 0 ? 0 : 16);
        if (c == 0) idx_s[stage * C::KT + r] = key;
      }
    }
    if constexpr (!LATENT) {
#pragma unroll
      for (int u = 0; u < NV_IT; ++u) {
        const int i = tid + u * C::THREADS;
        if (i < C::KT * C::VCH) {
          const int r = i / C::VCH, c = i % C::VCH;
          const int key = vrow[u];
          const __nv_bfloat16* src = vb + (int64_t)(key < 0 ? 0 : key) * v_rs + c * 8;
          cp_async16(sbase + C::OFF_V + stage * C::V_TILE + swz(r, c, C::VCH), src, key < 0 ? 0 : 16);
        }
      }
    }
  };
#pragma unroll
  for (int s = 0; s < C::STAGES - 1; ++s) {
    if (s < ntiles) load_tile(s, s);
    cp_async_commit();
  }

  float o[C::DVW / 8][4];
#pragma unroll
  for (int i = 0; i < C::DVW / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const int row0 = hw * 16 + g;  // this thread's rows: row0 and row0 + 8 (within the head group)

  for (int j = 0; j < ntiles; ++j) {
    const int stage = j % C::STAGES;
    cp_async_wait<C::STAGES - 2>();
    __syncthreads();
    {
      const int nt = j + C::STAGES - 1;
      if (nt < ntiles) load_tile(nt, nt % C::STAGES);
      cp_async_commit();
    }
    const uint32_t ks_base = sbase + C::OFF_K + stage * C::K_TILE;

    // ---- S = q K^T for 16 heads x 16 keys
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int kc = 0; kc < D_QK / 16; ++kc) {
      uint32_t a[4], bq[4];
      ldsm_x4(a, sbase + swz(hw * 16 + (lane & 15), 2 * kc + (lane >> 4), C::QCH));
      ldsm_x4(bq, ks_base + swz(vh * 16 + (lane & 7) + ((lane >> 4) << 3), 2 * kc + ((lane >> 3) & 1), C::QCH));
      mma_bf16(sacc[0], a, bq[0], bq[1]);
      mma_bf16(sacc[1], a, bq[2], bq[3]);
    }
    // ---- mask, scale, tile max
    const int* ids = idx_s + stage * C::KT;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = vh * 16 + nt * 8 + 2 * tig + (e & 1);
        const float s = ids[col] >= 0 ? sacc[nt][e] * scale_log2 : -INFINITY;
        sacc[nt][e] = s;
        mx[e >> 1] = fmaxf(mx[e >> 1], s);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    if (tig == 0) {
      red[vh * HG + row0] = mx[0];
      red[vh * HG + row0 + 8] = mx[1];
    }
    __syncthreads();
    float alpha[2], mnew[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float mt = fmaxf(red[row0 + 8 * r], red[HG + row0 + 8 * r]);
      mnew[r] = fmaxf(m_run[r], mt);
      alpha[r] = (mnew[r] == -INFINITY) ? 1.f : exp2f(m_run[r] - mnew[r]);
      m_run[r] = mnew[r];
    }
    // ---- P = exp2(S - m), written to shared memory as bf16
    const uint32_t pbase = C::P_IN_K ? ks_base : sbase + C::OFF_P;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float mm = mnew[e >> 1];
        p[e] = (mm == -INFINITY) ? 0.f : exp2f(sacc[nt][e] - mm);
      }
      l_run[0] = l_run[0] * (nt == 0 ? alpha[0] : 1.f) + p[0] + p[1];
      l_run[1] = l_run[1] * (nt == 0 ? alpha[1] : 1.f) + p[2] + p[3];
      const int col = vh * 16 + nt * 8 + 2 * tig;
      const uint32_t a0 = pbase + pswz(row0, col >> 3) + (col & 7) * 2;
      const uint32_t a1 = pbase + pswz(row0 + 8, col >> 3) + (col & 7) * 2;
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(a0), "r"(pack_bf16(p[0], p[1])));
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(a1), "r"(pack_bf16(p[2], p[3])));
    }
#pragma unroll
    for (int i = 0; i < C::DVW / 8; ++i) {
      o[i][0] *= alpha[0]; o[i][1] *= alpha[0];
      o[i][2] *= alpha[1]; o[i][3] *= alpha[1];
    }
    __syncthreads();

    // ---- O += P V over the tile's KT keys, this warp's DVW columns
    const uint32_t vbase = LATENT ? ks_base : sbase + C::OFF_V + stage * C::V_TILE;
    constexpr int VROW = LATENT ? C::QCH : C::VCH;
#pragma unroll
    for (int kc = 0; kc < C::KT / 16; ++kc) {
      uint32_t a[4];
      ldsm_x4(a, pbase + pswz(hw * 16 + (lane & 15), 2 * kc + (lane >> 4)));
      const int vrow = kc * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
      for (int np = 0; np < C::DVW / 16; ++np) {
        uint32_t bv[4];
        ldsm_x4_t(bv, vbase + swz(vrow, (vh * C::DVW) / 8 + 2 * np + (lane >> 4), VROW));
        mma_bf16(o[2 * np], a, bv[0], bv[1]);
        mma_bf16(o[2 * np + 1], a, bv[2], bv[3]);
      }
    }
  }
  cp_async_wait<0>();

  // ---- finish: row sums across the quad and the partner warp
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
  }
  __syncthreads();
  if (tig == 0) {
    red[2 * HG + vh * HG + row0] = l_run[0];
    red[2 * HG + vh * HG + row0 + 8] = l_run[1];
  }
  __syncthreads();
  float inv[2], lse_r[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const float l = red[2 * HG + row0 + 8 * r] + red[3 * HG + row0 + 8 * r];
    inv[r] = l > 0.f ? 1.f / l : 0.f;
    lse_r[r] = l > 0.f ? (m_run[r] + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
  const int head0 = hg * HG + row0;
  if (part_o == nullptr) {
    __nv_bfloat16* orow0 = out + ((int64_t)bt * Hq + head0) * D_V + vh * C::DVW;
    __nv_bfloat16* orow1 = orow0 + 8 * D_V;
#pragma unroll
    for (int nt = 0; nt < C::DVW / 8; ++nt) {
      const int c = nt * 8 + 2 * tig;
      *reinterpret_cast<uint32_t*>(orow0 + c) = pack_bf16(o[nt][0] * inv[0], o[nt][1] * inv[0]);
      *reinterpret_cast<uint32_t*>(orow1 + c) = pack_bf16(o[nt][2] * inv[1], o[nt][3] * inv[1]);
    }
    if (lse != nullptr && vh == 0 && tig == 0) {
      lse[(int64_t)bt * Hq + head0] = lse_r[0];
      lse[(int64_t)bt * Hq + head0 + 8] = lse_r[1];
    }
  } else {
    const int64_t nbt = gridDim.x;
    float* prow0 = part_o + (((int64_t)sp * nbt + bt) * Hq + head0) * D_V + vh * C::DVW;
    float* prow1 = prow0 + 8 * D_V;
#pragma unroll
    for (int nt = 0; nt < C::DVW / 8; ++nt) {
      const int c = nt * 8 + 2 * tig;
      *reinterpret_cast<float2*>(prow0 + c) = make_float2(o[nt][0] * inv[0], o[nt][1] * inv[0]);
      *reinterpret_cast<float2*>(prow1 + c) = make_float2(o[nt][2] * inv[1], o[nt][3] * inv[1]);
    }
    if (vh == 0 && tig == 0) {
      part_lse[((int64_t)sp * nbt + bt) * Hq + head0] = lse_r[0];
      part_lse[((int64_t)sp * nbt + bt) * Hq + head0 + 8] = lse_r[1];
    }
  }
}

// Merge split-key partials: O = sum_s exp(lse_s - lse) O_s, lse = log sum_s exp(lse_s).  The
// partials O_s are fp32, or bf16 when bf16_parts (the MLA kernel's: half the bytes to write and
// read back; lse_s stay fp32).
__global__ void __launch_bounds__(128)
attn_combine_kernel(const void* __restrict__ part_o, bool bf16_parts, const float* __restrict__ part_lse, int splits,
                    int64_t rows, int d_v, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  // Launched as a programmatic dependent of the attention kernel: it may start while that
  // kernel drains, and waits here until the kernel has finished and its partials are visible.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int64_t row = blockIdx.x;  // (b*T + t)*Hq + h
  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) mx = fmaxf(mx, part_lse[s * rows + row]);
  float wsum = 0.f;
  float wts[16];
  for (int s = 0; s < splits; ++s) {
    const float l = part_lse[s * rows + row];
    wts[s] = (mx == -INFINITY || l == -INFINITY) ? 0.f : __expf(l - mx);
    wsum += wts[s];
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  for (int c = threadIdx.x * 2; c < d_v; c += blockDim.x * 2) {
    float2 acc = make_float2(0.f, 0.f);
    for (int s = 0; s < splits; ++s) {
      const int64_t at = (s * rows + row) * d_v + c;
      const float2 v = bf16_parts
                           ? __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
                                 reinterpret_cast<const __nv_bfloat16*>(part_o) + at))
                           : *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(part_o) + at);
      acc.x += wts[s] * v.x;
      acc.y += wts[s] * v.y;
    }
    *reinterpret_cast<uint32_t*>(out + row * d_v + c) = pack_bf16(acc.x * inv, acc.y * inv);
  }
  if (lse != nullptr && threadIdx.x == 0) lse[row] = wsum > 0.f ? mx + __logf(wsum) : -INFINITY;
}

}  // namespace

int launch_attn_combine(const void* part_o, bool bf16_parts, const float* part_lse, int splits, int64_t rows,
                        int d_v, uint16_t* out, float* lse, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(128);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap its launch with the
  attr[0].val.programmaticStreamSerializationAllowed = 1;             // attention kernel's tail
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, attn_combine_kernel, part_o, bf16_parts, part_lse, splits, rows, d_v,
                                           reinterpret_cast<__nv_bfloat16*>(out), lse);
  if (e != cudaSuccess) {
    count_launch();
    set_cuda_error(e);
    return DSA_ERR_CUDA;
  }
  return check_launch();
}

namespace {

template <int D_QK, int D_V, int HG, bool LATENT>
int launch_cfg(const uint16_t* q, const uint16_t* kv, const uint16_t* v, int64_t kv_rs, int64_t kv_bs,
               int64_t v_rs, int64_t v_bs, int S_kv, const int32_t* idx, int B, int T, int Hq, int k,
               float sm_scale, uint16_t* out, float* lse, void* ws, int splits, const PageMap& pm,
               cudaStream_t stream) {
  using C = Cfg<D_QK, D_V, HG, LATENT>;
  auto kern = sparse_attn_mma_kernel<D_QK, D_V, HG, LATENT>;
  static bool attr_set[64] = {};  // per device; the attribute is idempotent
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  if (splits <= 0) splits = attn_num_splits(B, T, Hq, k);
  int kps = (k + splits - 1) / splits;
  kps = (kps + C::KT - 1) / C::KT * C::KT;
  const int64_t rows = (int64_t)B * T * Hq;
  float* part_o = nullptr;
  float* part_lse = nullptr;
  if (splits > 1) {
    part_o = reinterpret_cast<float*>(ws);
    part_lse = part_o + (int64_t)splits * rows * D_V;
  }
  dim3 grid((unsigned)(B * T), Hq / HG, splits);
  const float scale_log2 = sm_scale * 1.4426950408889634f;
  kern<<<grid, C::THREADS, C::SMEM, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(kv),
      reinterpret_cast<const __nv_bfloat16*>(v), kv_rs, kv_bs, v_rs, v_bs, S_kv, idx, T, Hq, k, kps,
      scale_log2, reinterpret_cast<__nv_bfloat16*>(out), lse, part_o, part_lse, pm);
  int st = check_launch();
  if (st != DSA_OK || splits == 1) return st;
  return launch_attn_combine(part_o, false, part_lse, splits, rows, D_V, out, lse, stream);
}

}  // namespace

int attn_num_splits(int B, int T, int Hq, int k) {
  if (Hq == 128) {
    // tensor-core MLA kernel: one CTA pair per (query, split), one CTA per SM.  Aim for a
    // single wave of pairs and keep at least 8 key tiles per split, so the fixed per-CTA work
    // (q into TMEM, the output write) stays small next to the gathers.
    const int64_t pairs = (int64_t)B * T;
    int splits = 1;
    while (pairs * splits * 2 * 2 <= 148 && k / (splits * 2) >= 512 && splits < 16) splits *= 2;
    return splits;
  }
  const int64_t base = (int64_t)B * T * (Hq >= 64 ? Hq / 64 : 1);
  int splits = 1;
  while (base * splits < kTargetCtas && k / (splits * 2) >= 128 && splits < 16) splits *= 2;
  return splits;
}

size_t attn_workspace_bytes(int B, int T, int Hq, int d_v, int k, int splits) {
  if (splits <= 0) splits = attn_num_splits(B, T, Hq, k);
  if (splits == 1) return 0;
  const size_t rows = (size_t)B * T * Hq;
  return (size_t)splits * rows * (size_t)(d_v + 1) * sizeof(float);
}

int launch_sparse_attn(const uint16_t* q, const uint16_t* kv, const uint16_t* v, int64_t kv_rs,
                       int64_t kv_bs, int64_t v_rs, int64_t v_bs, int S_kv, const int32_t* idx, int B, int T,
                       int Hq, int d_qk, int d_v, int k, float sm_scale, uint16_t* out, float* lse,
                       void* ws, const PageMap& pm, cudaStream_t stream, int splits) {
  if (B == 0 || T == 0) return DSA_OK;
  if (Hq == 128 && d_qk == 576 && d_v == 512) {
    // MLA latent form only: V must be the first d_v columns of the K row (tensor-core kernel)
    if (v != nullptr) return DSA_ERR_UNSUPPORTED_SHAPE;
    return launch_sparse_mla_tc(q, kv, kv_rs, kv_bs, S_kv, idx, B, T, k, sm_scale, out, lse, ws, splits, pm, stream);
  }
  if (Hq == 16 && d_qk == 128 && d_v == 128) {
    if (v == nullptr)
      return launch_cfg<128, 128, 16, true>(q, kv, v, kv_rs, kv_bs, v_rs, v_bs, S_kv, idx, B, T, Hq, k,
                                            sm_scale, out, lse, ws, splits, pm, stream);
    return launch_cfg<128, 128, 16, false>(q, kv, v, kv_rs, kv_bs, v_rs, v_bs, S_kv, idx, B, T, Hq, k,
                                           sm_scale, out, lse, ws, splits, pm, stream);
  }
  return DSA_ERR_UNSUPPORTED_SHAPE;
}

unsigned int attn_mma_take_status() {
  unsigned int v = 0, zero = 0;
  cudaMemcpyFromSymbol(&v, g_attn_mma_status, sizeof(v));
  if (v) cudaMemcpyToSymbol(g_attn_mma_status, &zero, sizeof(zero));
  return v;
}

}  // namespace dsa
