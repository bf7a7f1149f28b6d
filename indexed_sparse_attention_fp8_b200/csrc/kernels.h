// Internal launchers of the DSA library (C++ linkage; the C ABI is in include/dsa.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace dsa {

// Options of the indexer launch beyond storing every score row (the defaults do that).
struct IndexerMode {
  int kstride = 1;               // read every kstride-th key row (the sampling pass of the fused
                                 // selection; S_max and pool are then given in sampled rows)
  const float* tau = nullptr;    // fused selection: per-row thresholds [B * t_count] ...
  float2* cand = nullptr;        // ... candidate rows [B * t_count, cap] (score, key id as bits)
  int* cnt = nullptr;            // ... candidates per row, zeroed before the launch
  int cap = 0;
  const int* row_flag = nullptr; // only work items holding a flagged row run (repair pass)
};

int launch_index_scores(const uint8_t* q_idx, const float* w, const uint8_t* k_idx,
                        const int32_t* ctx_len, int B, int T, int S_max, int H_I, int d_I, int pool,
                        int t_begin, int t_count, float* scores, int64_t ld, const PageMap& pm,
                        cudaStream_t stream, const IndexerMode& md = IndexerMode());

// row_flag (optional, [B * t_count]): only the rows whose flag is non-zero are selected.
int launch_topk(const float* scores, int64_t ld, const int32_t* ctx_len, int B, int T, int S_max,
                int pool, int t_begin, int t_count, int k, int32_t* idx, cudaStream_t stream,
                const int* row_flag = nullptr);

// Fused selection (indexer scores never written in full):
//  * per row, the r-th largest of the scores of every `stride`-th key row, or -inf when all
//    visible keys fit the candidate buffer of `cap` entries;
int launch_sample_threshold(const float* samples, int64_t lds, const int32_t* ctx_len, int B, int T, int S_eff,
                            int pool, int stride, int t_begin, int t_count, int r, int cap, float* tau,
                            cudaStream_t stream);
//  * per row, the exact top-k of its candidates (score, key id); rows with fewer than k
//    candidates, or more than cap, get fail = 1 and are left for the repair pass.
int launch_topk_cand(const float2* cand, const int* cnt, int cap, const int32_t* ctx_len, int B, int T, int S_max,
                     int pool, int t_begin, int t_count, int k, int32_t* idx, int* fail, cudaStream_t stream);

// Split count the attention uses for a problem by default (1 = no split, no workspace).
int attn_num_splits(int B, int T, int Hq, int k);
// Workspace of the attention at `splits` key splits (0 = the default count).
size_t attn_workspace_bytes(int B, int T, int Hq, int d_v, int k, int splits = 0);
// Argument and shape checks of dsa_sparse_attn at `splits` key splits (0 = default), without
// launching anything; the same status dsa_sparse_attn would return before its first launch.
int check_sparse_attn(const uint16_t* q, const uint16_t* kv, const uint16_t* v, int64_t kv_rs,
                      int64_t kv_bs, int64_t v_rs, int64_t v_bs, int S_kv, const int32_t* idx, int B,
                      int T, int Hq, int d_qk, int d_v, int k, const uint16_t* out, const void* ws,
                      size_t ws_bytes, const dsa_paging* paging, int splits = 0);
// Checks of a dsa_paging (NULL is valid); S is the logical rows the call needs per sequence.
int check_paging(const dsa_paging* paging, int S);
// Selected ids >= S_kv are skipped on the device (and flagged in the status word).
int launch_sparse_attn(const uint16_t* q, const uint16_t* kv, const uint16_t* v,
                       int64_t kv_row_stride, int64_t kv_batch_stride, int64_t v_row_stride,
                       int64_t v_batch_stride, int S_kv, const int32_t* idx, int B, int T, int Hq,
                       int d_qk, int d_v, int k, float sm_scale, uint16_t* out, float* lse, void* ws,
                       const PageMap& pm, cudaStream_t stream, int splits = 0);
// Reads and clears the status word of the mma.sync attention (bit 1: an id >= S_kv).
unsigned int attn_mma_take_status();
// Reads and clears the status word of the pool kernel (bit 1: a page id out of range).
unsigned int pool_take_status();

// Reads and clears the device status word of the tensor-core indexer.
unsigned int indexer_take_status();
// Time limit of the bounded waits in the tensor-core indexer / attention (test hook).
void indexer_set_wait_limit(uint64_t ns);
void attn_tc_set_wait_limit(uint64_t ns);
// Launches the bounded-wait probe (see dsa_debug_wait_timeout).
int launch_wait_timeout_probe(uint64_t limit_ns, cudaStream_t stream);

// Tensor-core sparse MLA attention (128 heads, latent 576 / V 512); same split rule.
int launch_sparse_mla_tc(const uint16_t* q, const uint16_t* kv, int64_t kv_rs, int64_t kv_bs, int S_kv,
                         const int32_t* idx, int B, int T, int k, float sm_scale, uint16_t* out, float* lse,
                         void* ws, int splits, const PageMap& pm, cudaStream_t stream);
unsigned int attn_tc_take_status();
// Merges split-key attention partials (normalised O, fp32 or bf16, and log-sum-exp per split).
int launch_attn_combine(const void* part_o, bool bf16_parts, const float* part_lse, int splits, int64_t rows,
                        int d_v, uint16_t* out, float* lse, cudaStream_t stream);

// Context parallelism: the exact top-k over the union of per-shard selections (n_parts lists of
// kc (score, global id) per row, part p at part_stride elements from part 0).
constexpr int kMergeMaxCand = 16384;   // n_parts * kc, the candidates a row's CTA holds
int launch_topk_merge(const float* cand_score, const int32_t* cand_id, int n_parts, int64_t part_stride, int kc,
                      const int32_t* ctx_len, int B, int T, int S_total, int t_begin, int t_count, int k, int32_t* idx,
                      cudaStream_t stream);
// The scores of a shard's selected keys and their global ids (local id + id_offset; -1 stays -1
// with score -inf).
int launch_gather_selected(const float* scores, int64_t ld, const int32_t* idx, int B, int T, int t_begin,
                           int t_count, int k, int id_offset, float* cand_score, int32_t* cand_id, cudaStream_t stream);
unsigned int cp_take_status();
unsigned int merge_take_status();
// Global key ids -> the ids within the shard [s0, s0 + s_len) (others -1).
int launch_idx_localize(const int32_t* idx, int64_t n, int s0, int s_len, int32_t* out, cudaStream_t stream);

// IndexPool over `pool` (2, 4 or 8) consecutive keys.
int launch_index_pool(const uint8_t* k_idx, int B, int S_max, int d_I, int pool, uint8_t* k_pool,
                      const PageMap& pm, cudaStream_t stream);
int launch_index_pool_tail(const uint8_t* k_idx, const int32_t* ctx_len, int B, int T, int S_max, int d_I, int pool,
                           uint8_t* k_pool, const PageMap& pm, cudaStream_t stream);

}  // namespace dsa
