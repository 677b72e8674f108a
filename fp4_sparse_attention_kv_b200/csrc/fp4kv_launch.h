// Internal launch interface between the C ABI layer (api.cu) and the kernel files.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fp4kv {

cudaError_t launch_kv_quant_fp4(const uint16_t* x, int64_t n_rows, int d, int64_t x_stride,
                                const int64_t* dst_row, uint8_t* packed, uint8_t* scales,
                                int64_t cap_rows, int num_sms, cudaStream_t stream);
cudaError_t launch_swa_quant_fp8(const uint16_t* x, int64_t n_rows, int d, int64_t x_stride,
                                 const int64_t* dst_row, uint8_t* out, int64_t cap_rows, int num_sms,
                                 cudaStream_t stream);

// ----------------------------------------------------------------------------------------
// Indexer scoring (Full scan or pool gather), fused with the first-level histogram of the
// top-K select and, for the hierarchical Full layer, the block max over 8 positions.
// ----------------------------------------------------------------------------------------
struct IndexScoreParams {
  const void* q;            // [B][H_I][128] e4m3 codes or bf16 bits, or [B][H_I][64] e2m1 pairs
  const float* w;           // [B][H_I]
  int H_I;
  const void* keys;         // [B][cap][128] (bf16, e4m3) or [B][cap][64] (e2m1 pairs)
  int key_type;             // 0 bf16, 1 e4m3, 2 e2m1 with per-16 e4m3 scales
  const uint8_t* key_sf;    // e2m1: [B][cap][8] e4m3 scales
  const uint8_t* q_sf;      // e2m1: [B][H_I][8] e4m3 scales
  const float* key_scale;   // nullable [B][cap]
  int64_t cap;
  const int32_t* seq_lens;  // [B]
  int B;
  // pool mode (pool != nullptr): tile = 16 pool blocks of 8 rows
  const int32_t* pool;      // [B][npb]
  int npb;
  // outputs
  float* scores;            // [B][score_stride]; flat: index = position; pool: slot*8 + r
  int64_t score_stride;
  uint32_t* hist;           // nullable [B][4096]
  float* bmax;              // nullable [B][bmax_stride] (flat mode only)
  int64_t bmax_stride;
  uint32_t* bmax_hist;      // [B][4096] when bmax != nullptr
  // nullable [B][gmax_stride]: per group of 32 consecutive values (value index / 32) the
  // largest order key among its valid values (0 when none)
  uint32_t* gmax;
  int64_t gmax_stride;
  uint32_t* status;         // workspace status word
};
cudaError_t launch_index_score(const IndexScoreParams& p, int num_sms, cudaStream_t stream);

// ----------------------------------------------------------------------------------------
// Exact top-K select over per-segment fp32 values, given the first-level histogram: one
// kernel, one thread-block cluster per (problem, sequence).
// ----------------------------------------------------------------------------------------
struct SelectProblem {
  const float* values;      // [B][vstride], vstride a multiple of 8
  int64_t vstride;
  const int32_t* seq_lens;  // [B]
  int mode;                 // 0: n = seq_len; 1: n = ceil(seq_len / 8) (block ids);
                            // 2: n = npb*8 pool slots, position = pool[b][i/8]*8 + i%8
  const int32_t* pool;      // mode 2
  int npb;
  int k;
  const uint32_t* gmax;     // nullable [B][gstride]: largest order key per 32-value group
  int64_t gstride;          //   (groups below the K-th key's first digit are not read)
  uint32_t* hist;           // [B][4096] digit-1 histogram (from the scoring kernel); the
                            // select reads it and leaves it zeroed
  uint64_t* list;           // [B][vstride] overflow of the kept-entry lists
  int32_t* out_idx;         // [B][k]
  float* out_score;         // nullable [B][k]
  uint32_t* status;         // workspace status word (bit 0: a bounded wait gave up)
};
cudaError_t launch_topk_select(const SelectProblem* probs, int n_probs, int B, int num_sms, cudaStream_t stream);

// ----------------------------------------------------------------------------------------
// Sparse attention decode
// ----------------------------------------------------------------------------------------
struct AttnParams {
  const uint16_t* q;        // [B][H][d] bf16
  int B, H, d;
  const uint8_t* packed;    // [B][cap][d/2]
  const uint8_t* scales;    // [B][cap][d/16]
  int64_t cap;
  const int32_t* seq_lens;
  const int32_t* idx;       // [B][top_k]
  int top_k;
  // nullable: the sliding window's E4M3 rows [B][n_win][d] (ring slot = position % n_win),
  // attended in the same softmax as the selected rows by one extra chunk CTA (the last)
  const uint8_t* swa;
  int n_win;
  float sm_scale;
  float* out;               // [B][H][d]
  float* lse;               // nullable [B][H]
  // chunks of the top_k list, one CTA each (1 .. 16); the chunk CTAs of a (sequence, head
  // group) form one cluster and combine their partials after one cluster barrier
  int n_chunks;
  float* part_o;            // [B][n_hg][n_chunks][64][d] fp32 partial outputs
  float* part_ml;           // [B][n_hg][n_chunks][64][2] per-head reference and row sum
  uint32_t* status;
};
cudaError_t launch_sparse_attn(const AttnParams& p, int num_sms, cudaStream_t stream);

// ----------------------------------------------------------------------------------------
// Context-sharded decode: exact merge of per-range top-K candidates, and the log-sum-exp
// combine of per-range attention partials (csrc/shard.cu).
// ----------------------------------------------------------------------------------------
constexpr int kMaxShardParts = 64;
cudaError_t launch_topk_merge(const float* cand_score, const int32_t* cand_idx, int n_parts, int k_part,
                              const int32_t* part_base, int B, int top_k, int lo, int hi, int32_t* out_idx,
                              int32_t* out_local, float* out_score, cudaStream_t stream);
cudaError_t launch_lse_combine(const float* part_out, const float* part_lse, int n_parts, int64_t n_bh, int d,
                               float* out, float* lse, cudaStream_t stream);
// chunk CTAs (= cluster size) of the attention for these sizes
int attn_chunks(int B, int H, int top_k, int num_sms);

}  // namespace fp4kv
