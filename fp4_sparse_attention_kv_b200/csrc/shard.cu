// Context-sharded decode: when several GPUs split one sequence's context into position
// ranges, each runs the indexer top-K and the sparse attention over its own range; these
// two kernels join the ranges exactly.
//
//  * k_topk_merge: the exact top-K of the union of the per-range top-K lists. The union
//    holds the global top-K: a position among the global best K has fewer than K better
//    positions in all, so fewer than K in its own range, so its range kept it (ties are
//    broken by position in both, and a range's positions keep their global order).
//  * k_lse_combine: the attention over the union of disjoint row sets from the per-range
//    attentions: out = sum_r e^(lse_r - M) out_r / sum_r e^(lse_r - M), lse = M + ln(sum).
//
// Method: [PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로 줄이고 …", section
// "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2" (the indexer's top-K over all visible
// positions, attention over the selected ones); the split of the context across GPUs is this
// library's design, not the pages'.
#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"

namespace fp4kv {
namespace {

constexpr int kMergeThreads = 1024;

struct PartBases {
  int32_t v[kMaxShardParts];  // first global position of each part's range
};

// Ascending bitonic sort of n (a power of two) 64-bit keys in shared memory by the block.
__device__ void smem_bitonic(uint64_t* s, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const uint64_t a = s[i], c = s[j];
          const bool up = (i & size) == 0;
          if ((a > c) == up) {
            s[i] = c;
            s[j] = a;
          }
        }
      }
    }
  }
  __syncthreads();
}

// One CTA per sequence. Candidates are the parts' lists [n_parts][B][k_part] of range-local
// positions (negative: absent), made global by the part's base. Keys sort by score
// descending, then position ascending; the best top_k are re-keyed by position (their score
// kept in the low word) and sorted again, so the output is in ascending position order.
// out_local (nullable): the selection as positions local to [lo, hi), -1 elsewhere.
__global__ void __launch_bounds__(kMergeThreads) k_topk_merge(const float* __restrict__ cand_score,
                                                              const int32_t* __restrict__ cand_idx, int n_parts,
                                                              int k_part, int B, const PartBases bases,
                                                              int n_pow2, int top_k, int k_pow2, int lo, int hi,
                                                              int32_t* __restrict__ out_idx,
                                                              int32_t* __restrict__ out_local,
                                                              float* __restrict__ out_score) {
  extern __shared__ uint64_t s_keys[];
  uint64_t* s1 = s_keys;           // [n_pow2]
  uint64_t* s2 = s_keys + n_pow2;  // [k_pow2]
  const int b = blockIdx.x;
  const int n = n_parts * k_part;
  for (int i = threadIdx.x; i < n_pow2; i += blockDim.x) {
    uint64_t key = ~0ull;
    if (i < n) {
      const int r = i / k_part, j = i - r * k_part;
      const int64_t at = (int64_t(r) * B + b) * k_part + j;
      const int32_t pos = cand_idx[at];
      if (pos >= 0) key = (uint64_t(~order_key(cand_score[at])) << 32) | uint32_t(pos + bases.v[r]);
    }
    s1[i] = key;
  }
  smem_bitonic(s1, n_pow2);
  for (int i = threadIdx.x; i < k_pow2; i += blockDim.x) {
    uint64_t key = ~0ull;
    if (i < top_k && i < n_pow2) {
      const uint64_t k1 = s1[i];
      if (k1 != ~0ull) key = (uint64_t(uint32_t(k1)) << 32) | uint64_t(~uint32_t(k1 >> 32));
    }
    s2[i] = key;
  }
  smem_bitonic(s2, k_pow2);
  for (int i = threadIdx.x; i < top_k; i += blockDim.x) {
    const uint64_t k2 = s2[i];
    const bool valid = k2 != ~0ull;  // (a valid key's position is < 2^31)
    const int32_t pos = valid ? int32_t(k2 >> 32) : -1;
    out_idx[int64_t(b) * top_k + i] = pos;
    if (out_local != nullptr) out_local[int64_t(b) * top_k + i] = (valid && pos >= lo && pos < hi) ? pos - lo : -1;
    if (out_score != nullptr) out_score[int64_t(b) * top_k + i] = valid ? key_to_float(uint32_t(k2)) : -INFINITY;
  }
}

// One CTA per (sequence, head): weights from the parts' lse, then the weighted mean of their
// outputs over d. A part with lse = -inf (no row in its range) has weight 0.
__global__ void __launch_bounds__(128) k_lse_combine(const float* __restrict__ part_out,
                                                     const float* __restrict__ part_lse, int n_parts,
                                                     int64_t n_bh, int d, float* __restrict__ out,
                                                     float* __restrict__ lse) {
  const int64_t bh = blockIdx.x;
  float m = -INFINITY;
  for (int r = 0; r < n_parts; ++r) m = fmaxf(m, part_lse[int64_t(r) * n_bh + bh]);
  float sum = 0.0f;
  for (int r = 0; r < n_parts; ++r) {
    const float l = part_lse[int64_t(r) * n_bh + bh];
    sum += (m == -INFINITY || l == -INFINITY) ? 0.0f : expf(l - m);
  }
  const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = 0.0f;
    for (int r = 0; r < n_parts; ++r) {
      const float l = part_lse[int64_t(r) * n_bh + bh];
      if (m == -INFINITY || l == -INFINITY) continue;
      acc += expf(l - m) * part_out[(int64_t(r) * n_bh + bh) * d + c];
    }
    out[bh * d + c] = acc * inv;
  }
  if (lse != nullptr && threadIdx.x == 0) lse[bh] = sum > 0.0f ? m + logf(sum) : -INFINITY;
}

int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

}  // namespace

cudaError_t launch_topk_merge(const float* cand_score, const int32_t* cand_idx, int n_parts, int k_part,
                              const int32_t* part_base, int B, int top_k, int lo, int hi, int32_t* out_idx,
                              int32_t* out_local, float* out_score, cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  if (n_parts > kMaxShardParts) return cudaErrorInvalidValue;
  PartBases bases{};
  for (int r = 0; r < n_parts; ++r) bases.v[r] = part_base[r];
  const int n_pow2 = pow2_at_least(n_parts * k_part), k_pow2 = pow2_at_least(top_k);
  const size_t smem = sizeof(uint64_t) * size_t(n_pow2 + k_pow2);
  cudaError_t e = cudaFuncSetAttribute(k_topk_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_topk_merge<<<B, kMergeThreads, smem, stream>>>(cand_score, cand_idx, n_parts, k_part, B, bases, n_pow2, top_k,
                                                    k_pow2, lo, hi, out_idx, out_local, out_score);
  return cudaGetLastError();
}

cudaError_t launch_lse_combine(const float* part_out, const float* part_lse, int n_parts, int64_t n_bh, int d,
                               float* out, float* lse, cudaStream_t stream) {
  if (n_bh == 0) return cudaSuccess;
  k_lse_combine<<<static_cast<unsigned>(n_bh), 128, 0, stream>>>(part_out, part_lse, n_parts, n_bh, d, out, lse);
  return cudaGetLastError();
}

}  // namespace fp4kv
