// Exact top-K select per sequence: K largest fp32 values, ties to the lower position,
// returned as positions in ascending order padded with -1.
//
// Used for the indexer top-K ([PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로
// 줄이고 …", section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2": each Full or Reindex
// layer produces its own top-K indices) and for the candidate pool (section "계층적 희소
// 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기": the blocks with the highest block max).
//
// Values are mapped to order-preserving 32-bit keys. The scoring kernel has already built
// a histogram of the top 12 key bits per sequence. This kernel, launched with several CTAs
// per sequence:
//  1. finds the digit b* of the K-th largest key from that histogram (suffix sums);
//  2. streams its slice of the values: keys with digit > b* are certainly selected
//     ("sure", fewer than K in total), keys with digit == b* are candidates;
//  3. takes a ticket; the last CTA of the sequence resolves the candidates exactly with
//     three more radix passes on the key (8+8+4 bits) and, if the K-th key is tied, radix
//     passes on the position (lowest positions win), then bitonic-sorts the selected
//     positions and writes them. It also zeroes the histogram and counters, leaving the
//     workspace ready for the next call. No CTA ever waits on another.
#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"
#include "fp4kv_sm100.cuh"

namespace fp4kv {
namespace {

constexpr int kSelThreads = 512;
constexpr int kMaxSel = 4096;
constexpr int kMaxProblems = 2;

struct SelectArgs {
  SelectProblem p[kMaxProblems];
};

FP4KV_DEV int64_t n_values(const SelectProblem& P, int b) {
  int64_t len = P.seq_lens[b];
  if (len < 0) len = 0;
  if (P.mode == 0) return len < P.vstride ? len : P.vstride;
  if (P.mode == 1) {
    const int64_t nb = (len + 7) / 8;
    return nb < P.vstride ? nb : P.vstride;
  }
  return int64_t(P.npb) * 8;
}

FP4KV_DEV int64_t position_of(const SelectProblem& P, int b, int64_t i) {
  if (P.mode != 2) return i;
  const int64_t j = P.pool[int64_t(b) * P.npb + i / 8];
  return j * 8 + (i % 8);
}

// Block-wide: find the digit d (scanning from the highest digit down) at which the running
// count of `h[0..nbins)` reaches `r` (r >= 1). Returns d and the count strictly above d.
// If the total is below r, returns d = -1 and above = total.
__device__ void find_digit_desc(const uint32_t* h, int nbins, uint32_t r, int* d_out,
                                uint32_t* above_out, uint32_t* s_scan) {
  const int tid = threadIdx.x;
  const int per = (nbins + kSelThreads - 1) / kSelThreads;
  // thread tid owns the per-digit chunk counted from the top: digits [hi-per, hi)
  const int hi = nbins - tid * per;
  uint32_t sum = 0;
  for (int d = hi - 1; d >= hi - per && d >= 0; --d) sum += h[d];
  // inclusive scan over threads (thread 0 = highest digits)
  const int lane = tid & 31, w = tid >> 5;
  uint32_t x = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_scan[w] = x;
  __syncthreads();
  if (w == 0) {
    uint32_t v = lane < kSelThreads / 32 ? s_scan[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < kSelThreads / 32) s_scan[32 + lane] = v;  // inclusive warp prefix
  }
  __syncthreads();
  const uint32_t incl = x + (w > 0 ? s_scan[32 + w - 1] : 0u);
  const uint32_t excl = incl - sum;
  const uint32_t total = s_scan[32 + kSelThreads / 32 - 1];
  if (tid == 0) {
    s_scan[64] = 0xffffffffu;  // digit
    s_scan[65] = total;
  }
  __syncthreads();
  if (total >= r && excl < r && incl >= r) {
    uint32_t acc = excl;
    for (int d = hi - 1; d >= hi - per && d >= 0; --d) {
      if (acc + h[d] >= r) {
        s_scan[64] = static_cast<uint32_t>(d);
        s_scan[65] = acc;
        break;
      }
      acc += h[d];
    }
  }
  __syncthreads();
  *d_out = s_scan[64] == 0xffffffffu ? -1 : static_cast<int>(s_scan[64]);
  *above_out = s_scan[65];
  __syncthreads();
}

// Same, scanning from the lowest digit up (used for the smallest positions among ties).
__device__ void find_digit_asc(const uint32_t* h, int nbins, uint32_t r, int* d_out,
                               uint32_t* below_out, uint32_t* s_val) {
  if (threadIdx.x == 0) {
    uint32_t acc = 0;
    int dd = nbins - 1;
    for (int d = 0; d < nbins; ++d) {
      if (acc + h[d] >= r) { dd = d; break; }
      acc += h[d];
    }
    s_val[0] = static_cast<uint32_t>(dd);
    s_val[1] = acc;
  }
  __syncthreads();
  *d_out = static_cast<int>(s_val[0]);
  *below_out = s_val[1];
  __syncthreads();
}

// Block-wide ascending bitonic sort of N = kSelThreads * E keys held in shared memory.
// Each thread keeps E consecutive keys in registers: strides below E are exchanged inside
// the thread, strides up to 16 E through warp shuffles, and only the widest strides through
// shared memory (one barrier pair each). Every stage is unrolled at compile time.
template <typename T, int E>
__device__ void block_sort(T* s) {
  constexpr int N = kSelThreads * E;
  const int tid = threadIdx.x;
  T v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = s[tid * E + e];
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride >= 32 * E) {
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) s[tid * E + e] = v[e];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const T p = s[i ^ stride];
          const bool keep_min = ((i & stride) == 0) == ((i & size) == 0);
          v[e] = keep_min ? (v[e] < p ? v[e] : p) : (v[e] < p ? p : v[e]);
        }
      } else if (stride >= E) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const T p = __shfl_xor_sync(0xffffffffu, v[e], stride / E);
          const bool keep_min = ((i & stride) == 0) == ((i & size) == 0);
          v[e] = keep_min ? (v[e] < p ? v[e] : p) : (v[e] < p ? p : v[e]);
        }
      } else {
        T nv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const T p = v[e ^ stride];
          const bool keep_min = ((i & stride) == 0) == ((i & size) == 0);
          nv[e] = keep_min ? (v[e] < p ? v[e] : p) : (v[e] < p ? p : v[e]);
        }
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = nv[e];
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int e = 0; e < E; ++e) s[tid * E + e] = v[e];
  __syncthreads();
}

// candidate = (order key << 32) | value index
FP4KV_DEV uint32_t cand_key(uint64_t c) { return static_cast<uint32_t>(c >> 32); }
FP4KV_DEV int32_t cand_idx(uint64_t c) { return static_cast<int32_t>(c & 0xffffffffu); }

template <bool kShared>
FP4KV_DEV uint64_t load_cand(const uint64_t* c, uint32_t i) {
  if constexpr (kShared) return c[i];
  return __ldcg(reinterpret_cast<const unsigned long long*>(c) + i);
}

// Exact resolution of the candidates (all sharing the top 12 key bits `bstar`): finds the
// r-th largest key ustar among them and, when that key is tied, the largest position
// pos_star that is still taken (lowest positions win). Candidates live in shared memory
// (kShared) or, when too many, in global memory.
template <bool kShared>
__device__ void resolve_candidates(const SelectProblem& P, int b, const uint64_t* cand,
                                   uint32_t n_cand, uint32_t r, int bstar, uint32_t* s_hist,
                                   uint32_t* s_scan, uint32_t* ustar_out, int64_t* pos_star_out) {
  const int tid = threadIdx.x;
  uint32_t prefix = static_cast<uint32_t>(bstar);
  int consumed = kHistBits;
  const int widths[3] = {8, 8, 4};
  uint32_t cnt_eq = 0;
  for (int pass = 0; pass < 3; ++pass) {
    const int wbits = widths[pass];
    const int shift = 32 - consumed - wbits;
    const int nb = 1 << wbits;
    for (int i = tid; i < nb; i += kSelThreads) s_hist[i] = 0;
    __syncthreads();
    for (uint32_t c = tid; c < n_cand; c += kSelThreads) {
      const uint32_t key = cand_key(load_cand<kShared>(cand, c));
      if ((key >> (shift + wbits)) == prefix) atomicAdd(&s_hist[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    int d;
    uint32_t ab;
    find_digit_desc(s_hist, nb, r, &d, &ab, s_scan);
    r -= ab;
    cnt_eq = s_hist[d];
    prefix = (prefix << wbits) | static_cast<uint32_t>(d);
    consumed += wbits;
    __syncthreads();
  }
  *ustar_out = prefix;
  *pos_star_out = INT64_MAX;
  if (r < cnt_eq) {
    // lowest r positions among the keys equal to ustar: passes of 8 bits over 32 bits
    uint64_t pprefix = 0;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) s_hist[i] = 0;
      __syncthreads();
      for (uint32_t c = tid; c < n_cand; c += kSelThreads) {
        const uint64_t cv = load_cand<kShared>(cand, c);
        if (cand_key(cv) != prefix) continue;
        const uint64_t pos = static_cast<uint64_t>(position_of(P, b, cand_idx(cv)));
        if ((pos >> (shift + 8)) == pprefix) atomicAdd(&s_hist[(pos >> shift) & 255], 1u);
      }
      __syncthreads();
      int d;
      uint32_t below;
      find_digit_asc(s_hist, 256, r, &d, &below, s_scan);
      r -= below;
      pprefix = (pprefix << 8) | static_cast<uint64_t>(d);
    }
    *pos_star_out = static_cast<int64_t>(pprefix);
  }
}

// Appends the taken candidates to s_sel at *s_cnt (one shared atomic per warp).
template <bool kShared>
__device__ void collect_candidates(const SelectProblem& P, int b, const uint64_t* cand,
                                   uint32_t n_cand, bool take_all, uint32_t ustar,
                                   int64_t pos_star, uint64_t* s_sel, uint32_t* s_cnt) {
  const int lane = threadIdx.x & 31;
  for (uint32_t c0 = 0; c0 < n_cand; c0 += kSelThreads) {
    const uint32_t c = c0 + threadIdx.x;
    bool take = false;
    uint64_t item = 0;
    if (c < n_cand) {
      const uint64_t cv = load_cand<kShared>(cand, c);
      const int32_t i = cand_idx(cv);
      const int64_t pos = position_of(P, b, i);
      const uint32_t key = cand_key(cv);
      take = take_all || key > ustar || (key == ustar && pos <= pos_star);
      item = (static_cast<uint64_t>(pos) << 32) | static_cast<uint32_t>(i);
    }
    const uint32_t m = __ballot_sync(0xffffffffu, take);
    if (m == 0) continue;
    const int leader = __ffs(m) - 1;
    uint32_t base = 0;
    if (lane == leader) base = atomicAdd(s_cnt, static_cast<uint32_t>(__popc(m)));
    base = __shfl_sync(0xffffffffu, base, leader);
    const uint32_t slot = base + static_cast<uint32_t>(__popc(m & ((1u << lane) - 1u)));
    if (take && slot < kMaxSel) s_sel[slot] = item;
  }
}

constexpr int kCandSmem = 6144;  // candidates staged in shared memory when they fit
constexpr size_t kSelSmem = size_t(kMaxSel) * 8 + size_t(kCandSmem) * 8;

__global__ void __launch_bounds__(kSelThreads) k_topk_select(const SelectArgs args) {
  const SelectProblem& P = args.p[blockIdx.z];
  const int b = blockIdx.y;
  if (static_cast<int>(blockIdx.x) >= P.slices) return;
  // s_sel: the selected (position, index) pairs; its first 16 KiB also serve as the
  // histogram of phase 1 and of the radix passes (never live at the same time).
  extern __shared__ __align__(16) uint8_t sel_smem[];
  uint64_t* s_sel = reinterpret_cast<uint64_t*>(sel_smem);
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_sel);
  uint64_t* s_cand = s_sel + kMaxSel;
  __shared__ uint32_t s_scan[96];
  __shared__ uint32_t s_cnt;
  __shared__ bool s_last;
  const int tid = threadIdx.x;
  // a kernel launched after this one as a programmatic dependent may start its own
  // prologue now (it waits for this grid's completion before reading the results)
  griddep_launch_dependents();

  const int64_t n = n_values(P, b);
  const float* vals = P.values + int64_t(b) * P.vstride;
  uint32_t* hist = P.hist + int64_t(b) * kHistBins;
  uint32_t* ctr = P.counters + int64_t(b) * 4;
  int32_t* sure = P.sure + int64_t(b) * P.k;
  uint64_t* cand = reinterpret_cast<uint64_t*>(P.cand) + int64_t(b) * P.vstride;

  // 1. digit of the K-th largest key
  for (int i = tid; i < kHistBins; i += kSelThreads) s_hist[i] = __ldcg(hist + i);
  __syncthreads();
  int bstar;
  uint32_t above;
  find_digit_desc(s_hist, kHistBins, static_cast<uint32_t>(P.k), &bstar, &above, s_scan);
  // bstar == -1: fewer than K valid values; every valid value is "sure"

  // 2. filter this CTA's slice
  const int64_t lo = n * blockIdx.x / P.slices;
  const int64_t hi = n * (blockIdx.x + 1) / P.slices;
  // Each batch of 8 values per thread is classified in registers; one block-wide prefix
  // sum of the (sure, candidate) counts then gives every thread its output slots, and one
  // global atomic per list and batch reserves the CTA's range (appends racing on the
  // per-sequence counters would cost a memory round trip each).
  constexpr int kBatch = 8;
  __shared__ uint32_t s_wsum[kSelThreads / 32];
  __shared__ uint32_t s_base[2];
  const int lane = tid & 31, warp = tid >> 5;
  for (int64_t base = lo; base < hi; base += int64_t(kSelThreads) * kBatch) {
    float v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t i = base + int64_t(u) * kSelThreads + tid;
      v[u] = i < hi ? __ldg(vals + i) : -INFINITY;
    }
    uint32_t smask = 0, cmask = 0, keys[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t i = base + int64_t(u) * kSelThreads + tid;
      keys[u] = 0;
      if (i < hi && (v[u] != -INFINITY || P.mode != 2)) {
        keys[u] = order_key(v[u]);
        const int digit = static_cast<int>(keys[u] >> (32 - kHistBits));
        if (digit > bstar) smask |= 1u << u;
        else if (digit == bstar) cmask |= 1u << u;
      }
    }
    // counts packed as (sure << 16) | candidates: a batch holds at most 4096 of each
    const uint32_t cnt = (static_cast<uint32_t>(__popc(smask)) << 16) | static_cast<uint32_t>(__popc(cmask));
    uint32_t x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      uint32_t t = lane < kSelThreads / 32 ? s_wsum[lane] : 0u;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      if (lane < kSelThreads / 32) s_wsum[lane] = t;  // inclusive prefix over warps
      if (lane == kSelThreads / 32 - 1) {
        s_base[0] = (t >> 16) ? atomicAdd(&ctr[0], t >> 16) : 0u;
        s_base[1] = (t & 0xffffu) ? atomicAdd(&ctr[1], t & 0xffffu) : 0u;
      }
    }
    __syncthreads();
    const uint32_t excl = x - cnt + (warp > 0 ? s_wsum[warp - 1] : 0u);
    uint32_t so = s_base[0] + (excl >> 16), co = s_base[1] + (excl & 0xffffu);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int64_t i = base + int64_t(u) * kSelThreads + tid;
      if ((smask >> u) & 1u) {
        if (so < static_cast<uint32_t>(P.k)) sure[so] = static_cast<int32_t>(i);
        ++so;
      }
      if ((cmask >> u) & 1u) {
        if (co < static_cast<uint32_t>(P.vstride))
          cand[co] = (static_cast<uint64_t>(keys[u]) << 32) | static_cast<uint32_t>(i);
        ++co;
      }
    }
    __syncthreads();  // s_wsum and s_base are reused by the next batch
  }

  // 3. ticket: the last CTA of this sequence finalises
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t t = atomicAdd(&ctr[2], 1u);
    s_last = (t == static_cast<uint32_t>(P.slices - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const uint32_t n_sure = min(__ldcg(&ctr[0]), static_cast<uint32_t>(P.k));
  const uint32_t n_cand = min(__ldcg(&ctr[1]), static_cast<uint32_t>(P.vstride));
  const uint32_t r = static_cast<uint32_t>(P.k) > n_sure ? static_cast<uint32_t>(P.k) - n_sure : 0u;
  const bool take_all = n_cand <= r;
  const bool in_smem = n_cand <= static_cast<uint32_t>(kCandSmem);
  if (in_smem) {
    for (uint32_t c = tid; c < n_cand; c += kSelThreads)
      s_cand[c] = __ldcg(reinterpret_cast<const unsigned long long*>(cand) + c);
    __syncthreads();
  }
  uint32_t ustar = 0;
  int64_t pos_star = INT64_MAX;
  if (!take_all && r > 0) {
    if (in_smem)
      resolve_candidates<true>(P, b, s_cand, n_cand, r, bstar, s_hist, s_scan, &ustar, &pos_star);
    else
      resolve_candidates<false>(P, b, cand, n_cand, r, bstar, s_hist, s_scan, &ustar, &pos_star);
  }

  // collect the selected (position, value index) pairs: the sure list is compact and all
  // of it is taken (n_sure <= K <= kMaxSel); taken candidates are appended after it
  if (tid == 0) s_cnt = n_sure;
  for (uint32_t c = tid; c < n_sure; c += kSelThreads) {
    const int32_t i = __ldcg(sure + c);
    s_sel[c] = (static_cast<uint64_t>(position_of(P, b, i)) << 32) | static_cast<uint32_t>(i);
  }
  __syncthreads();
  if (r > 0 || take_all) {
    if (in_smem)
      collect_candidates<true>(P, b, s_cand, n_cand, take_all, ustar, pos_star, s_sel, &s_cnt);
    else
      collect_candidates<false>(P, b, cand, n_cand, take_all, ustar, pos_star, s_sel, &s_cnt);
  }
  __syncthreads();
  int m = static_cast<int>(s_cnt);
  if (m > P.k) m = P.k;
  const int nsort = m <= kSelThreads * 4 ? kSelThreads * 4 : kSelThreads * 8;
  int32_t* oi = P.out_idx + int64_t(b) * P.k;
  float* os = P.out_score ? P.out_score + int64_t(b) * P.k : nullptr;
  if (P.mode != 2) {
    // position == value index: sort 32-bit positions (padding sorts last)
    uint32_t* s_pos = reinterpret_cast<uint32_t*>(s_cand);
    for (int i = tid; i < nsort; i += kSelThreads)
      s_pos[i] = i < m ? static_cast<uint32_t>(s_sel[i] >> 32) : 0xffffffffu;
    __syncthreads();
    if (nsort == kSelThreads * 4) block_sort<uint32_t, 4>(s_pos);
    else block_sort<uint32_t, 8>(s_pos);
    for (int j = tid; j < P.k; j += kSelThreads) {
      if (j < m) {
        oi[j] = static_cast<int32_t>(s_pos[j]);
        if (os) os[j] = vals[s_pos[j]];
      } else {
        oi[j] = -1;
        if (os) os[j] = -INFINITY;
      }
    }
  } else {
    for (int i = m + tid; i < nsort; i += kSelThreads) s_sel[i] = ~0ull;
    __syncthreads();
    if (nsort == kSelThreads * 4) block_sort<uint64_t, 4>(s_sel);
    else block_sort<uint64_t, 8>(s_sel);
    for (int j = tid; j < P.k; j += kSelThreads) {
      if (j < m) {
        oi[j] = static_cast<int32_t>(s_sel[j] >> 32);
        if (os) os[j] = vals[static_cast<uint32_t>(s_sel[j] & 0xffffffffu)];
      } else {
        oi[j] = -1;
        if (os) os[j] = -INFINITY;
      }
    }
  }
  // leave the workspace zeroed for the next call
  for (int i = tid; i < kHistBins; i += kSelThreads) hist[i] = 0;
  if (tid < 4) ctr[tid] = 0;
}

}  // namespace

int select_slices(int64_t n_values, int B, int num_sms) {
  int64_t s = (2 * int64_t(num_sms)) / B;  // two CTAs per SM: one wave
  const int64_t cap = (n_values + 4095) / 4096;
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  if (s > 65535) s = 65535;
  return static_cast<int>(s);
}

cudaError_t launch_topk_select(const SelectProblem* probs, int n_probs, int B,
                               cudaStream_t stream) {
  if (n_probs < 1 || n_probs > kMaxProblems || B == 0) return cudaSuccess;
  SelectArgs args{};
  int gx = 1;
  for (int i = 0; i < n_probs; ++i) {
    args.p[i] = probs[i];
    if (probs[i].slices > gx) gx = probs[i].slices;
  }
  dim3 grid(gx, B, n_probs);
  cudaError_t e = cudaFuncSetAttribute(k_topk_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSelSmem));
  if (e != cudaSuccess) return e;
  k_topk_select<<<grid, kSelThreads, kSelSmem, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace fp4kv
