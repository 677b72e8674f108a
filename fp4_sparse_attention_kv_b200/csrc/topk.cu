// Exact top-K select per sequence: K largest fp32 values, ties to the lower position,
// returned as positions in ascending order padded with -1.
//
// Used for the indexer top-K ([PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로
// 줄이고 …", section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2": each Full or Reindex
// layer produces its own top-K indices) and for the candidate pool (section "계층적 희소
// 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기": the blocks with the highest block max).
//
// Values are mapped to order-preserving 32-bit keys. The scoring kernel has already built a
// histogram of the top 12 key bits (digit 1) per sequence. Two kernels follow, each with
// several CTAs per sequence, every CTA owning one slice of the values:
//  filter  finds the digit-1 value b1 of the K-th largest key, keeps the keys with digit 1
//          >= b1 (in position order, in its slice's own region of the list array), counts
//          those above b1 ("sure") and builds a histogram of the next 12 bits (digit 2) of
//          the keys with digit 1 == b1;
//  finish  (a programmatic dependent of filter) finds the digit-2 value b2 of the K-th key,
//          drops from its slice list the keys with digit 1 == b1 and digit 2 < b2, and takes
//          a ticket; the last CTA of the sequence resolves the few keys left in the (b1, b2)
//          bin exactly (the last 8 key bits, then the lowest positions among equal keys),
//          and writes the selection by one ordered compaction of the slice lists. Slices are
//          in position order and each list is in position order, so positions come out
//          ascending without a sort (the pool mode, whose positions need not grow with the
//          value index, sorts its at most 4096 selected pairs). That CTA also zeroes the
//          histograms and counters, leaving the workspace ready for the next call.
// No CTA ever waits on another CTA.
#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"
#include "fp4kv_sm100.cuh"

namespace fp4kv {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kPer = 8;                         // consecutive values per thread and batch
constexpr int kBatchVals = kSelThreads * kPer;  // 4096
constexpr int kMaxSel = 4096;
constexpr int kMaxProblems = 2;
constexpr int kStage = 6144;  // kept entries the finishing CTA stages in shared memory

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

// Slice s of n values: [s * per, min(n, (s + 1) * per)), per a multiple of 8.
FP4KV_DEV int64_t slice_per(int64_t n, int slices) {
  const int64_t q = int64_t(slices) * 8;
  return (n + q - 1) / q * 8;
}

FP4KV_DEV int64_t position_of(const SelectProblem& P, int b, int64_t i) {
  if (P.mode != 2) return i;
  const int64_t j = P.pool[int64_t(b) * P.npb + i / 8];
  return j * 8 + (i % 8);
}

// entry = (order key << 32) | value index
FP4KV_DEV uint32_t ent_key(uint64_t c) { return static_cast<uint32_t>(c >> 32); }
FP4KV_DEV int32_t ent_idx(uint64_t c) { return static_cast<int32_t>(c & 0xffffffffu); }
FP4KV_DEV int digit1(uint32_t key) { return static_cast<int>(key >> 20); }
FP4KV_DEV int digit2(uint32_t key) { return static_cast<int>((key >> 8) & 0xfffu); }

// Block-wide exclusive prefix sum in thread order; *total receives the block sum.
// Every thread of the block must call it (it contains barriers).
FP4KV_DEV uint32_t block_excl_scan(uint32_t v, uint32_t* s_wsum, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < kSelWarps ? s_wsum[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kSelWarps) s_wsum[lane] = t;
  }
  __syncthreads();
  const uint32_t excl = x - v + (warp > 0 ? s_wsum[warp - 1] : 0u);
  *total = s_wsum[kSelWarps - 1];
  __syncthreads();
  return excl;
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
    uint32_t v = lane < kSelWarps ? s_scan[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < kSelWarps) s_scan[32 + lane] = v;  // inclusive warp prefix
  }
  __syncthreads();
  const uint32_t incl = x + (w > 0 ? s_scan[32 + w - 1] : 0u);
  const uint32_t excl = incl - sum;
  const uint32_t total = s_scan[32 + kSelWarps - 1];
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

// The same search over a 4096-bin histogram in global memory, read straight into registers:
// thread t owns the 8 bins [4096 - 8 (t + 1), 4096 - 8 t) (two 16-byte loads), so no
// shared-memory copy is made and the crossing thread finds the digit in its own registers.
// Also returns the count of the found bin (0 if none).
__device__ void find_digit_desc_g(const uint32_t* g_hist, uint32_t r, int* d_out, uint32_t* above_out,
                                  uint32_t* count_out, uint32_t* s_scan) {
  static_assert(kHistBins == kSelThreads * 8, "8 bins per thread");
  const int tid = threadIdx.x;
  const int lo = kHistBins - 8 * (tid + 1);
  const uint4 a = __ldcg(reinterpret_cast<const uint4*>(g_hist + lo));
  const uint4 c = __ldcg(reinterpret_cast<const uint4*>(g_hist + lo + 4));
  const uint32_t h[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
  uint32_t sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) sum += h[i];
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
    uint32_t v = lane < kSelWarps ? s_scan[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < kSelWarps) s_scan[32 + lane] = v;  // inclusive warp prefix
    if (lane == 0) {
      s_scan[64] = 0xffffffffu;  // digit
      s_scan[65] = 0;            // count above it
      s_scan[66] = 0;            // its count
    }
  }
  __syncthreads();
  const uint32_t incl = x + (w > 0 ? s_scan[32 + w - 1] : 0u);
  const uint32_t excl = incl - sum;
  const uint32_t total = s_scan[32 + kSelWarps - 1];
  if (total < r) {
    if (tid == 0) s_scan[65] = total;
  } else if (excl < r && incl >= r) {
    uint32_t acc = excl;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      if (acc + h[i] >= r) {
        s_scan[64] = static_cast<uint32_t>(lo + i);
        s_scan[65] = acc;
        s_scan[66] = h[i];
        break;
      }
      acc += h[i];
    }
  }
  __syncthreads();
  *d_out = s_scan[64] == 0xffffffffu ? -1 : static_cast<int>(s_scan[64]);
  *above_out = s_scan[65];
  *count_out = s_scan[66];
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
// shared memory (one barrier pair each).
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

// --------------------------------------------------------------------------------------
// filter
// --------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kSelThreads) k_select_filter(const SelectArgs args) {
  // the finishing kernel is a programmatic dependent: it may be scheduled from now on
  griddep_launch_dependents();
  griddep_wait();  // this grid is one too: the scores and histograms are complete past here
  const SelectProblem& P = args.p[blockIdx.z];
  const int b = blockIdx.y, s = blockIdx.x;
  if (s >= P.slices) return;
  __shared__ __align__(16) uint32_t s_h[kHistBins];  // digit-1 histogram, then this slice's digit-2 one
  __shared__ uint32_t s_scan[96];
  __shared__ uint32_t s_wsum[kSelWarps];
  const int tid = threadIdx.x;

  const int64_t n = n_values(P, b);
  const int64_t per = slice_per(n, P.slices);
  const int64_t lo = per * s;
  const int64_t hi = lo + per < n ? lo + per : n;
  const float* vals = P.values + int64_t(b) * P.vstride;
  uint32_t* ctr = P.counters + int64_t(b) * kSelCounters;
  uint64_t* list = P.list + int64_t(b) * P.vstride;

  // digit 1 of the K-th largest key (b1 = -1: fewer than K valid values, all are kept)
  for (int i = tid; i < kHistBins; i += kSelThreads) s_h[i] = 0;
  int b1;
  uint32_t above, b1_count;
  find_digit_desc_g(P.hist + int64_t(b) * kHistBins, static_cast<uint32_t>(P.k), &b1, &above, &b1_count, s_scan);
  (void)above;
  (void)b1_count;

  // keys with digit 1 >= b1, in position order, into list[lo ..)
  uint32_t run = 0, n_sure = 0;
  // the next batch's values are loaded before this batch is classified and compacted
  float4 na = make_float4(0.f, 0.f, 0.f, 0.f), nc = na;
  if (lo + int64_t(tid) * kPer < hi) {  // a multiple of 8 below vstride (a multiple of 8)
    na = __ldg(reinterpret_cast<const float4*>(vals + lo + int64_t(tid) * kPer));
    nc = __ldg(reinterpret_cast<const float4*>(vals + lo + int64_t(tid) * kPer + 4));
  }
  for (int64_t base = lo; base < hi; base += kBatchVals) {
    const int64_t i0 = base + int64_t(tid) * kPer;
    const float v[kPer] = {na.x, na.y, na.z, na.w, nc.x, nc.y, nc.z, nc.w};
    if (i0 + kBatchVals < hi) {
      na = __ldg(reinterpret_cast<const float4*>(vals + i0 + kBatchVals));
      nc = __ldg(reinterpret_cast<const float4*>(vals + i0 + kBatchVals + 4));
    }
    uint32_t keep = 0, keys[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      keys[u] = 0;
      if (i0 + u < hi && (P.mode != 2 || v[u] != -INFINITY)) {
        keys[u] = order_key(v[u]);
        const int d = digit1(keys[u]);
        if (d > b1) {
          keep |= 1u << u;
          ++n_sure;
        } else if (d == b1) {
          keep |= 1u << u;
          atomicAdd(&s_h[digit2(keys[u])], 1u);
        }
      }
    }
    uint32_t total;
    uint32_t o = run + block_excl_scan(static_cast<uint32_t>(__popc(keep)), s_wsum, &total);
#pragma unroll
    for (int u = 0; u < kPer; ++u)
      if ((keep >> u) & 1u)
        list[lo + o++] = (static_cast<uint64_t>(keys[u]) << 32) | static_cast<uint32_t>(i0 + u);
    run += total;
  }
  uint32_t sure_total;
  block_excl_scan(n_sure, s_wsum, &sure_total);  // (block sum)
  if (tid == 0) {
    P.cnt1[int64_t(b) * kMaxSlices + s] = run;
    if (sure_total) atomicAdd(&ctr[0], sure_total);
    if (s == 0) ctr[1] = static_cast<uint32_t>(b1 + 1);
  }
  // merge this slice's digit-2 histogram into the sequence's
  uint32_t* h2 = P.hist2 + int64_t(b) * kHistBins;
  for (int i = tid; i < kHistBins; i += kSelThreads) {
    const uint32_t c = s_h[i];
    if (c) atomicAdd(&h2[i], c);
  }
}

// --------------------------------------------------------------------------------------
// finish
// --------------------------------------------------------------------------------------
// Entry j (0 <= j < total) of the concatenated slice lists.
FP4KV_DEV uint64_t kept_entry(const uint64_t* list, const uint32_t* s_off, int slices, int64_t per,
                              uint32_t j) {
  int lo = 0, hi = slices - 1;  // last slice with s_off[slice] <= j
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_off[mid] <= j) lo = mid;
    else hi = mid - 1;
  }
  return __ldcg(reinterpret_cast<const unsigned long long*>(list) + per * lo + (j - s_off[lo]));
}

constexpr size_t kFinSmem = size_t(kStage) * 8 + size_t(kMaxSel) * 8 + size_t(kMaxSlices + 1) * 4;

__global__ void __launch_bounds__(kSelThreads) k_select_finish(const SelectArgs args) {
  griddep_wait();  // the filter grid has completed and its writes are visible
  griddep_launch_dependents();
  const SelectProblem& P = args.p[blockIdx.z];
  const int b = blockIdx.y, s = blockIdx.x;
  if (s >= P.slices) return;
  extern __shared__ __align__(16) uint8_t fin_smem[];
  uint64_t* s_stage = reinterpret_cast<uint64_t*>(fin_smem);       // [kStage]
  uint64_t* s_sel = s_stage + kStage;                              // [kMaxSel]
  uint32_t* s_h = reinterpret_cast<uint32_t*>(s_sel);              // digit-2 histogram (aliases s_sel)
  uint32_t* s_off = reinterpret_cast<uint32_t*>(s_sel + kMaxSel);  // [kMaxSlices + 1]
  __shared__ uint32_t s_scan[96];
  __shared__ uint32_t s_wsum[kSelWarps];
  __shared__ uint32_t s_hist8[256];
  __shared__ bool s_last;
  const int tid = threadIdx.x;

  const int64_t n = n_values(P, b);
  const int64_t per = slice_per(n, P.slices);
  const int64_t lo = per * s;
  uint32_t* ctr = P.counters + int64_t(b) * kSelCounters;
  uint64_t* list = P.list + int64_t(b) * P.vstride;
  uint32_t* h2g = P.hist2 + int64_t(b) * kHistBins;
  const int b1 = static_cast<int>(__ldcg(&ctr[1])) - 1;
  const uint32_t n_sure = __ldcg(&ctr[0]);
  const uint32_t k = static_cast<uint32_t>(P.k);
  const uint32_t r = k > n_sure ? k - n_sure : 0u;  // keys still to take from digit 1 == b1

  // digit 2 of the K-th key: b2 = -1 takes every key of the b1 bin; b2 = 4096 takes none
  int b2 = kHistBins;
  uint32_t above2 = 0, bin_count = 0;
  if (r > 0 && b1 >= 0) find_digit_desc_g(h2g, r, &b2, &above2, &bin_count, s_scan);
  // the digit-1 histogram has been read by the filter grid (complete): zero this CTA's share
  {
    const int per_cta = (kHistBins + P.slices - 1) / P.slices;
    uint32_t* h1 = P.hist + int64_t(b) * kHistBins;
    for (int i = s * per_cta + tid; i < min(kHistBins, (s + 1) * per_cta); i += kSelThreads) h1[i] = 0;
  }

  // drop the keys of the b1 bin below b2 from this slice's list (in place, order kept)
  const uint32_t cnt = __ldcg(P.cnt1 + int64_t(b) * kMaxSlices + s);
  uint32_t run = 0;
  for (uint32_t j0 = 0; j0 < cnt; j0 += kSelThreads * 4) {
    uint64_t e[4];
    uint32_t keep = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t j = j0 + tid * 4 + u;
      e[u] = 0;
      if (j < cnt) {
        e[u] = __ldcg(reinterpret_cast<const unsigned long long*>(list) + lo + j);
        const uint32_t key = ent_key(e[u]);
        if (digit1(key) != b1 || digit2(key) >= b2) keep |= 1u << u;
      }
    }
    uint32_t total;
    uint32_t o = run + block_excl_scan(static_cast<uint32_t>(__popc(keep)), s_wsum, &total);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if ((keep >> u) & 1u) list[lo + o++] = e[u];
    run += total;
  }
  __syncthreads();
  if (tid == 0) {
    P.cnt2[int64_t(b) * kMaxSlices + s] = run;
    __threadfence();
    const uint32_t t = atomicAdd(&ctr[2], 1u);
    s_last = (t == static_cast<uint32_t>(P.slices - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA of the sequence: offsets of the slice lists ----
  uint32_t total_kept;
  {
    const uint32_t c = tid < P.slices ? __ldcg(P.cnt2 + int64_t(b) * kMaxSlices + tid) : 0u;
    const uint32_t ex = block_excl_scan(c, s_wsum, &total_kept);
    if (tid < P.slices) s_off[tid] = ex;
    if (tid == 0) s_off[P.slices] = total_kept;
    __syncthreads();
  }
  const bool staged = total_kept <= static_cast<uint32_t>(kStage);
  if (staged) {  // one warp per slice list
    const int lane = tid & 31;
    for (int sl = tid >> 5; sl < P.slices; sl += kSelWarps) {
      const uint32_t o = s_off[sl], n_sl = s_off[sl + 1] - o;
      const unsigned long long* src = reinterpret_cast<const unsigned long long*>(list) + per * sl;
      for (uint32_t j = lane; j < n_sl; j += 32) s_stage[o + j] = __ldcg(src + j);
    }
    __syncthreads();
  }
  auto entry = [&](uint32_t j) -> uint64_t {
    return staged ? s_stage[j] : kept_entry(list, s_off, P.slices, per, j);
  };

  // ---- the (b1, b2) bin: r2 of its keys are taken ----
  const uint32_t r2 = r > above2 ? r - above2 : 0u;
  const bool in_range = b1 >= 0 && b2 >= 0 && b2 < kHistBins;
  const bool bin_all = !in_range || r2 >= bin_count;
  const uint32_t pre24 = in_range ? (static_cast<uint32_t>(b1) << 12) | static_cast<uint32_t>(b2) : 0u;
  uint32_t ustar = 0;
  int64_t pos_star = INT64_MAX;
  if (in_range && !bin_all && r2 > 0) {
    // the last 8 key bits
    for (int i = tid; i < 256; i += kSelThreads) s_hist8[i] = 0;
    __syncthreads();
    for (uint32_t j = tid; j < total_kept; j += kSelThreads) {
      const uint32_t key = ent_key(entry(j));
      if ((key >> 8) == pre24) atomicAdd(&s_hist8[key & 255u], 1u);
    }
    __syncthreads();
    int d3;
    uint32_t above3;
    find_digit_desc(s_hist8, 256, r2, &d3, &above3, s_scan);
    ustar = (pre24 << 8) | static_cast<uint32_t>(d3);
    uint32_t rr = r2 - above3;
    const uint32_t cnt_eq = s_hist8[d3];
    __syncthreads();
    if (rr < cnt_eq) {
      // the rr lowest positions among the keys equal to ustar: 8-bit passes over 32 bits
      uint64_t pprefix = 0;
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kSelThreads) s_hist8[i] = 0;
        __syncthreads();
        for (uint32_t j = tid; j < total_kept; j += kSelThreads) {
          const uint64_t cv = entry(j);
          if (ent_key(cv) != ustar) continue;
          const uint64_t pos = static_cast<uint64_t>(position_of(P, b, ent_idx(cv)));
          if ((pos >> (shift + 8)) == pprefix) atomicAdd(&s_hist8[(pos >> shift) & 255], 1u);
        }
        __syncthreads();
        int d;
        uint32_t below;
        find_digit_asc(s_hist8, 256, rr, &d, &below, s_scan);
        rr -= below;
        pprefix = (pprefix << 8) | static_cast<uint64_t>(d);
      }
      pos_star = static_cast<int64_t>(pprefix);
    }
  }

  // ---- ordered compaction of the selected keys ----
  int32_t* oi = P.out_idx + int64_t(b) * P.k;
  float* os = P.out_score ? P.out_score + int64_t(b) * P.k : nullptr;
  uint32_t m = 0;
  for (uint32_t j0 = 0; j0 < total_kept; j0 += kSelThreads * 4) {
    uint64_t e[4];
    uint32_t take = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t j = j0 + tid * 4 + u;
      e[u] = 0;
      if (j < total_kept) {
        e[u] = entry(j);
        const uint32_t key = ent_key(e[u]);
        bool t = true;  // digit 1 > b1, or digit 2 > b2, or the whole (b1, b2) bin
        if (!bin_all && (key >> 8) == pre24)
          t = r2 > 0 && (key > ustar || (key == ustar && position_of(P, b, ent_idx(e[u])) <= pos_star));
        if (t) take |= 1u << u;
      }
    }
    uint32_t total;
    uint32_t o = m + block_excl_scan(static_cast<uint32_t>(__popc(take)), s_wsum, &total);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (!((take >> u) & 1u)) continue;
      if (o < k) {
        const int32_t i = ent_idx(e[u]);
        if (P.mode != 2) {
          oi[o] = i;
          if (os) os[o] = key_to_float(ent_key(e[u]));
        } else {
          s_sel[o] = (static_cast<uint64_t>(position_of(P, b, i)) << 32) | static_cast<uint32_t>(i);
        }
      }
      ++o;
    }
    m += total;
  }
  if (m > k) m = k;
  if (P.mode == 2) {
    // pool slots: positions need not grow with the value index, sort (position, index)
    const int nsort = m <= static_cast<uint32_t>(kSelThreads * 4) ? kSelThreads * 4 : kSelThreads * 8;
    for (int i = static_cast<int>(m) + tid; i < nsort; i += kSelThreads) s_sel[i] = ~0ull;
    __syncthreads();
    if (nsort == kSelThreads * 4) block_sort<uint64_t, 4>(s_sel);
    else block_sort<uint64_t, 8>(s_sel);
    for (uint32_t j = tid; j < m; j += kSelThreads) {
      oi[j] = static_cast<int32_t>(s_sel[j] >> 32);
      if (os) os[j] = P.values[int64_t(b) * P.vstride + static_cast<uint32_t>(s_sel[j] & 0xffffffffu)];
    }
  }
  for (uint32_t j = m + tid; j < k; j += kSelThreads) {
    oi[j] = -1;
    if (os) os[j] = -INFINITY;
  }
  // leave the workspace zeroed for the next call (the digit-1 histogram was zeroed by all
  // the finishing CTAs)
  for (int i = tid; i < kHistBins; i += kSelThreads) h2g[i] = 0;
  if (tid < kSelCounters) ctr[tid] = 0;
}

}  // namespace

int select_slices(int64_t n_values, int B, int num_sms) {
  int64_t s = (2 * int64_t(num_sms)) / B;  // two CTAs per SM: one wave
  const int64_t cap = (n_values + kBatchVals - 1) / kBatchVals;
  if (s > cap) s = cap;
  if (s > kMaxSlices) s = kMaxSlices;
  if (s < 1) s = 1;
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
  cudaError_t e = cudaFuncSetAttribute(k_select_finish, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kFinSmem));
  if (e != cudaSuccess) return e;
  // both kernels are programmatic dependents of the kernel before them on the stream
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k_select_filter, args);
  if (e != cudaSuccess) return e;
  cfg.dynamicSmemBytes = kFinSmem;
  e = cudaLaunchKernelEx(&cfg, k_select_finish, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4kv
