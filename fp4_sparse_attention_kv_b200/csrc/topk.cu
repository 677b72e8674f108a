// Exact top-K select per sequence: the K largest fp32 values, ties to the lower position,
// returned as positions in ascending order padded with -1.
//
// Used for the indexer top-K ([PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로
// 줄이고 …", section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2": each Full or Reindex
// layer produces its own top-K indices) and for the candidate pool (section "계층적 희소
// 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기": the blocks with the highest block max).
//
// Values are mapped to order-preserving 32-bit keys. The scoring kernel has already built a
// histogram of the top 12 key bits (digit 1) of every sequence. Two kernels follow:
//  filter  (every SM busy: S slices per sequence, 8 warps per slice, each warp one contiguous
//          sub-slice read with fully coalesced 16-byte loads, two batches in flight) finds the
//          digit-1 value b1 of the K-th largest key, keeps the keys with digit 1 >= b1 of its
//          sub-slice in position order (a ballot prefix inside the warp, no block barrier) in
//          the sub-slice's own region of the list array, and histograms the next 12 bits
//          (digit 2) of the keys with digit 1 == b1;
//  finish  (a programmatic dependent; one CTA per sequence) finds the digit-2 value b2 of the
//          K-th key, stages the few thousand kept entries in shared memory (regions in
//          position order), resolves the (b1, b2) bin exactly only when it is taken in part
//          (the last 8 key bits, then the lowest positions among equal keys), and writes the
//          selection with one ordered compaction: positions come out ascending without a
//          sort (the pool mode, whose positions need not grow with the value index, sorts
//          its at most 4096 selected pairs). It also zeroes the histograms and counters,
//          leaving the workspace ready for the next call.
// No CTA ever waits on another CTA.
#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"
#include "fp4kv_sm100.cuh"

namespace fp4kv {
namespace {

constexpr int kFThreads = 256;               // filter CTA
constexpr int kFWarps = kFThreads / 32;      // sub-slices per slice
constexpr int kGroups = 8;                   // 16-byte loads per lane and batch
constexpr int kWarpBatch = 32 * 4 * kGroups; // 1024 values
constexpr int kNThreads = 1024;              // finish CTA
constexpr int kNWarps = kNThreads / 32;
constexpr int kMaxSel = 4096;
constexpr int kMaxProblems = 2;
constexpr int kStage = 12288;                // kept entries the finish CTA stages in shared memory
static_assert(kFWarps == kSelRegions, "one kept-entry region per filter warp");
static_assert(kMaxSlices * kFWarps <= 4 * kNThreads, "region counts: four per finishing thread");

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

// Slice s of n values over `slices` CTAs, sub-slice w of it: [lo, hi), multiples of 128
// values (whole 16-byte lane groups of a warp) except at n.
struct Region {
  int64_t lo, hi;
};
FP4KV_DEV Region region_of(int64_t n, int slices, int s, int w) {
  const int64_t per_s = ((n + slices - 1) / slices + kWarpBatch - 1) / kWarpBatch * kWarpBatch;
  const int64_t slo = min(n, per_s * s), shi = min(n, slo + per_s);
  const int64_t per_w = ((shi - slo + kFWarps - 1) / kFWarps + 127) / 128 * 128;
  const int64_t lo = min(shi, slo + per_w * w);
  return {lo, min(shi, lo + per_w)};
}

FP4KV_DEV int64_t position_of(const SelectProblem& P, int b, int64_t i) {
  if (P.mode != 2) return i;
  const int64_t j = P.pool[int64_t(b) * P.npb + i / 8];
  return j * 8 + (i % 8);
}

FP4KV_DEV uint32_t ent_key(uint64_t c) { return static_cast<uint32_t>(c >> 32); }
FP4KV_DEV int32_t ent_idx(uint64_t c) { return static_cast<int32_t>(c & 0xffffffffu); }
FP4KV_DEV int digit1(uint32_t key) { return static_cast<int>(key >> 20); }
FP4KV_DEV int digit2(uint32_t key) { return static_cast<int>((key >> 8) & 0xfffu); }

FP4KV_DEV uint32_t warp_incl_scan(uint32_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Block-wide exclusive prefix sum over the kT threads; *total gets the block sum. s_w: kT / 32
// words. Every thread calls it (barriers inside).
template <int kT>
FP4KV_DEV uint32_t block_excl_scan(uint32_t v, uint32_t* s_w, uint32_t* total) {
  constexpr int kW = kT / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const uint32_t x = warp_incl_scan(v);
  if (lane == 31) s_w[w] = x;
  __syncthreads();
  if (w == 0) {
    uint32_t t = lane < kW ? s_w[lane] : 0u;
    t = warp_incl_scan(t);
    if (lane < kW) s_w[lane] = t;
  }
  __syncthreads();
  const uint32_t excl = x - v + (w > 0 ? s_w[w - 1] : 0u);
  *total = s_w[kW - 1];
  __syncthreads();
  return excl;
}

// Block-wide (kT threads): thread t owns kPer bins counted from the top, h[nbins - kPer (t+1)
// .. nbins - kPer t), given in vals[] highest first. Finds the bin d at which the count from
// the top reaches r (r >= 1): d, the count above it and its own count. If the total is below
// r: d = -1, above = total, cnt = 0. Every thread calls it.
template <int kT, int kPer>
FP4KV_DEV void block_find_desc(const uint32_t (&vals)[kPer], int nbins, uint32_t r, int* d_out,
                               uint32_t* above_out, uint32_t* cnt_out, uint32_t* s_w, uint32_t* s_res) {
  const int tid = threadIdx.x;
  const int hi = nbins - kPer * tid;
  uint32_t sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (hi - 1 - i >= 0) sum += vals[i];
  if (tid == 0) {
    s_res[0] = 0xffffffffu;
    s_res[1] = 0;
    s_res[2] = 0;
  }
  uint32_t total;
  const uint32_t excl = block_excl_scan<kT>(sum, s_w, &total);  // (its barriers order s_res)
  if (total < r) {
    if (tid == 0) s_res[1] = total;
  } else if (excl < r && excl + sum >= r) {
    uint32_t acc = excl;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (hi - 1 - i >= 0) {
        if (acc + vals[i] >= r) {
          s_res[0] = static_cast<uint32_t>(hi - 1 - i);
          s_res[1] = acc;
          s_res[2] = vals[i];
          break;
        }
        acc += vals[i];
      }
    }
  }
  __syncthreads();
  *d_out = s_res[0] == 0xffffffffu ? -1 : static_cast<int>(s_res[0]);
  *above_out = s_res[1];
  *cnt_out = s_res[2];
  __syncthreads();
}

// Block-wide ascending bitonic sort of N = kNThreads * E keys held in shared memory.
// Each thread keeps E consecutive keys in registers: strides below E are exchanged inside
// the thread, strides up to 16 E through warp shuffles, and only the widest strides through
// shared memory (one barrier pair each).
template <typename T, int E>
__device__ void block_sort(T* s) {
  constexpr int N = kNThreads * E;
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

FP4KV_DEV float4 ld_vals4(const float* p, bool ok) {
  return ok ? __ldcg(reinterpret_cast<const float4*>(p)) : make_float4(0.f, 0.f, 0.f, 0.f);
}

// --------------------------------------------------------------------------------------
// filter
// --------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kFThreads) k_select_filter(const SelectArgs args) {
  // the finishing kernel is a programmatic dependent: it may be scheduled from now on
  griddep_launch_dependents();
  __shared__ __align__(16) uint32_t s_h2[kHistBins];  // digit-2 histogram of this slice
  __shared__ uint32_t s_w[kFThreads / 32];
  __shared__ uint32_t s_res[4];
  __shared__ uint32_t s_sure;
  const SelectProblem& P = args.p[blockIdx.z];
  const int b = blockIdx.y, s = blockIdx.x;
  if (s >= P.slices) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kHistBins; i += kFThreads) s_h2[i] = 0;
  if (tid == 0) s_sure = 0;
  griddep_wait();  // the scores and the digit-1 histogram are complete past here

  const int64_t n = n_values(P, b);
  const uint32_t k = static_cast<uint32_t>(P.k);
  const float* vals = P.values + int64_t(b) * P.vstride;
  uint64_t* list = P.list + int64_t(b) * P.vstride;

  // digit 1 of the K-th largest key (b1 = -1: fewer than K values, all are kept)
  int b1;
  {
    static_assert(kHistBins == kFThreads * 16, "16 bins per thread");
    const uint32_t* h1 = P.hist + int64_t(b) * kHistBins;
    const int lo16 = kHistBins - 16 * (tid + 1);
    uint32_t h[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = __ldcg(reinterpret_cast<const uint4*>(h1 + lo16 + 4 * (3 - q)));
      h[4 * q] = v.w;
      h[4 * q + 1] = v.z;
      h[4 * q + 2] = v.y;
      h[4 * q + 3] = v.x;
    }
    uint32_t above1, cnt1;
    block_find_desc<kFThreads, 16>(h, kHistBins, k, &b1, &above1, &cnt1, s_w, s_res);
  }

  // this warp's sub-slice: keys with digit 1 >= b1, in position order, into list[lo ..)
  const Region R = region_of(n, P.slices, s, warp);
  uint32_t run = 0, sure = 0;
  float4 cur[kGroups], nxt[kGroups];
#pragma unroll
  for (int g = 0; g < kGroups; ++g) {
    const int64_t i = R.lo + 128 * g + 4 * lane;
    cur[g] = ld_vals4(vals + i, i < R.hi);
  }
  for (int64_t base = R.lo; base < R.hi; base += kWarpBatch) {
#pragma unroll
    for (int g = 0; g < kGroups; ++g) {  // the next batch is loaded while this one is kept
      const int64_t i = base + kWarpBatch + 128 * g + 4 * lane;
      nxt[g] = ld_vals4(vals + i, i < R.hi);
    }
#pragma unroll
    for (int g = 0; g < kGroups; ++g) {
      const int64_t i0 = base + 128 * g + 4 * lane;
      const float v[4] = {cur[g].x, cur[g].y, cur[g].z, cur[g].w};
      uint32_t keep = 0, key[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        key[u] = order_key(v[u]);
        const bool valid = i0 + u < R.hi && (P.mode != 2 || v[u] != -INFINITY);
        const int d = digit1(key[u]);
        if (valid && d > b1) {
          keep |= 1u << u;
          ++sure;
        } else if (valid && d == b1) {
          keep |= 1u << u;
          atomicAdd(&s_h2[digit2(key[u])], 1u);
        }
      }
      const uint32_t c = __popc(keep);
      const uint32_t incl = warp_incl_scan(c);
      if (__any_sync(0xffffffffu, keep != 0)) {
        // (run + the kept count never exceeds the sub-slice length: the region holds them)
        uint64_t* dst = list + R.lo + run + (incl - c);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if ((keep >> u) & 1u)
            *dst++ = (static_cast<uint64_t>(key[u]) << 32) | static_cast<uint32_t>(i0 + u);
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
#pragma unroll
    for (int g = 0; g < kGroups; ++g) cur[g] = nxt[g];
  }
  sure = __reduce_add_sync(0xffffffffu, sure);
  uint32_t* ctr = P.counters + int64_t(b) * kSelCounters;
  if (lane == 0) {
    P.cnt[(int64_t(b) * P.slices + s) * kFWarps + warp] = run;
    if (sure) atomicAdd(&s_sure, sure);
  }
  __syncthreads();
  if (tid == 0) {
    if (s_sure) atomicAdd(&ctr[0], s_sure);
    if (s == 0) ctr[1] = static_cast<uint32_t>(b1 + 1);
  }
  // merge this slice's digit-2 histogram into the sequence's
  uint32_t* h2 = P.hist2 + int64_t(b) * kHistBins;
  for (int i4 = tid; i4 < kHistBins / 4; i4 += kFThreads) {
    const uint4 c = reinterpret_cast<const uint4*>(s_h2)[i4];
    if ((c.x | c.y | c.z | c.w) == 0u) continue;
    if (c.x) atomicAdd(&h2[4 * i4], c.x);
    if (c.y) atomicAdd(&h2[4 * i4 + 1], c.y);
    if (c.z) atomicAdd(&h2[4 * i4 + 2], c.z);
    if (c.w) atomicAdd(&h2[4 * i4 + 3], c.w);
  }
}

// --------------------------------------------------------------------------------------
// finish
// --------------------------------------------------------------------------------------
struct FinSmem {
  uint64_t stage[kStage];            // kept entries, regions concatenated in position order
  uint64_t sel[kMaxSel];             // the pool mode's selected (position, index) pairs
  uint32_t roff[kNThreads * 4 + 1];  // region offsets in the concatenation
  uint32_t h8[256];
  uint32_t w[kNWarps];
  uint32_t res[4];
};
constexpr size_t kFinSmem = sizeof(FinSmem);

// Entry j of the concatenated kept lists: staged, or read straight from its region.
FP4KV_DEV uint64_t kept_entry(const FinSmem& S, bool staged, const uint64_t* list, int64_t n, int slices,
                              int n_regions, uint32_t j) {
  if (staged) return S.stage[j];
  int lo = 0, hi = n_regions - 1;  // last region with roff <= j
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (S.roff[mid] <= j) lo = mid;
    else hi = mid - 1;
  }
  const Region R = region_of(n, slices, lo / kFWarps, lo % kFWarps);
  return __ldcg(reinterpret_cast<const unsigned long long*>(list) + R.lo + (j - S.roff[lo]));
}

__global__ void __launch_bounds__(kNThreads) k_select_finish(const SelectArgs args) {
  // the attention that follows may be scheduled from now on
  griddep_launch_dependents();
  griddep_wait();  // the filter grid has completed and its writes are visible
  extern __shared__ __align__(16) uint8_t fin_raw[];
  FinSmem& S = *reinterpret_cast<FinSmem*>(fin_raw);
  const SelectProblem& P = args.p[blockIdx.z];
  const int b = blockIdx.y;
  const int tid = threadIdx.x;
  const int64_t n = n_values(P, b);
  const uint32_t k = static_cast<uint32_t>(P.k);
  uint32_t* ctr = P.counters + int64_t(b) * kSelCounters;
  uint32_t* h1 = P.hist + int64_t(b) * kHistBins;
  uint32_t* h2 = P.hist2 + int64_t(b) * kHistBins;
  const uint64_t* list = P.list + int64_t(b) * P.vstride;
  const int b1 = static_cast<int>(__ldcg(&ctr[1])) - 1;
  const uint32_t n_sure = __ldcg(&ctr[0]);
  const bool have_b1 = b1 >= 0;

  // ---- digit 2 of the K-th key ----
  int b2 = -1;
  uint32_t r3 = 0, cnt_b2 = 0;
  {
    static_assert(kHistBins == kNThreads * 4, "4 bins per thread");
    const int lo4 = kHistBins - 4 * (tid + 1);
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(h2 + lo4));
    const uint32_t h[4] = {v.w, v.z, v.y, v.x};
    const uint32_t r2 = have_b1 && k > n_sure ? k - n_sure : 1u;
    int d;
    uint32_t above, cnt;
    block_find_desc<kNThreads, 4>(h, kHistBins, r2, &d, &above, &cnt, S.w, S.res);
    if (have_b1) {
      b2 = d;
      r3 = r2 - above;
      cnt_b2 = cnt;
    }
  }
  // the histograms have been read (the digit-1 one by the whole filter grid): clear them
  for (int i = tid; i < kHistBins; i += kNThreads) {
    h1[i] = 0;
    h2[i] = 0;
  }

  // ---- region offsets (regions in position order) and staging ----
  const int n_regions = P.slices * kFWarps;
  uint32_t total_kept;
  {
    uint32_t c[4], sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rg = 4 * tid + i;
      c[i] = rg < n_regions ? __ldcg(P.cnt + int64_t(b) * n_regions + rg) : 0u;
      sum += c[i];
    }
    uint32_t excl = block_excl_scan<kNThreads>(sum, S.w, &total_kept);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rg = 4 * tid + i;
      if (rg < n_regions) S.roff[rg] = excl;
      excl += c[i];
    }
    if (tid == 0) S.roff[n_regions] = total_kept;
    __syncthreads();
  }
  const bool staged = total_kept <= static_cast<uint32_t>(kStage);
  if (staged) {
    // entry j of the concatenation: its region by binary search over the offsets; eight
    // entries' loads per thread are in flight before any is stored
    constexpr int kBatch = 8;
    for (uint32_t jb = tid; jb < total_kept; jb += kNThreads * kBatch) {
      uint64_t v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const uint32_t j = jb + u * kNThreads;
        v[u] = 0;
        if (j < total_kept) {
          int lo = 0, hi = n_regions - 1;  // last region with roff <= j
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (S.roff[mid] <= j) lo = mid;
            else hi = mid - 1;
          }
          const Region R = region_of(n, P.slices, lo / kFWarps, lo % kFWarps);
          v[u] = __ldcg(reinterpret_cast<const unsigned long long*>(list) + R.lo + (j - S.roff[lo]));
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const uint32_t j = jb + u * kNThreads;
        if (j < total_kept) S.stage[j] = v[u];
      }
    }
    __syncthreads();
  }
  auto entry = [&](uint32_t j) -> uint64_t { return kept_entry(S, staged, list, n, P.slices, n_regions, j); };

  // ---- the (b1, b2) bin, when only r3 of its cnt_b2 keys are taken ----
  const bool tie = have_b1 && b2 >= 0 && r3 < cnt_b2;
  const uint32_t pre24 = tie ? (static_cast<uint32_t>(b1) << 12) | static_cast<uint32_t>(b2) : 0u;
  uint32_t ustar = 0;
  int64_t pos_star = INT64_MAX;
  if (tie) {
    if (tid < 256) S.h8[tid] = 0;
    __syncthreads();
    for (uint32_t j = tid; j < total_kept; j += kNThreads) {
      const uint32_t key = ent_key(entry(j));
      if ((key >> 8) == pre24) atomicAdd(&S.h8[key & 255u], 1u);
    }
    __syncthreads();
    uint32_t hv[1] = {tid < 256 ? S.h8[255 - tid] : 0u};
    int d3;
    uint32_t above3, cnt3;
    block_find_desc<kNThreads, 1>(hv, 256, r3, &d3, &above3, &cnt3, S.w, S.res);
    ustar = (pre24 << 8) | static_cast<uint32_t>(d3);
    uint32_t rr = r3 - above3;  // keys equal to ustar to take, lowest positions first
    if (rr < cnt3) {
      // 8-bit passes over the 32-bit positions, from the top
      uint64_t pprefix = 0;
      for (int shift = 24; shift >= 0; shift -= 8) {
        if (tid < 256) S.h8[tid] = 0;
        __syncthreads();
        for (uint32_t j = tid; j < total_kept; j += kNThreads) {
          const uint64_t e = entry(j);
          if (ent_key(e) != ustar) continue;
          const uint64_t pos = static_cast<uint64_t>(position_of(P, b, ent_idx(e)));
          if ((pos >> (shift + 8)) == pprefix) atomicAdd(&S.h8[(pos >> shift) & 255], 1u);
        }
        __syncthreads();
        // lowest digit first: thread t holds bin t, as the (255 - t)-th bin from the top
        uint32_t hp[1] = {tid < 256 ? S.h8[tid] : 0u};
        int dv;
        uint32_t below, cntd;
        block_find_desc<kNThreads, 1>(hp, 256, rr, &dv, &below, &cntd, S.w, S.res);
        const int dd = dv < 0 ? 255 : 255 - dv;
        rr -= below;
        pprefix = (pprefix << 8) | static_cast<uint64_t>(dd);
      }
      pos_star = static_cast<int64_t>(pprefix);
    }
  }
  auto selected = [&](uint64_t e) -> bool {
    if (!have_b1) return true;
    const uint32_t key = ent_key(e);
    const int d1 = digit1(key);
    if (d1 != b1) return d1 > b1;
    const int d2 = digit2(key);
    if (d2 != b2) return d2 > b2;
    if (!tie) return true;
    return key > ustar || (key == ustar && position_of(P, b, ent_idx(e)) <= pos_star);
  };

  // ---- ordered compaction: thread t owns one contiguous run of the concatenation ----
  int32_t* oi = P.out_idx + int64_t(b) * P.k;
  float* os = P.out_score ? P.out_score + int64_t(b) * P.k : nullptr;
  const uint32_t per = (total_kept + kNThreads - 1) / kNThreads;
  const uint32_t j0 = min(total_kept, per * tid), j1 = min(total_kept, j0 + per);
  uint32_t m_own = 0;
  for (uint32_t j = j0; j < j1; ++j) m_own += selected(entry(j)) ? 1u : 0u;
  uint32_t m_all;
  uint32_t o = block_excl_scan<kNThreads>(m_own, S.w, &m_all);
  for (uint32_t j = j0; j < j1 && o < k; ++j) {
    const uint64_t e = entry(j);
    if (!selected(e)) continue;
    const int32_t i = ent_idx(e);
    if (P.mode != 2) {
      oi[o] = i;
      if (os) os[o] = key_to_float(ent_key(e));
    } else {
      S.sel[o] = (static_cast<uint64_t>(position_of(P, b, i)) << 32) | static_cast<uint32_t>(i);
    }
    ++o;
  }
  const uint32_t m = m_all < k ? m_all : k;
  if (P.mode == 2) {
    // pool slots: positions need not grow with the value index, sort (position, index)
    __syncthreads();
    for (uint32_t i = m + tid; i < static_cast<uint32_t>(kMaxSel); i += kNThreads) S.sel[i] = ~0ull;
    __syncthreads();
    block_sort<uint64_t, kMaxSel / kNThreads>(S.sel);
    const float* vals = P.values + int64_t(b) * P.vstride;
    for (uint32_t j = tid; j < m; j += kNThreads) {
      oi[j] = static_cast<int32_t>(S.sel[j] >> 32);
      if (os) os[j] = vals[static_cast<uint32_t>(S.sel[j] & 0xffffffffu)];
    }
  }
  for (uint32_t j = m + tid; j < k; j += kNThreads) {
    oi[j] = -1;
    if (os) os[j] = -INFINITY;
  }
  if (tid < kSelCounters) ctr[tid] = 0;  // (every thread read them above, before the barriers)
}

}  // namespace

int select_slices(int64_t n_values, int B, int num_sms) {
  // about two filter CTAs per SM (what their registers allow) over the whole grid, at least
  // 4096 values each
  int64_t s = (2 * int64_t(num_sms)) / B;
  const int64_t cap = (n_values + 4095) / 4096;
  if (s > cap) s = cap;
  if (s > kMaxSlices) s = kMaxSlices;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

cudaError_t launch_topk_select(const SelectProblem* probs, int n_probs, int B, cudaStream_t stream) {
  if (n_probs < 1 || n_probs > kMaxProblems || B == 0) return cudaSuccess;
  SelectArgs args{};
  int gx = 1;
  for (int i = 0; i < n_probs; ++i) {
    args.p[i] = probs[i];
    if (probs[i].slices > gx) gx = probs[i].slices;
  }
  cudaError_t e = cudaFuncSetAttribute(k_select_finish, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kFinSmem));
  if (e != cudaSuccess) return e;
  // both kernels are programmatic dependents of the kernel before them on the stream
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(gx, B, n_probs);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k_select_filter, args);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(1, B, n_probs);
  cfg.blockDim = dim3(kNThreads);
  cfg.dynamicSmemBytes = kFinSmem;
  e = cudaLaunchKernelEx(&cfg, k_select_finish, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4kv
