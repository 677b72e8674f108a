// Exact top-K select per sequence: the K largest fp32 values, ties to the lower position,
// returned as positions in ascending order padded with -1.
//
// Used for the indexer top-K ([PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로
// 줄이고 …", section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2": each Full or Reindex
// layer produces its own top-K indices) and for the candidate pool (section "계층적 희소
// 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기": the blocks with the highest block max).
//
// Values are mapped to order-preserving 32-bit keys. The scoring kernel has already built a
// histogram of the top 12 key bits (digit 1) of every sequence. One kernel follows, with one
// thread-block cluster of C CTAs per (problem, sequence); CTA r owns slice r of the values,
// warp w of it sub-slice w (slices and sub-slices in position order):
//  1. every CTA finds the digit-1 value b1 of the K-th largest key from the histogram, as two
//     float thresholds: "digit 1 >= b1" is v >= f_lo, "digit 1 > b1" is v >= f_hi;
//  2. each warp streams its sub-slice through a ring of shared-memory buffers filled by bulk
//     asynchronous copies (the copy engine keeps every buffer's bytes in flight), keeps the
//     values >= f_lo in position order (a warp prefix, no block barrier) in its own list, and
//     the CTA histograms the next 12 key bits (digit 2) of the keys with digit 1 == b1;
//  3. the CTAs add up the digit-2 histograms through distributed shared memory (CTA r sums
//     segment r of the bins in place) and every CTA finds the digit-2 value b2 of the K-th key;
//  4. only when the (b1, b2) bin is taken in part: the last 8 key bits, then the lowest
//     positions among the keys equal to the K-th key, are resolved the same way;
//  5. every CTA counts what it takes, reads the counts of the CTAs before it and writes its
//     positions at that offset: ascending without a sort. A Reindex pool whose blocks are not
//     in ascending order gathers its at most 4096 selected pairs in CTA 0, which sorts them.
// The CTAs also clear the scoring kernel's histogram for the next call. Cluster barriers are
// the only synchronisation between CTAs; every mbarrier wait is bounded in time.
// Kernels that live a few microseconds run mostly from a cold instruction cache, so the loop
// bodies here are kept short.
#include <cfloat>

#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"
#include "fp4kv_sm100.cuh"

namespace fp4kv {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 1024;              // values per ring buffer (4 KiB)
constexpr int kMaxDepth = 2;              // ring buffers per warp
constexpr int kWarpCap = 256;             // kept entries per warp held in shared memory
constexpr int kMaxCluster = 16;
constexpr int kMaxSel = 4096;
constexpr int kMaxProblems = 2;

struct SelectArgs {
  SelectProblem p[kMaxProblems];
  int depth;  // ring buffers per warp
};

struct SelSmem {
  uint32_t h2[kHistBins];               // digit-2 histogram; segment r is summed in place
  uint64_t list[kWarps][kWarpCap];      // kept entries: (order key << 32) | value index
  uint64_t bar[kWarps][kMaxDepth];      // ring mbarriers
  uint32_t h8[256];                     // last 8 key bits of the (b1, b2) bin
  uint32_t hp[2][256];                  // position digits among the keys equal to the K-th
  uint32_t hsum[256];                   // a 256-bin histogram summed over the cluster
  uint32_t wcnt[kWarps];                // kept entries per warp
  uint32_t wsel[kWarps];                // selected entries per warp
  uint32_t w[kWarps];                   // block scans
  uint32_t res[4];
  uint32_t sure;                        // keys of this CTA with digit 1 > b1
  uint32_t seg_total;                   // sum of this CTA's summed digit-2 segment
  uint32_t sel_total;                   // entries this CTA selects
  uint32_t bc[4];                       // block broadcasts
};
// the ring follows; after the filter phase CTA 0 reuses it for the pool mode's sorted pairs
constexpr size_t kSmemFixed = (sizeof(SelSmem) + 127) / 128 * 128;
size_t select_smem(int depth) { return kSmemFixed + size_t(kWarps) * depth * kChunk * sizeof(float); }
static_assert(kWarps * kChunk * sizeof(float) >= kMaxSel * sizeof(uint64_t), "pairs fit a depth-1 ring");

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

FP4KV_DEV uint32_t ent_key(uint64_t c) { return static_cast<uint32_t>(c >> 32); }
FP4KV_DEV int32_t ent_idx(uint64_t c) { return static_cast<int32_t>(c & 0xffffffffu); }
FP4KV_DEV int digit1(uint32_t key) { return static_cast<int>(key >> 20); }
FP4KV_DEV int digit2(uint32_t key) { return static_cast<int>((key >> 8) & 0xfffu); }

// distributed shared memory (the cluster's CTAs): the address of `p` in CTA `rank`, and loads
// and stores there (volatile with a memory clobber: never moved across a cluster barrier)
FP4KV_DEV uint32_t dsmem_map(const void* p, uint32_t rank) {
  uint32_t r;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
FP4KV_DEV uint32_t dsmem_ld(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
FP4KV_DEV void dsmem_st64(uint32_t addr, uint64_t v) {
  asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}
// sum over the cluster's CTAs of the u32 at `p` (each CTA's copy); the loads are all issued
// before any is added
FP4KV_DEV uint32_t cluster_sum(const uint32_t* p, uint32_t C) {
  uint32_t v[kMaxCluster];
#pragma unroll
  for (uint32_t q = 0; q < kMaxCluster; ++q) v[q] = q < C ? dsmem_ld(dsmem_map(p, q)) : 0u;
  uint32_t s = 0;
#pragma unroll
  for (int q = 0; q < kMaxCluster; ++q) s += v[q];
  return s;
}

FP4KV_DEV uint32_t warp_incl_scan(uint32_t x) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Block-wide exclusive prefix sum; *total gets the block sum. Every thread calls it.
FP4KV_DEV uint32_t block_excl_scan(uint32_t v, uint32_t* s_w, uint32_t* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const uint32_t x = warp_incl_scan(v);
  if (lane == 31) s_w[w] = x;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) {
    const uint32_t t = s_w[i];
    before += i < w ? t : 0u;
    all += t;
  }
  __syncthreads();
  *total = all;
  return x - v + before;
}

// Block-wide: thread t owns `per` bins counted from the top, h[nbins - per (t + 1) .. nbins -
// per t), given in vals[] highest first. Finds the bin d at which the count from the top
// reaches r (r >= 1): d, the count above it and its own count. If the total is below r:
// d = -1, above = total, cnt = 0. Every thread calls it.
template <int kPer>
FP4KV_DEV void block_find_desc(const uint32_t (&vals)[kPer], int per, int nbins, uint32_t r, int* d_out,
                               uint32_t* above_out, uint32_t* cnt_out, uint32_t* s_w, uint32_t* s_res) {
  const int tid = threadIdx.x;
  const int hi = nbins - per * tid;
  uint32_t sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (i < per && hi - 1 - i >= 0) sum += vals[i];
  if (tid == 0) {
    s_res[0] = 0xffffffffu;
    s_res[1] = 0;
    s_res[2] = 0;
  }
  uint32_t total;
  const uint32_t excl = block_excl_scan(sum, s_w, &total);  // (its barriers order s_res)
  if (total < r) {
    if (tid == 0) s_res[1] = total;
  } else if (excl < r && excl + sum >= r) {
    uint32_t acc = excl;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (i < per && hi - 1 - i >= 0) {
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

// Block-wide ascending bitonic sort of kMaxSel keys held in shared memory (8 per thread).
// Strides below 8 are exchanged inside a thread, strides up to 128 through warp shuffles,
// and only the widest ones through shared memory (one barrier pair each).
__device__ void block_sort_pairs(uint64_t* s) {
  constexpr int E = kMaxSel / kThreads;
  const int tid = threadIdx.x;
  uint64_t v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = s[tid * E + e];
#pragma unroll
  for (int size = 2; size <= kMaxSel; size <<= 1) {
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
          const uint64_t p = s[i ^ stride];
          const bool keep_min = ((i & stride) == 0) == ((i & size) == 0);
          v[e] = keep_min ? (v[e] < p ? v[e] : p) : (v[e] < p ? p : v[e]);
        }
      } else if (stride >= E) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const uint64_t p = __shfl_xor_sync(0xffffffffu, v[e], stride / E);
          const bool keep_min = ((i & stride) == 0) == ((i & size) == 0);
          v[e] = keep_min ? (v[e] < p ? v[e] : p) : (v[e] < p ? p : v[e]);
        }
      } else {
        uint64_t nv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const uint64_t p = v[e ^ stride];
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

// The float whose order key is bin << 20, as a threshold: for finite v (or -inf),
// order_key(v) >= bin << 20 exactly when v >= thresh(bin). Keys below the key of -inf map to
// -inf; keys at or above the key of +inf to NaN (no finite value reaches them).
FP4KV_DEV float thresh(int bin) {
  if (bin <= 0) return -INFINITY;
  const uint64_t t = uint64_t(bin) << 20;
  if (t <= 0x007FFFFFull) return -INFINITY;
  if (t >= 0xFF800000ull) return __int_as_float(0x7FC00000);
  return key_to_float(static_cast<uint32_t>(t));
}

__global__ void __launch_bounds__(kThreads, 1) k_topk_select(const SelectArgs args) {
  // the attention (or the next kernel) may be scheduled from now on
  griddep_launch_dependents();
  extern __shared__ __align__(128) uint8_t sel_raw[];
  SelSmem& S = *reinterpret_cast<SelSmem*>(sel_raw);
  float* ring = reinterpret_cast<float*>(sel_raw + kSmemFixed);           // [warp][depth][kChunk]
  uint64_t* s_pairs = reinterpret_cast<uint64_t*>(sel_raw + kSmemFixed);  // pool pairs (after the filter)
  const SelectProblem& P = args.p[blockIdx.z];
  const int D = args.depth;
  const int b = blockIdx.y;
  const uint32_t C = cluster_nctas(), r = cluster_ctarank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < kHistBins; i += kThreads) S.h2[i] = 0;
  if (tid < 256) S.h8[tid] = 0;
  if (tid == 0) S.sure = 0;
  if (lane < D) mbar_init(&S.bar[warp][lane], 1);
  fence_mbar_init();
  __syncwarp();
  griddep_wait();  // the scores and the digit-1 histogram are complete past here

  const int64_t n = n_values(P, b);
  const uint32_t k = static_cast<uint32_t>(P.k);
  const float* vals = P.values + int64_t(b) * P.vstride;
  uint64_t* glist = P.list + int64_t(b) * P.vstride;
  uint32_t* hist1 = P.hist + int64_t(b) * kHistBins;
  // slices in position order, multiples of 128 values (whole 16-byte lane groups)
  const int64_t per_cta = ((n + C - 1) / C + 127) / 128 * 128;
  const int64_t lo = min(n, per_cta * r), hi = min(n, lo + per_cta);
  const int64_t per_w = ((hi - lo + kWarps - 1) / kWarps + 127) / 128 * 128;
  const int64_t wlo = min(hi, lo + per_w * warp), whi = min(hi, wlo + per_w);
  const int n_chunks = static_cast<int>((whi - wlo + kChunk - 1) / kChunk);
  float* wring = ring + size_t(warp) * D * kChunk;
  // chunk c of the sub-slice into buffer c % D: [c0, c1) rounded up to whole 16-byte units
  // (at most 3 values past c1, inside the row: vstride is a multiple of 8 and >= n)
  auto issue = [&](int c) {
    const int64_t c0 = wlo + int64_t(c) * kChunk, c1 = min(whi, c0 + kChunk);
    const uint32_t bytes = static_cast<uint32_t>(((c1 - c0 + 3) / 4) * 16);
    uint64_t* bar = &S.bar[warp][c % D];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_g2s(wring + (c % D) * kChunk, vals + c0, bytes, bar);
  };
  if (lane == 0)
    for (int c = 0; c < D && c < n_chunks; ++c) issue(c);

  // ---- 1. digit 1 of the K-th largest key (b1 = -1: fewer than K values, all are kept) ----
  int b1;
  {
    static_assert(kHistBins == kThreads * 8, "8 bins per thread");
    const int lo8 = kHistBins - 8 * (tid + 1);
    const uint4 va = __ldcg(reinterpret_cast<const uint4*>(hist1 + lo8));
    const uint4 vb = __ldcg(reinterpret_cast<const uint4*>(hist1 + lo8 + 4));
    const uint32_t h[8] = {vb.w, vb.z, vb.y, vb.x, va.w, va.z, va.y, va.x};  // highest bin first
    uint32_t above1, cnt1;
    block_find_desc<8>(h, 8, kHistBins, k, &b1, &above1, &cnt1, S.w, S.res);
  }
  const float f_lo = b1 < 0 ? -INFINITY : thresh(b1);
  const float f_hi = b1 < 0 ? -INFINITY : thresh(b1 + 1);

  // ---- 2. keep digit 1 >= b1 per warp, in position order; digit-2 histogram of b1 ----
  // v >= f_keep is v >= f_lo without -inf (an empty pool slot) and NaN
  const float f_keep = f_lo == -INFINITY ? -FLT_MAX : f_lo;
  uint32_t run = 0, sure = 0;
  int c_fail = -1;
#pragma unroll 1
  for (int c = 0; c < n_chunks; ++c) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_timed(&S.bar[warp][c % D], (c / D) & 1));
    if (!ok) {
      c_fail = c;
      break;
    }
    const float* buf = wring + (c % D) * kChunk;
    const int64_t base = wlo + int64_t(c) * kChunk;
    const int n_here = static_cast<int>(min(int64_t(kChunk), whi - base));
    // the lane's 32 values of the chunk: group g (128 values), element u at 128 g + 4 lane + u
    float4 q[kChunk / 128];
#pragma unroll
    for (int g = 0; g < kChunk / 128; ++g) q[g] = *reinterpret_cast<const float4*>(buf + 128 * g + 4 * lane);
    uint32_t mask = 0;  // bit 4 g + u: value (g, u) is kept
#pragma unroll
    for (int g = 0; g < kChunk / 128; ++g) {
      mask |= (q[g].x >= f_keep ? 1u : 0u) << (4 * g);
      mask |= (q[g].y >= f_keep ? 2u : 0u) << (4 * g);
      mask |= (q[g].z >= f_keep ? 4u : 0u) << (4 * g);
      mask |= (q[g].w >= f_keep ? 8u : 0u) << (4 * g);
    }
    if (n_here < kChunk) {  // the sub-slice's last chunk: values past its end are stale
#pragma unroll
      for (int g = 0; g < kChunk / 128; ++g)
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (128 * g + 4 * lane + u >= n_here) mask &= ~(1u << (4 * g + u));
    }
    __syncwarp();  // every lane holds the chunk in registers: lane 0 refills the buffer now
    if (lane == 0 && c + D < n_chunks) {
      fence_proxy_async_smem();
      issue(c + D);
    }
    if (__any_sync(0xffffffffu, mask != 0u)) {
      // per-group kept counts (<= 4) one byte each, groups 0-3 in w0 and 4-7 in w1; an
      // inclusive scan over the lanes stays below 256 per byte (no carries between bytes)
      uint32_t w0 = 0, w1 = 0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        w0 |= static_cast<uint32_t>(__popc((mask >> (4 * g)) & 15u)) << (8 * g);
        w1 |= static_cast<uint32_t>(__popc((mask >> (16 + 4 * g)) & 15u)) << (8 * g);
      }
      uint32_t i0 = w0, i1 = w1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y0 = __shfl_up_sync(0xffffffffu, i0, o), y1 = __shfl_up_sync(0xffffffffu, i1, o);
        if (lane >= o) {
          i0 += y0;
          i1 += y1;
        }
      }
      const uint32_t t0 = __shfl_sync(0xffffffffu, i0, 31), t1 = __shfl_sync(0xffffffffu, i1, 31);
      const uint32_t e0 = i0 - w0, e1 = i1 - w1;  // exclusive, byte-wise (no borrows)
      uint32_t goff = run;                        // first list slot of group g
#pragma unroll
      for (int g = 0; g < kChunk / 128; ++g) {
        const int sh = 8 * (g & 3);
        uint32_t o = goff + (((g < 4 ? e0 : e1) >> sh) & 0xffu);
        goff += ((g < 4 ? t0 : t1) >> sh) & 0xffu;
        const uint32_t bits = (mask >> (4 * g)) & 15u;
        if (bits == 0u) continue;
        const float v[4] = {q[g].x, q[g].y, q[g].z, q[g].w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (!((bits >> u) & 1u)) continue;
          const uint32_t key = order_key(v[u]);
          if (digit1(key) == b1) atomicAdd(&S.h2[digit2(key)], 1u);
          else ++sure;  // (kept keys have digit 1 >= b1)
          const uint64_t e = (static_cast<uint64_t>(key) << 32) |
                             static_cast<uint32_t>(base + 128 * g + 4 * lane + u);
          if (o < static_cast<uint32_t>(kWarpCap)) S.list[warp][o] = e;
          else glist[wlo + o] = e;  // (a warp keeps at most its sub-slice: the region holds them)
          ++o;
        }
      }
      run = goff;
    }
  }
  if (c_fail >= 0 && lane == 0) {
    atomicOr(P.status, kFlagWaitTimeout);
    // copies still in flight into this warp's ring land (bounded) before the CTA moves on
    for (int c = c_fail; c < n_chunks && c < c_fail + D; ++c)
      (void)mbar_wait_timed(&S.bar[warp][c % D], (c / D) & 1);
  }
  sure = __reduce_add_sync(0xffffffffu, sure);
  if (lane == 0) {
    S.wcnt[warp] = run;
    if (sure) atomicAdd(&S.sure, sure);
  }
  __syncthreads();
  cluster_sync_all();  // (1) digit-2 histograms and sure counts of every CTA are visible

  // every CTA has read the digit-1 histogram: clear this CTA's share for the next call
  {
    const int seg1 = kHistBins / static_cast<int>(C);
    for (int i = static_cast<int>(r) * seg1 + tid; i < static_cast<int>(r + 1) * seg1; i += kThreads) hist1[i] = 0;
  }
  const bool have_b1 = b1 >= 0;
  const int seg = kHistBins / static_cast<int>(C);
  if (tid == 0) S.bc[0] = cluster_sum(&S.sure, C);
  if (have_b1) {  // sum segment r of the digit-2 histograms in place
    uint32_t tsum = 0;
    for (int bin = static_cast<int>(r) * seg + tid; bin < static_cast<int>(r + 1) * seg; bin += kThreads) {
      const uint32_t sv = cluster_sum(&S.h2[bin], C);
      S.h2[bin] = sv;
      tsum += sv;
    }
    tsum = __reduce_add_sync(0xffffffffu, tsum);
    if (lane == 0) S.w[warp] = tsum;
    __syncthreads();
    if (tid == 0) {
      uint32_t t = 0;
      for (int i = 0; i < kWarps; ++i) t += S.w[i];
      S.seg_total = t;
    }
  }
  __syncthreads();
  cluster_sync_all();  // (2) summed segments and their totals are visible
  const uint32_t n_sure = S.bc[0];

  // ---- 3. digit 2 of the K-th key ----
  int b2 = -1;
  uint32_t r3 = 0, cnt_b2 = 0;
  if (have_b1) {
    const uint32_t r2 = k > n_sure ? k - n_sure : 1u;  // keys to take from the b1 bin
    if (warp == 0) {  // the segment (CTA) holding the r2-th key from the top; keys above it
      const uint32_t t = static_cast<uint32_t>(lane) < C ? dsmem_ld(dsmem_map(&S.seg_total, static_cast<uint32_t>(lane))) : 0u;
      uint32_t sfx = t;  // segments lane .. C - 1
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, sfx, o);
        if (lane + o < 32) sfx += y;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, static_cast<uint32_t>(lane) < C && sfx >= r2);
      const int qs = hit ? 31 - __clz(static_cast<int>(hit)) : 0;
      const uint32_t s_q = __shfl_sync(0xffffffffu, sfx, qs), t_q = __shfl_sync(0xffffffffu, t, qs);
      const uint32_t s_0 = __shfl_sync(0xffffffffu, sfx, 0);
      if (lane == 0) {
        S.bc[1] = static_cast<uint32_t>(qs);
        S.bc[2] = hit ? s_q - t_q : s_0;
      }
    }
    __syncthreads();
    const uint32_t qs = S.bc[1], cum = S.bc[2];
    // the bins of segment qs (summed in CTA qs): thread t owns `per` of them from the top
    const int per = seg >= kThreads ? seg / kThreads : 1;
    const int top = static_cast<int>(qs) * seg + seg - per * tid;
    uint32_t hv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      hv[i] = (i < per && per * tid + i < seg) ? dsmem_ld(dsmem_map(&S.h2[top - 1 - i], qs)) : 0u;
    int d;
    uint32_t above, cnt;
    block_find_desc<8>(hv, per, seg, r2 - cum, &d, &above, &cnt, S.w, S.res);
    b2 = static_cast<int>(qs) * seg + d;  // (the segment holds the crossing)
    r3 = r2 - cum - above;                // keys to take from the (b1, b2) bin
    cnt_b2 = cnt;
  }
  const bool tie = have_b1 && r3 < cnt_b2;  // the (b1, b2) bin is taken in part
  const uint32_t pre24 = tie ? (static_cast<uint32_t>(b1) << 12) | static_cast<uint32_t>(b2) : 0u;
  const uint32_t wcnt = S.wcnt[warp];
  auto entry = [&](uint32_t j) -> uint64_t {
    return j < static_cast<uint32_t>(kWarpCap) ? S.list[warp][j]
                                               : __ldcg(reinterpret_cast<const unsigned long long*>(glist) + wlo + j);
  };

  // ---- 4. the (b1, b2) bin: the last 8 key bits, then the lowest positions ----
  uint32_t ustar = 0;
  int64_t pos_star = INT64_MAX;
  if (tie) {
    for (uint32_t j = lane; j < wcnt; j += 32) {
      const uint32_t key = ent_key(entry(j));
      if ((key >> 8) == pre24) atomicAdd(&S.h8[key & 255u], 1u);
    }
    __syncthreads();
    cluster_sync_all();  // (3) last-8-bit histograms visible
    if (tid < 256) S.hsum[tid] = cluster_sum(&S.h8[tid], C);
    __syncthreads();
    uint32_t hv[1] = {tid < 256 ? S.hsum[255 - tid] : 0u};
    int d3;
    uint32_t above3, cnt3;
    block_find_desc<1>(hv, 1, 256, r3, &d3, &above3, &cnt3, S.w, S.res);
    ustar = (pre24 << 8) | static_cast<uint32_t>(d3);
    uint32_t rr = r3 - above3;  // keys equal to ustar to take, lowest positions first
    if (rr < cnt3) {
      uint64_t pprefix = 0;
      for (int pass = 0; pass < 4; ++pass) {  // 8-bit passes over the positions, from the top
        const int shift = 24 - 8 * pass;
        uint32_t* hp = S.hp[pass & 1];
        if (tid < 256) hp[tid] = 0;
        __syncthreads();
        for (uint32_t j = lane; j < wcnt; j += 32) {
          const uint64_t e = entry(j);
          if (ent_key(e) != ustar) continue;
          const uint64_t pos = static_cast<uint64_t>(position_of(P, b, ent_idx(e)));
          if ((pos >> (shift + 8)) == pprefix) atomicAdd(&hp[(pos >> shift) & 255], 1u);
        }
        __syncthreads();
        cluster_sync_all();  // (4 + pass) position-digit histograms visible
        if (tid < 256) S.hsum[tid] = cluster_sum(&hp[tid], C);
        __syncthreads();
        // lowest digit first: thread t holds bin t as the (255 - t)-th bin from the top
        uint32_t hq[1] = {tid < 256 ? S.hsum[tid] : 0u};
        int dv;
        uint32_t below, cntd;
        block_find_desc<1>(hq, 1, 256, rr, &dv, &below, &cntd, S.w, S.res);
        rr -= below;
        pprefix = (pprefix << 8) | static_cast<uint64_t>(dv < 0 ? 255 : 255 - dv);
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

  // ---- 5. count, place and write the selection ----
  // A Reindex pool whose valid blocks are strictly ascending in slot order keeps positions
  // ascending in slot order: then no sort is needed. Thread t checks slots [8 t, 8 t + 8)
  // and that its first valid block exceeds every valid block before it (8 slots per thread).
  bool in_order = true;
  if (P.mode == 2) {
    const int32_t* pl = P.pool + int64_t(b) * P.npb;
    int32_t mx = -1, first = -1;
    bool ok = true;
    for (int i = tid * 8; i < P.npb && i < tid * 8 + 8; ++i) {
      const int32_t j = pl[i];
      if (j < 0) continue;
      if (first < 0) first = j;
      ok = ok && j > mx;
      mx = j;
    }
    int32_t run_max = mx;  // inclusive running max over the threads of the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, run_max, o);
      if (lane >= o) run_max = max(run_max, y);
    }
    int32_t prev = __shfl_up_sync(0xffffffffu, run_max, 1);
    if (lane == 0) prev = -1;
    if (lane == 31) S.w[warp] = static_cast<uint32_t>(run_max + 1);
    __syncthreads();
    for (int i = 0; i < warp; ++i) prev = max(prev, static_cast<int32_t>(S.w[i]) - 1);
    ok = ok && (first < 0 || first > prev);
    in_order = __syncthreads_and(ok) != 0;
  }
  {
    uint32_t m = 0;
    for (uint32_t j = lane; j < wcnt; j += 32) m += selected(entry(j)) ? 1u : 0u;
    m = __reduce_add_sync(0xffffffffu, m);
    if (lane == 0) S.wsel[warp] = m;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t t = 0;
    for (int w = 0; w < kWarps; ++w) t += S.wsel[w];
    S.sel_total = t;
  }
  __syncthreads();
  cluster_sync_all();  // (5) per-CTA selection counts visible
  if (tid < 32) {
    uint32_t before = 0, all = 0;
    if (static_cast<uint32_t>(lane) < C) {
      const uint32_t c = dsmem_ld(dsmem_map(&S.sel_total, static_cast<uint32_t>(lane)));
      all = c;
      before = static_cast<uint32_t>(lane) < r ? c : 0u;
    }
    before = __reduce_add_sync(0xffffffffu, before);
    all = __reduce_add_sync(0xffffffffu, all);
    if (lane == 0) {
      S.bc[1] = before;
      S.bc[2] = all;
    }
  }
  __syncthreads();
  uint32_t off = S.bc[1];
  const uint32_t total_sel = S.bc[2];
  for (int w = 0; w < warp; ++w) off += S.wsel[w];
  int32_t* oi = P.out_idx + int64_t(b) * P.k;
  float* os = P.out_score ? P.out_score + int64_t(b) * P.k : nullptr;
  for (uint32_t j0 = 0; j0 < wcnt; j0 += 32) {
    const uint32_t j = j0 + lane;
    const uint64_t e = j < wcnt ? entry(j) : 0ull;
    const bool t = j < wcnt && selected(e);
    const uint32_t bal = __ballot_sync(0xffffffffu, t);
    const uint32_t o = off + __popc(bal & ((1u << lane) - 1u));
    if (t && o < k) {
      const int32_t i = ent_idx(e);
      if (in_order) {
        oi[o] = static_cast<int32_t>(position_of(P, b, i));
        if (os) os[o] = key_to_float(ent_key(e));
      } else {  // (position, value index) into CTA 0's pair buffer
        dsmem_st64(dsmem_map(s_pairs + o, 0),
                   (static_cast<uint64_t>(position_of(P, b, i)) << 32) | static_cast<uint32_t>(i));
      }
    }
    off += __popc(bal);
  }
  const uint32_t m = total_sel < k ? total_sel : k;
  if (in_order) {
    for (uint32_t j = m + r * kThreads + tid; j < k; j += C * kThreads) {
      oi[j] = -1;
      if (os) os[j] = -INFINITY;
    }
  }
  __syncthreads();
  cluster_sync_all();  // (6) remote reads done, pool pairs delivered: CTAs may leave
  if (!in_order && r == 0) {
    for (uint32_t i = m + tid; i < static_cast<uint32_t>(kMaxSel); i += kThreads) s_pairs[i] = ~0ull;
    __syncthreads();
    block_sort_pairs(s_pairs);
    for (uint32_t j = tid; j < k; j += kThreads) {
      if (j < m) {
        oi[j] = static_cast<int32_t>(s_pairs[j] >> 32);
        if (os) os[j] = vals[static_cast<uint32_t>(s_pairs[j] & 0xffffffffu)];
      } else {
        oi[j] = -1;
        if (os) os[j] = -INFINITY;
      }
    }
  }
}

// per device, cluster size 2^i and ring depth: clusters that can be resident at once
// (0: not asked yet, -1: none)
int g_sel_clusters[64][5][kMaxDepth + 1] = {};

int sel_max_clusters(int cluster, int depth) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  int li = 0;
  while ((1 << li) < cluster) ++li;
  int& known = g_sel_clusters[dev & 63][li][depth];
  if (known == 0) {
    known = -1;
    if (cluster > 8 && cudaFuncSetAttribute(k_topk_select, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      return known;
    cudaLaunchConfig_t q = {};
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.gridDim = dim3(cluster, 1, 1);
    q.blockDim = dim3(kThreads);
    q.dynamicSmemBytes = select_smem(depth);
    q.attrs = qa;
    q.numAttrs = 1;
    int nc = 0;
    if (cudaOccupancyMaxActiveClusters(&nc, k_topk_select, &q) == cudaSuccess && nc > 0) known = nc;
    (void)cudaGetLastError();
  }
  return known;
}

}  // namespace

cudaError_t launch_topk_select(const SelectProblem* probs, int n_probs, int B, int num_sms, cudaStream_t stream) {
  if (n_probs < 1 || n_probs > kMaxProblems || B == 0) return cudaSuccess;
  SelectArgs args{};
  int64_t n_max = 0;
  for (int i = 0; i < n_probs; ++i) {
    args.p[i] = probs[i];
    const int64_t nv = probs[i].mode == 2 ? int64_t(probs[i].npb) * 8 : probs[i].vstride;
    if (nv > n_max) n_max = nv;
  }
  cudaError_t e = cudaFuncSetAttribute(k_topk_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(select_smem(kMaxDepth)));
  if (e != cudaSuccess) return e;
  // CTAs per sequence: a power of two up to 16, at least 4096 values each, the whole grid
  // within about one CTA per SM, and every cluster resident at once
  int cluster = 1;
  while (cluster < kMaxCluster && n_max / (2 * cluster) >= 4096 &&
         int64_t(B) * n_probs * 2 * cluster <= num_sms)
    cluster *= 2;
  auto depth_for = [&](int c) {
    const int64_t per_warp = (n_max + int64_t(c) * kWarps - 1) / (int64_t(c) * kWarps);
    const int64_t chunks = (per_warp + kChunk - 1) / kChunk;
    return static_cast<int>(chunks < 1 ? 1 : (chunks > kMaxDepth ? kMaxDepth : chunks));
  };
  while (cluster > 1) {
    const int nc = sel_max_clusters(cluster, depth_for(cluster));
    if (nc >= B * n_probs) break;
    cluster >>= 1;
  }
  args.depth = depth_for(cluster);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // a programmatic dependent of the scoring kernel before it on the stream
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cluster, B, n_probs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = select_smem(args.depth);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, k_topk_select, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4kv
