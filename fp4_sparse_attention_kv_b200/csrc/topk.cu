// Exact top-K select per sequence: the K largest fp32 values, ties to the lower position,
// returned as positions in ascending order padded with -1.
//
// Used for the indexer top-K ([PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로
// 줄이고 …", section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2": each Full or Reindex
// layer produces its own top-K indices) and for the candidate pool (section "계층적 희소
// 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기": the blocks with the highest block max).
//
// Values are mapped to order-preserving 32-bit keys. The scoring kernel has already built a
// histogram of the top 12 key bits (digit 1) of every sequence and, for the scores, the
// largest key of every group of 32 consecutive values. One kernel follows, with one
// thread-block cluster of C CTAs per (problem, sequence); CTA r owns slice r of the values,
// warp w of it sub-slice w (slices and sub-slices in position order):
//  1. every CTA finds the digit-1 value b1 of the K-th largest key from the histogram, as a
//     float threshold: "digit 1 >= b1" is v >= f_lo;
//  2. each warp reads only the groups of its sub-slice whose largest key reaches b1 (a few
//     percent of them for the top 2048 of a million), 16 groups in flight at a time, keeps
//     the values >= f_lo in position order (a ballot prefix, no block barrier) in its own
//     list, and the CTA histograms the next 12 key bits (digit 2) of the keys with
//     digit 1 == b1;
//  3. after one cluster barrier, warp 0 of every CTA adds up the CTAs' coarse digit-2 bins
//     (digit 2 / 64) and then the 64 fine bins of the coarse bin that holds the K-th key,
//     through distributed shared memory, and finds its digit-2 value b2 (no second barrier);
//  4. when the (b1, b2) bin is taken in part and holds at most 64 keys, every CTA publishes
//     those keys (rank value: key, then lower position) with its count of certain
//     selections; a larger bin is resolved by histograms of the last 8 key bits and then of
//     the positions among the keys equal to the K-th key, one cluster barrier each;
//  5. after the next barrier every CTA ranks the published keys, reads the counts of the CTAs
//     before it and writes its positions at that offset: ascending without a sort. A Reindex
//     pool whose blocks are not in ascending order gathers its at most 4096 selected pairs in
//     CTA 0, which sorts them.
// The CTAs also clear the scoring kernel's histogram for the next call. Cluster barriers are
// the only synchronisation between CTAs; nothing waits on a flag.
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
constexpr int kBatch = 16;                // 32-value groups a warp loads at once
constexpr int kWords = 8;                 // 32-group words of group maxima loaded at once
constexpr int kCandCap = 32 * kWords;     // candidate groups a warp lists per round
constexpr int kWarpCap = 256;             // kept entries per warp held in shared memory
constexpr int kMaxCluster = 16;
constexpr int kMaxSel = 4096;
constexpr int kMaxProblems = 2;
constexpr int kTieCap = 64;               // a (b1, b2) bin of at most this many keys is ranked directly

struct SelectArgs {
  SelectProblem p[kMaxProblems];
};

struct SelSmem {
  uint64_t pairs[kMaxSel];              // pool mode: (position, value index), CTA 0 sorts them
  uint32_t h2[kHistBins];               // digit 2 of this CTA's kept keys with digit 1 = b1
  uint64_t list[kWarps][kWarpCap];      // kept entries: (order key << 32) | value index
  uint32_t cand[kWarps][kCandCap];      // candidate groups of a round, in position order
  uint32_t h2c[64];                     // the same keys' digit 2 / 64 (coarse digit-2 bins)
  uint32_t h8[256];                     // last 8 key bits of the (b1, b2) bin
  uint32_t hp[2][256];                  // position digits among the keys equal to the K-th
  uint32_t hsum[256];                   // a 256-bin histogram summed over the cluster
  uint64_t tie[kTieCap];                // this CTA's keys of a partly taken (b1, b2) bin: rank values
  uint64_t tall[kTieCap];               // the whole cluster's, gathered
  uint32_t tsrc[kTieCap];               // CTA of each gathered one
  uint32_t tsel[kMaxCluster];           // how many of each CTA's are taken
  uint32_t tie_n;
  uint32_t wcnt[kWarps];                // kept entries per warp
  uint32_t wsel[kWarps];                // selected entries per warp
  uint32_t w[kWarps];                   // block scans
  uint32_t res[4];
  uint32_t sure;                        // keys of this CTA with digit 1 > b1
  uint32_t sel_total;                   // entries this CTA takes for certain (before the small-bin ranking)
  uint32_t bc[4];                       // block broadcasts
};
constexpr size_t kSelSmem = sizeof(SelSmem);

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
FP4KV_DEV uint64_t dsmem_ld64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
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

// the sums over the cluster's CTAs of the u32 at p0 and at p1 (all 2 C loads issued first)
FP4KV_DEV void cluster_sum2(const uint32_t* p0, const uint32_t* p1, uint32_t C, uint32_t* s0, uint32_t* s1) {
  uint32_t v0[kMaxCluster], v1[kMaxCluster];
#pragma unroll
  for (uint32_t q = 0; q < kMaxCluster; ++q) {
    v0[q] = q < C ? dsmem_ld(dsmem_map(p0, q)) : 0u;
    v1[q] = q < C ? dsmem_ld(dsmem_map(p1, q)) : 0u;
  }
  uint32_t a = 0, c = 0;
#pragma unroll
  for (int q = 0; q < kMaxCluster; ++q) {
    a += v0[q];
    c += v1[q];
  }
  *s0 = a;
  *s1 = c;
}

// An L2 load the compiler keeps in program order (volatile, with a memory clobber): a batch's
// loads are then all in flight before the first of them is consumed, which the compiler
// otherwise does not guarantee under this kernel's register limit
FP4KV_DEV float ld_cg_ordered(const float* p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
  return v;
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

// Warp-wide: lane l holds the counts of bins 2 l and 2 l + 1 counted from the top. Finds the
// bin (from the top) at which the count from the top reaches r (r >= 1), the count above it
// and its own count, in every lane; if the total is below r, the lowest bin (63) with the
// total above it and a count of 0.
FP4KV_DEV void warp_find_desc2(uint32_t x0, uint32_t x1, uint32_t r, int* pos, uint32_t* above, uint32_t* cnt) {
  const uint32_t sum = x0 + x1;
  const uint32_t incl = warp_incl_scan(sum);
  const uint32_t excl = incl - sum;
  const uint32_t hit = __ballot_sync(0xffffffffu, excl < r && incl >= r);
  if (hit == 0u) {
    *pos = 63;
    *above = __shfl_sync(0xffffffffu, incl, 31);
    *cnt = 0;
    return;
  }
  const int l = __ffs(static_cast<int>(hit)) - 1;
  const uint32_t e = __shfl_sync(0xffffffffu, excl, l), a0 = __shfl_sync(0xffffffffu, x0, l);
  const uint32_t a1 = __shfl_sync(0xffffffffu, x1, l);
  const bool first = e + a0 >= r;
  *pos = 2 * l + (first ? 0 : 1);
  *above = first ? e : e + a0;
  *cnt = first ? a0 : a1;
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
  const SelectProblem& P = args.p[blockIdx.z];
  const int b = blockIdx.y;
  const uint32_t C = cluster_nctas(), r = cluster_ctarank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int i = tid; i < kHistBins; i += kThreads) S.h2[i] = 0;
  if (tid < 256) S.h8[tid] = 0;
  if (tid < 64) S.h2c[tid] = 0;
  if (tid < kMaxCluster) S.tsel[tid] = 0;
  if (tid == 0) {
    S.sure = 0;
    S.tie_n = 0;
  }
  griddep_wait();  // the scores, group maxima and digit-1 histogram are complete past here

  const int64_t n = n_values(P, b);
  const uint32_t k = static_cast<uint32_t>(P.k);
  const float* vals = P.values + int64_t(b) * P.vstride;
  uint64_t* glist = P.list + int64_t(b) * P.vstride;
  uint32_t* hist1 = P.hist + int64_t(b) * kHistBins;
  // slices in position order, multiples of 128 values
  const int64_t per_cta = ((n + C - 1) / C + 127) / 128 * 128;
  const int64_t lo = min(n, per_cta * r), hi = min(n, lo + per_cta);
  const int64_t per_w = ((hi - lo + kWarps - 1) / kWarps + 127) / 128 * 128;
  const int64_t wlo = min(hi, lo + per_w * warp), whi = min(hi, wlo + per_w);
  // the warp's 32-value groups (wlo is a multiple of 128, so they are the scan's groups)
  const int64_t n_grp = (whi - wlo + 31) / 32;
  const uint32_t* gk = P.gmax != nullptr ? P.gmax + int64_t(b) * P.gstride + wlo / 32 : nullptr;
  // group maxima of groups g0 + 32 j + lane (0xffffffff without maxima: every group is read,
  // 0 past the sub-slice); the first round's load while the first digit is found
  uint32_t gkv[kWords];
  auto load_gmax = [&](int64_t g0) {
#pragma unroll
    for (int j = 0; j < kWords; ++j) {
      const int64_t g = g0 + 32 * j + lane;
      gkv[j] = g < n_grp ? (gk != nullptr ? __ldcg(gk + g) : 0xffffffffu) : 0u;
    }
  };
  load_gmax(0);

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

  // ---- 2. keep digit 1 >= b1 per warp, in position order; digit-2 histogram of b1 ----
  // v >= f_keep is v >= f_lo without -inf (an empty pool slot) and NaN. A group whose largest
  // key is below f_keep's holds nothing to keep and is not read.
  const float f_keep = f_lo == -INFINITY ? -FLT_MAX : f_lo;
  const uint32_t k_keep = order_key(f_keep);
  const uint32_t below = (1u << lane) - 1u;
  uint32_t run = 0, sure = 0;
#pragma unroll 1
  for (int64_t g0 = 0; g0 < n_grp; g0 += kCandCap) {
    // list the round's candidate groups (all of its maxima are already loading)
    if (g0 > 0) load_gmax(g0);
    uint32_t n_cand = 0;
#pragma unroll
    for (int j = 0; j < kWords; ++j) {
      const uint32_t cm = __ballot_sync(0xffffffffu, gkv[j] >= k_keep);  // (0 past the end)
      if ((cm >> lane) & 1u) S.cand[warp][n_cand + __popc(cm & below)] = static_cast<uint32_t>(g0 + 32 * j + lane);
      n_cand += __popc(cm);
    }
    __syncwarp();
    // read them kBatch at a time (lane l: value l of each group), keep in position order
#pragma unroll 1
    for (uint32_t c0 = 0; c0 < n_cand; c0 += kBatch) {
      int32_t gq[kBatch];  // group within the sub-slice (-1: none)
      float v[kBatch];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        gq[q] = c0 + q < n_cand ? static_cast<int32_t>(S.cand[warp][c0 + q]) : -1;
        const int64_t i = wlo + 32 * int64_t(gq[q]) + lane;
        v[q] = -INFINITY;
        if (gq[q] >= 0 && i < whi) v[q] = ld_cg_ordered(vals + i);
      }
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        if (gq[q] < 0) break;
        const bool keep = v[q] >= f_keep;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) {
          const uint32_t key = order_key(v[q]);
          const uint32_t o = run + __popc(bal & below);
          const uint64_t e = (static_cast<uint64_t>(key) << 32) | static_cast<uint32_t>(wlo + 32 * int64_t(gq[q]) + lane);
          if (o < static_cast<uint32_t>(kWarpCap)) S.list[warp][o] = e;
          else glist[wlo + o] = e;  // (a warp keeps at most its sub-slice: the region holds them)
        }
        run += __popc(bal);
      }
    }
    __syncwarp();  // the candidate list is read before the next round rewrites it
  }
  // the digit-2 histograms of the kept keys with digit 1 == b1 and the count of those above
  // it, one kept entry per lane (inside the loop above, the histogram atomics ran with one or
  // two lanes active per group and cost ~2 us of the select on 1 M values)
  for (uint32_t j = lane; j < run; j += 32) {
    const uint32_t key = ent_key(j < static_cast<uint32_t>(kWarpCap) ? S.list[warp][j] : glist[wlo + j]);
    if (digit1(key) == b1) {
      atomicAdd(&S.h2[digit2(key)], 1u);
      atomicAdd(&S.h2c[digit2(key) >> 6], 1u);
    } else {
      ++sure;  // (kept keys have digit 1 >= b1)
    }
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

  // ---- 3. digit 2 of the K-th key, from the cluster's digit-2 histogram: its 64 coarse bins
  // (digit 2 / 64) from the top, then the 64 bins of the coarse bin that holds the crossing.
  // Warp 0 alone; the histograms are final since barrier (1).
  int b2 = -1;
  uint32_t r3 = 0, cnt_b2 = 0;
  if (have_b1) {
    if (warp == 0) {
      // (the counts above b1 and the coarse bins load in one round trip)
      const uint32_t su = static_cast<uint32_t>(lane) < C ? dsmem_ld(dsmem_map(&S.sure, static_cast<uint32_t>(lane))) : 0u;
      uint32_t x0, x1;
      cluster_sum2(&S.h2c[63 - 2 * lane], &S.h2c[62 - 2 * lane], C, &x0, &x1);
      const uint32_t n_sure = __reduce_add_sync(0xffffffffu, su);
      const uint32_t r2 = k > n_sure ? k - n_sure : 1u;  // keys to take from the b1 bin
      int pc;
      uint32_t above_c, cnt_c;
      warp_find_desc2(x0, x1, r2, &pc, &above_c, &cnt_c);
      const int cb = 63 - pc;
      cluster_sum2(&S.h2[64 * cb + 63 - 2 * lane], &S.h2[64 * cb + 62 - 2 * lane], C, &x0, &x1);
      int pf;
      uint32_t above_f, cnt_f;
      warp_find_desc2(x0, x1, r2 - above_c, &pf, &above_f, &cnt_f);
      if (lane == 0) {
        S.bc[0] = static_cast<uint32_t>(64 * cb + 63 - pf);
        S.bc[1] = r2 - above_c - above_f;  // keys to take from the (b1, b2) bin
        S.bc[2] = cnt_f;
      }
    }
    __syncthreads();
    b2 = static_cast<int>(S.bc[0]);
    r3 = S.bc[1];
    cnt_b2 = S.bc[2];
    __syncthreads();  // (S.bc is reused below)
  }
  const bool tie = have_b1 && r3 < cnt_b2;  // the (b1, b2) bin is taken in part
  // a small such bin is ranked directly, key first and then the lower position; a larger one
  // (many equal or near-equal keys) by histograms of the last 8 key bits and the positions
  const bool small_tie = tie && cnt_b2 <= static_cast<uint32_t>(kTieCap);
  const uint32_t pre24 = have_b1 ? (static_cast<uint32_t>(b1) << 12) | static_cast<uint32_t>(b2) : 0u;
  const uint32_t wcnt = S.wcnt[warp];
  auto entry = [&](uint32_t j) -> uint64_t {
    return j < static_cast<uint32_t>(kWarpCap) ? S.list[warp][j]
                                               : __ldcg(reinterpret_cast<const unsigned long long*>(glist) + wlo + j);
  };
  // rank value of an entry: larger = taken first (larger key, then lower position)
  auto rank_value = [&](uint64_t e) -> uint64_t {
    const uint32_t pos = static_cast<uint32_t>(position_of(P, b, ent_idx(e)));
    return (static_cast<uint64_t>(ent_key(e)) << 32) | static_cast<uint64_t>(0xffffffffu - pos);
  };

  // ---- 4. a large partly taken (b1, b2) bin: the last 8 key bits, then the lowest positions ----
  uint32_t ustar = 0;
  int64_t pos_star = INT64_MAX;
  if (tie && !small_tie) {
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
  // taken for certain (every entry when the bin is not ranked directly)
  auto certain = [&](uint64_t e) -> bool {
    if (!have_b1) return true;
    const uint32_t key = ent_key(e);
    const uint32_t k24 = key >> 8;
    if (k24 != pre24) return k24 > pre24;
    if (!tie) return true;
    if (small_tie) return false;
    return key > ustar || (key == ustar && position_of(P, b, ent_idx(e)) <= pos_star);
  };
  auto in_small_tie = [&](uint64_t e) -> bool { return small_tie && (ent_key(e) >> 8) == pre24; };

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
  {  // what this CTA takes for certain, and the keys of a small partly taken bin
    uint32_t m = 0;
    for (uint32_t j = lane; j < wcnt; j += 32) {
      const uint64_t e = entry(j);
      m += certain(e) ? 1u : 0u;
      if (in_small_tie(e)) {
        const uint32_t slot = atomicAdd(&S.tie_n, 1u);
        if (slot < static_cast<uint32_t>(kTieCap)) S.tie[slot] = rank_value(e);
      }
    }
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
  cluster_sync_all();  // (5) per-CTA certain counts and small-bin keys visible
  if (warp == 0) {
    // gather the small bin's keys of every CTA, take its r3 best, and place this CTA after
    // everything the CTAs before it take
    const bool q_ok = static_cast<uint32_t>(lane) < C;
    const uint32_t cq = q_ok ? dsmem_ld(dsmem_map(&S.sel_total, static_cast<uint32_t>(lane))) : 0u;
    uint32_t nq = 0;
    if (small_tie && q_ok) nq = min(dsmem_ld(dsmem_map(&S.tie_n, static_cast<uint32_t>(lane))), static_cast<uint32_t>(kTieCap));
    const uint32_t incl = warp_incl_scan(nq);  // CTA q's keys go to [incl_q - n_q, incl_q)
    const uint32_t n_all = min(__shfl_sync(0xffffffffu, incl, 31), static_cast<uint32_t>(kTieCap));
    for (uint32_t i0 = 0; i0 < n_all; i0 += 32) {
      const uint32_t i = i0 + lane;
      uint32_t q = 0, qbase = 0;  // the CTA whose range holds i, and where that range starts
      for (uint32_t qq = 0; qq < C; ++qq) {
        const uint32_t end_q = __shfl_sync(0xffffffffu, incl, static_cast<int>(qq));
        if (i >= end_q) {
          q = qq + 1;
          qbase = end_q;
        }
      }
      if (i < n_all) {
        S.tall[i] = dsmem_ld64(dsmem_map(&S.tie[i - qbase], q));
        S.tsrc[i] = q;
      }
    }
    __syncwarp();
    for (uint32_t i = lane; i < n_all; i += 32) {
      const uint64_t v = S.tall[i];
      uint32_t better = 0;
      for (uint32_t j = 0; j < n_all; ++j) better += S.tall[j] > v ? 1u : 0u;
      if (better < r3) atomicAdd(&S.tsel[S.tsrc[i]], 1u);
    }
    __syncwarp();
    const uint32_t tq = q_ok ? cq + S.tsel[lane] : 0u;
    const uint32_t before = __reduce_add_sync(0xffffffffu, static_cast<uint32_t>(lane) < r ? tq : 0u);
    const uint32_t all = __reduce_add_sync(0xffffffffu, tq);
    if (lane == 0) {
      S.bc[1] = before;
      S.bc[2] = all;
      S.bc[3] = n_all;
    }
  }
  // (6) this CTA has read everything it needs from the others: arrive now, wait only before
  // leaving, so that the barrier's latency hides behind the writes below. When the pool
  // mode's pairs go to CTA 0, arrive after they are delivered instead.
  if (in_order) cluster_arrive();
  __syncthreads();
  const uint32_t n_tie_all = S.bc[3];
  auto selected = [&](uint64_t e) -> bool {
    if (certain(e)) return true;
    if (!in_small_tie(e)) return false;
    const uint64_t v = rank_value(e);
    uint32_t better = 0;
    for (uint32_t j = 0; j < n_tie_all; ++j) better += S.tall[j] > v ? 1u : 0u;
    return better < r3;
  };
  if (small_tie) {  // per-warp counts with the small bin's keys that are taken
    uint32_t m = 0;
    for (uint32_t j = lane; j < wcnt; j += 32) m += selected(entry(j)) ? 1u : 0u;
    m = __reduce_add_sync(0xffffffffu, m);
    __syncthreads();
    if (lane == 0) S.wsel[warp] = m;
    __syncthreads();
  }
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
        dsmem_st64(dsmem_map(S.pairs + o, 0),
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
  if (!in_order) {
    __syncthreads();
    cluster_arrive();
  }
  cluster_wait();  // (6) remote reads done, pool pairs delivered: CTAs may leave
  if (!in_order && r == 0) {
    for (uint32_t i = m + tid; i < static_cast<uint32_t>(kMaxSel); i += kThreads) S.pairs[i] = ~0ull;
    __syncthreads();
    block_sort_pairs(S.pairs);
    for (uint32_t j = tid; j < k; j += kThreads) {
      if (j < m) {
        oi[j] = static_cast<int32_t>(S.pairs[j] >> 32);
        if (os) os[j] = vals[static_cast<uint32_t>(S.pairs[j] & 0xffffffffu)];
      } else {
        oi[j] = -1;
        if (os) os[j] = -INFINITY;
      }
    }
  }
}

// per device and cluster size 2^i: clusters that can be resident at once (0: not asked
// yet, -1: none)
int g_sel_clusters[64][5] = {};

int sel_max_clusters(int cluster) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  int li = 0;
  while ((1 << li) < cluster) ++li;
  int& known = g_sel_clusters[dev & 63][li];
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
    q.dynamicSmemBytes = kSelSmem;
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
                                       static_cast<int>(kSelSmem));
  if (e != cudaSuccess) return e;
  // CTAs per sequence: a power of two up to 16, at least 2048 values each, the whole grid
  // within about one CTA per SM, and every cluster resident at once
  int cluster = 1;
  while (cluster < kMaxCluster && n_max / (2 * cluster) >= 2048 &&
         int64_t(B) * n_probs * 2 * cluster <= num_sms)
    cluster *= 2;
  while (cluster > 1) {
    const int nc = sel_max_clusters(cluster);
    if (nc >= B * n_probs) break;
    cluster >>= 1;
  }
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
  cfg.dynamicSmemBytes = kSelSmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, k_topk_select, args);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4kv
