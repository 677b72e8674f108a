// sparse_attn_decode: gather the top-K rows of the FP4 cache, dequantize them exactly and
// run softmax attention for every query head (one latent row is both key and value).
//
// Method: [PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로 줄이고 …", section
// "890바이트를 만든 나머지 절반, FP4 KV 캐시와 지속 캐시 재설계" (the cache is dequantized before
// attention; FP4 serves storage only) and section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는
// CSA2" (attention over the top-K indices; a Reuse layer attends over the indices of the layer
// before it); [ingu627] section "MoE 라우팅과 하드웨어 병목의 분리 매칭" (64 query heads share a
// single KV head).
//
// Numerics:
//  * v_hat = e2m1 x e4m3 is exact in fp16 (at most 6 significant bits, |v| in [2^-10, 2688]).
//  * q (bf16) is multiplied per head by a power of two 2^k so that max|q| lies in
//    [2^14, 2^15), then rounded to fp16: exact for every element within 2^29 of the head's
//    max; 2^-k is folded back into the logit scale.
//  * S = q . v_hat on tensor cores (fp16 x fp16 -> fp32); softmax in fp32 with exp2 against a
//    per-head reference m. The reference moves only when a logit exceeds it by more than 2^9
//    (so p < 2^9); it is then set 2^3 above the new maximum, and O and the row sums are
//    rescaled once for every head that moved.
//  * P is split as P_hi + P_lo, both fp16, after scaling by 2^6 (fp16 stays in range and P_lo
//    out of the subnormal range); P.V is two MMAs, so P carries ~22 bits into the product.
//
// Kernel (one CTA per (chunk of the index list, group of 64 heads, sequence); 13 warps):
//  * the tile is 128 selected entries. S^T = V_hat Q^T (M = 128 entries, N = 64 heads,
//    K = 512) and O^T += V_hat^T P^T (M = 128 dims x 4, K = 128 entries) run on tcgen05 with
//    fp32 accumulators in TMEM. An MMA costs the same for N = 64 and N = 128, so for three of
//    the four dim tiles P_hi and P_lo are one N = 128 operand (heads, then the same heads
//    again) with separate accumulators that are added at the end; the fourth dim tile, for
//    which the 512 TMEM columns have no room left beside S^T, takes two N = 64 MMAs per step
//    into one accumulator.
//  * warps 8-11 gather: each thread loads one selected row (256 B codes + 32 B scales) with
//    16-byte loads, dequantizes it 64 dims at a time into a 128-byte-swizzled fp16 chunk
//    buffer (8 chunks = the tile's 128 KiB V_hat) that serves as the K-major A operand of
//    S^T and as the MN-major A operand of O^T;
//  * warp 12: TMEM allocation and the single MMA-issuing thread;
//  * warps 0-7 convert Q, then own the 128 TMEM lanes in pairs (warp w: lane quarter w % 4,
//    heads 32 (w / 4) .. + 32): per tile each thread reads its entry's 32 logits, keeps 32
//    per-head running row sums in registers, and writes its half of the entry's row of P^T
//    (MN-major B operand). Cross-lane reductions happen only when a reference moves and
//    once at the end, for the per-head row sums; each thread writes its TMEM lane of O^T
//    straight to the workspace.
//  Per-chunk barriers let the next tile's dequantization overlap the current tile's P.V.
//  * Chunks of the index list go to different CTAs, and the chunk CTAs of one (sequence,
//    head group) form one thread-block cluster. At the end each writes its partial (O and
//    the per-head reference m and row sum l) to the workspace, where it stays in L2; after
//    one cluster barrier CTA r sums its share of the output dims over the chunks with the
//    log-sum-exp weights and writes them, so no second kernel runs.
//  * With a sliding window (the pages' SWA branch, its KV kept in FP8), the last chunk's CTA
//    runs one more tile: the window's E4M3 rows (exact in fp16), in the same softmax as the
//    selected rows, so the window and the sparse selection share one normalisation.
// Every mbarrier wait is bounded in time. Decisions that lead to a named barrier are made
// uniform across the softmax warps by a barrier vote, so a timed-out wait cannot strand a
// warp; on timeout the kernel sets a status bit and winds down.
#include <type_traits>

#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"
#include "fp4kv_sm100.cuh"

namespace fp4kv {
namespace {

constexpr int kD = 512;           // latent width the kernel is built for
constexpr int kHeadsPerCta = 64;  // N of both MMAs (absent heads are zero rows)
constexpr int kTile = 128;        // selected entries per tile
constexpr int kChunks = 8;        // 64-dim chunks of a row
constexpr float kPScale = 64.0f;  // P is stored as p * 2^6
constexpr float kMoveLog2 = 9.0f;     // a logit above m + 9 moves the reference ...
constexpr float kHeadroomLog2 = 3.0f; // ... to 3 above the new maximum
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kSoftWarps = 8;
constexpr int kGatherWarps = 4;
constexpr int kMmaWarp = kSoftWarps + kGatherWarps;
constexpr int kAttnThreads = 32 * (kMmaWarp + 1);  // 416
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr uint32_t kFlagMisaligned = 2u;
constexpr int kMaxCluster = 16;   // chunk CTAs of one (sequence, head group)

constexpr uint32_t kQChunkBytes = kHeadsPerCta * 128;  // 64 heads x 64 dims x 2 B
constexpr uint32_t kVChunkBytes = kTile * 128;         // 128 entries x 64 dims x 2 B
constexpr uint32_t kPBytes = kTile * 128;              // 128 entries x 64 heads x 2 B
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffV = kOffQ + kChunks * kQChunkBytes;
constexpr uint32_t kOffPh = kOffV + kChunks * kVChunkBytes;
constexpr uint32_t kOffPl = kOffPh + kPBytes;
constexpr uint32_t kOffBar = kOffPl + kPBytes;  // 24 mbarriers
constexpr uint32_t kOffC = kOffBar + 256;       // [64] log2-domain logit scale per head
constexpr uint32_t kOffRed = kOffC + 256;       // [4][64] cross-warp exchange
constexpr uint32_t kOffM = kOffRed + 1024;      // [64] per-head reference (log2 domain)
constexpr uint32_t kOffA = kOffM + 256;         // [64] rescale factor of the last move
constexpr uint32_t kOffL = kOffA + 256;         // [64] row sums at the end
constexpr uint32_t kOffMT = kOffL + 256;        // [64] reference + 9: a logit above it moves it
constexpr uint32_t kOffM6 = kOffMT + 256;       // [64] reference - 6: 2^(z - it) is p * 2^6
constexpr uint32_t kOffTmem = kOffM6 + 256;
constexpr uint32_t kSmemAttn = kOffTmem + 16;
static_assert(kSmemAttn <= 232448, "shared memory");
// At the end the V_hat region holds the [64 heads][512 dims] fp32 output tile.
static_assert(kChunks * kVChunkBytes == kHeadsPerCta * kD * 4, "output staging");

// TMEM columns: O^T of dim tile c < 3 at [128c, +64) (P_hi) and [128c + 64, +64) (P_lo);
// dim tile 3 at [384, 448) (both halves); S^T at [448, 512). One S^T slot is enough: S^T of
// tile t + 1 needs V_hat rows that only the end of P.V(t) frees, and P.V(t) starts after
// every softmax warp has read S^T(t).
constexpr uint32_t kColS = 448;
constexpr int kPairTiles = 3;  // dim tiles with separate P_hi and P_lo accumulators
FP4KV_DEV uint32_t o_col(int c) { return 128u * static_cast<uint32_t>(c); }
static_assert(4096 / kTile <= 32, "the per-thread validity mask holds one bit per tile");

enum { B_VREADY = 0, B_VFREE = 8, B_SFULL = 16, B_SFREE = 18, B_PREADY = 20, B_PFREE = 21,
       B_QREADY = 22, B_DONE = 23 };

FP4KV_DEV void softmax_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSoftThreads) : "memory"); }
// Barrier among the softmax warps that also ORs a predicate over them.
FP4KV_DEV bool softmax_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.or.pred po, 1, %2, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}"
      : "=r"(r) : "r"(v ? 1u : 0u), "n"(kSoftThreads) : "memory");
  return r != 0;
}

// 2^x by the hardware's approximate base-2 exponential (PTX ex2.approx.ftz.f32: a few units
// in the last place, results below 2^-126 flushed to zero). The probabilities are at most
// 2^9 and feed a sum of at least 1, and the combine's chunk weights are at most 1 with the
// largest exactly 1, so neither the approximation nor the flush is visible beside the fp16
// hi / lo split of P.
FP4KV_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Butterfly transpose-reduction of 32 values per lane across the warp: on return, lane l
// holds the reduction over all 32 lanes of value l.
template <bool kMax>
FP4KV_DEV float butterfly32(const float (&v)[32]) {
  const int lane = threadIdx.x & 31;
  float a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const bool hi = lane & 16;
    const float r = __shfl_xor_sync(0xffffffffu, hi ? v[i] : v[i + 16], 16);
    const float keep = hi ? v[i + 16] : v[i];
    a[i] = kMax ? fmaxf(keep, r) : keep + r;
  }
  float b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 8;
    const float r = __shfl_xor_sync(0xffffffffu, hi ? a[i] : a[i + 8], 8);
    const float keep = hi ? a[i + 8] : a[i];
    b[i] = kMax ? fmaxf(keep, r) : keep + r;
  }
  float c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 4;
    const float r = __shfl_xor_sync(0xffffffffu, hi ? b[i] : b[i + 4], 4);
    const float keep = hi ? b[i + 4] : b[i];
    c[i] = kMax ? fmaxf(keep, r) : keep + r;
  }
  float d[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 2;
    const float r = __shfl_xor_sync(0xffffffffu, hi ? c[i] : c[i + 2], 2);
    const float keep = hi ? c[i + 2] : c[i];
    d[i] = kMax ? fmaxf(keep, r) : keep + r;
  }
  const bool hi = lane & 1;
  const float r = __shfl_xor_sync(0xffffffffu, hi ? d[0] : d[1], 1);
  const float keep = hi ? d[1] : d[0];
  return kMax ? fmaxf(keep, r) : keep + r;
}

// Wait policies (all return the same value in every lane of the warp). The gather warps
// wait for buffers during the softmax and the MMAs: they poll rarely. The softmax warps
// wait on the critical path.
#ifndef ATTN_GATHER_SLEEP_NS
#define ATTN_GATHER_SLEEP_NS 128
#endif
FP4KV_DEV bool gather_wait(uint64_t* bar, uint32_t parity) {
#if ATTN_GATHER_SLEEP_NS > 0
  return __all_sync(0xffffffffu, mbar_wait_sleepy(bar, parity, ATTN_GATHER_SLEEP_NS));
#else
  return __all_sync(0xffffffffu, mbar_wait_timed(bar, parity));
#endif
}
// (every lane polls: one lane polling and broadcasting resumed the warp measurably later)
FP4KV_DEV bool softmax_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait_timed(bar, parity));
}

FP4KV_DEV void fail_wait(const AttnParams& p, volatile uint32_t* abort_flag) {
  atomicOr(p.status, kFlagWaitTimeout);
  *abort_flag = 1;
}

// Loads the rows of tile t at `pos` (rows row0 + 8 i + qd of the tile, qd = lane / 4,
// i < NG; pos < 0: an all-zero row) and dequantizes them into the V_hat chunk buffers, one
// chunk pair at a time as the P.V of the previous tile frees it. The four lanes of a quad
// share a row, so one warp load covers the same 64-byte slice of eight rows (32 different
// rows per load would multiply the requests in flight, which every load/store instruction
// of the CTA then queues behind). Lane j = lane % 4 holds, for chunk pair cp (dims
// [128 cp, +128) = code bytes [64 cp, +64)), the code bytes [64 cp + 16 j, +16): dims
// [128 cp + 32 j, +32), scale groups 8 cp + 2 j and + 1. Warp-collective; returns false
// (in every lane) if a wait timed out.
template <int NG>
FP4KV_DEV bool load_dequant(uint8_t* smem, uint64_t* bars, const uint8_t* packed_b,
                            const uint8_t* scales_b, const int32_t (&pos)[NG], int row0, int t) {
  const int lane = threadIdx.x & 31, qd = lane >> 2, j = lane & 3;
  uint4 pk[4][NG];  // [chunk pair][row group]
  uint2 s8[NG];     // [row group]: the row's scale bytes [8 j, +8) (those of chunk pair j)
#pragma unroll
  for (int i = 0; i < NG; ++i) {
    if (pos[i] >= 0) {
      const uint8_t* prow = packed_b + int64_t(pos[i]) * (kD / 2) + 16 * j;
#pragma unroll
      for (int cp = 0; cp < 4; ++cp) pk[cp][i] = ld_nc_v4(prow + 64 * cp);
      s8[i] = ld_nc_v2_64b(scales_b + int64_t(pos[i]) * (kD / kGroup) + 8 * j);
    } else {
#pragma unroll
      for (int cp = 0; cp < 4; ++cp) pk[cp][i] = make_uint4(0, 0, 0, 0);
      s8[i] = make_uint2(0, 0);
    }
  }
  bool ok = true;  // (no break inside this fully unrolled loop: registers stay registers)
#pragma unroll
  for (int cp = 0; cp < 4; ++cp) {
    // (both chunks of the pair are released by the same commit point of P.V; this wait is
    // on the critical path, so it polls without sleeping)
    if (ok && !__all_sync(0xffffffffu, mbar_wait_timed(&bars[B_VFREE + 2 * cp], (t & 1) ^ 1) &&
                                           mbar_wait_timed(&bars[B_VFREE + 2 * cp + 1], (t & 1) ^ 1)))
      ok = false;
    if (!ok) continue;
    const int jc = 2 * cp + (j >> 1);  // chunk of this lane's 32 dims
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      const int r = row0 + 8 * i + qd;
      // scale bytes 8 cp + 2 j, + 1 of row r: held by quad lane cp, word j / 2
      const uint32_t w0 = __shfl_sync(0xffffffffu, s8[i].x, 4 * qd + cp);
      const uint32_t w1 = __shfl_sync(0xffffffffu, s8[i].y, 4 * qd + cp);
      const uint32_t sw = ((j >> 1) ? w1 : w0) >> (16 * (j & 1));
      const uint32_t sA = e4m3x2_to_f16x2(static_cast<uint16_t>((sw & 0xffu) * 0x101u));
      const uint32_t sB = e4m3x2_to_f16x2(static_cast<uint16_t>(((sw >> 8) & 0xffu) * 0x101u));
      const uint4 src = pk[cp][i];
      uint8_t* vrow = smem + kOffV + jc * kVChunkBytes + r * 128;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // 8-dim unit uu of this lane's 32 dims; lanes j and j + 2 (same units, different
        // chunks) go in a staggered order so that a store phase hits distinct banks
        const bool st = (j & 2) != 0;
        const int uu0 = k, uu1 = k ^ 2;
        const uint32_t w = st ? (uu1 == 0 ? src.x : uu1 == 1 ? src.y : uu1 == 2 ? src.z : src.w)
                              : (uu0 == 0 ? src.x : uu0 == 1 ? src.y : uu0 == 2 ? src.z : src.w);
        const uint32_t s2 = (st ? uu1 : uu0) < 2 ? sA : sB;
        uint4 o;
        o.x = hmul2_f16(e2m1x2_to_f16x2(w & 0xffu), s2);
        o.y = hmul2_f16(e2m1x2_to_f16x2((w >> 8) & 0xffu), s2);
        o.z = hmul2_f16(e2m1x2_to_f16x2((w >> 16) & 0xffu), s2);
        o.w = hmul2_f16(e2m1x2_to_f16x2(w >> 24), s2);
        const int unit = 4 * (j & 1) + (st ? uu1 : uu0);
        *reinterpret_cast<uint4*>(vrow + ((unit ^ (r & 7)) << 4)) = o;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&bars[B_VREADY + 2 * cp]);
      mbar_arrive(&bars[B_VREADY + 2 * cp + 1]);
    }
  }
  return ok;
}

// The window tile's rows: E4M3 codes, one byte per dim (row pos of this sequence's window
// rows), with load_dequant's lane mapping and V_hat layout (lane j of a quad converts dims
// [128 cp + 32 j, +32) of its row for chunk pair cp). The window tile runs once per CTA, so
// each chunk pair's bytes are loaded just before they are converted.
template <int NG>
FP4KV_DEV bool load_dequant_win(uint8_t* smem, uint64_t* bars, const uint8_t* win_b,
                                const int32_t (&pos)[NG], int row0, int t) {
  const int lane = threadIdx.x & 31, qd = lane >> 2, j = lane & 3;
  bool ok = true;
#pragma unroll
  for (int cp = 0; cp < 4; ++cp) {
    uint4 c8[NG][2];
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      if (pos[i] >= 0) {
        const uint8_t* src = win_b + int64_t(pos[i]) * kD + 128 * cp + 32 * j;
        c8[i][0] = ld_nc_v4(src);
        c8[i][1] = ld_nc_v4(src + 16);
      } else {
        c8[i][0] = c8[i][1] = make_uint4(0, 0, 0, 0);
      }
    }
    if (ok && !__all_sync(0xffffffffu, mbar_wait_timed(&bars[B_VFREE + 2 * cp], (t & 1) ^ 1) &&
                                           mbar_wait_timed(&bars[B_VFREE + 2 * cp + 1], (t & 1) ^ 1)))
      ok = false;
    if (!ok) continue;
    const int jc = 2 * cp + (j >> 1);  // chunk of this lane's 32 dims
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      const int r = row0 + 8 * i + qd;
      uint8_t* vrow = smem + kOffV + jc * kVChunkBytes + r * 128;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int uu = (j & 2) ? (k ^ 2) : k;  // staggered as in load_dequant
        const uint4 h = (uu >> 1) ? c8[i][1] : c8[i][0];  // (selects: no local-memory indexing)
        const uint32_t w0 = (uu & 1) ? h.z : h.x, w1 = (uu & 1) ? h.w : h.y;  // dims [8 uu, +8)
        uint4 o;
        o.x = e4m3x2_to_f16x2(static_cast<uint16_t>(w0 & 0xffffu));
        o.y = e4m3x2_to_f16x2(static_cast<uint16_t>(w0 >> 16));
        o.z = e4m3x2_to_f16x2(static_cast<uint16_t>(w1 & 0xffffu));
        o.w = e4m3x2_to_f16x2(static_cast<uint16_t>(w1 >> 16));
        const int unit = 4 * (j & 1) + uu;
        *reinterpret_cast<uint4*>(vrow + ((unit ^ (r & 7)) << 4)) = o;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&bars[B_VREADY + 2 * cp]);
      mbar_arrive(&bars[B_VREADY + 2 * cp + 1]);
    }
  }
  return ok;
}

// CTA `rank` of a cluster of C chunk CTAs: sums 16-byte units (head, 4 dims) of its dim slice
// [rank * 512 / C, +512 / C) over the C chunk partials with the log-sum-exp weights
// 2^(m_c - M) / (2^6 L) (O holds p * 2^6) and writes them; CTA 0 also writes the lse. Each
// thread loads its units' partials and their heads' (m, l) of every chunk at once (one L2
// round trip) and forms the weights itself: 16 / C units per thread and batch.
template <int C>
FP4KV_DEV void combine_slice(const AttnParams& p, int b, int hbase, int nh, uint32_t rank, int64_t part0) {
  constexpr int kSlice4 = kD / 4 / C;  // 16-byte units per head in the slice
  constexpr int kPer = 16 / C;         // units per thread and batch
  const int tid = threadIdx.x;
  const int n_units = nh * kSlice4;
  const int d0 = static_cast<int>(rank) * kSlice4 * 4;
  const bool al16 = (reinterpret_cast<uintptr_t>(p.out) & 15u) == 0;
  const float4* part4 = reinterpret_cast<const float4*>(p.part_o + part0 * (kHeadsPerCta * kD));
  const float2* ml2 = reinterpret_cast<const float2*>(p.part_ml + part0 * kHeadsPerCta * 2);
  for (int u0 = tid; u0 < n_units; u0 += kAttnThreads * kPer) {
    float4 v[kPer][C];
    float2 ml[kPer][C];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int u = u0 + j * kAttnThreads;
      const int h = u / kSlice4, d = d0 + 4 * (u % kSlice4);
#pragma unroll
      for (int c = 0; c < C; ++c) {
        v[j][c] = u < n_units ? __ldcg(part4 + (int64_t(c) * kHeadsPerCta * kD + h * kD + d) / 4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        ml[j][c] = u < n_units ? __ldcg(ml2 + c * kHeadsPerCta + h) : make_float2(0.f, 0.f);
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int u = u0 + j * kAttnThreads;
      if (u >= n_units) continue;
      const int h = u / kSlice4, d = d0 + 4 * (u % kSlice4);
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < C; ++c)
        if (ml[j][c].y > 0.0f) M = fmaxf(M, ml[j][c].x);
      float Lt = 0.0f;
      float w[C];
#pragma unroll
      for (int c = 0; c < C; ++c) {
        w[c] = ml[j][c].y > 0.0f ? ex2_approx(ml[j][c].x - M) : 0.0f;
        Lt += w[c] * ml[j][c].y;
      }
      const float inv = Lt > 0.0f ? 1.0f / (kPScale * Lt) : 0.0f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const float wc = w[c] * inv;
        acc.x += wc * v[j][c].x; acc.y += wc * v[j][c].y; acc.z += wc * v[j][c].z; acc.w += wc * v[j][c].w;
      }
      float* dst = p.out + (int64_t(b) * p.H + hbase + h) * kD + d;
      if (al16) {
        *reinterpret_cast<float4*>(dst) = acc;
      } else {  // the output is only 8-byte aligned
        reinterpret_cast<float2*>(dst)[0] = make_float2(acc.x, acc.y);
        reinterpret_cast<float2*>(dst)[1] = make_float2(acc.z, acc.w);
      }
      if (rank == 0 && d == 0 && p.lse != nullptr)
        p.lse[int64_t(b) * p.H + hbase + h] = Lt > 0.0f ? M * kLn2 + logf(Lt) : -INFINITY;
    }
  }
}

// kWin: with the sliding-window tile (a separate instantiation, so that the plain sparse
// attention keeps its code size and registers).
template <bool kWin>
__global__ void __launch_bounds__(kAttnThreads, 1) k_sparse_attn_tc(const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // the swizzled operand layouts need 1 KiB alignment
    if (threadIdx.x == 0) atomicOr(p.status, kFlagMisaligned);
    return;
  }
  // The kernel that follows on the stream waits for this grid to complete; let it be
  // scheduled now.
  griddep_launch_dependents();
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  float* sC = reinterpret_cast<float*>(smem + kOffC);
  float* sRed = reinterpret_cast<float*>(smem + kOffRed);
  float* sM = reinterpret_cast<float*>(smem + kOffM);
  float* sA = reinterpret_cast<float*>(smem + kOffA);
  float* sL = reinterpret_cast<float*>(smem + kOffL);
  float* sMT = reinterpret_cast<float*>(smem + kOffMT);
  float* sM6 = reinterpret_cast<float*>(smem + kOffM6);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffTmem);
  volatile uint32_t* s_abort = s_tmem + 1;
  volatile uint32_t* s_fail = s_tmem + 2;  // a softmax wait gave up: this CTA's partial is void

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int n_chunks = gridDim.x;
  const int hbase = hg * kHeadsPerCta;
  const int nh = min(kHeadsPerCta, p.H - hbase);
  int64_t len = p.seq_lens[b];
  if (len > p.cap) len = p.cap;
  const int e_begin = int(int64_t(p.top_k) * chunk / n_chunks);
  const int e_end = int(int64_t(p.top_k) * (chunk + 1) / n_chunks);
  const int n_sel_tiles = (e_end - e_begin + kTile - 1) / kTile;
  // the last chunk's CTA also attends over the sliding window: one more tile, after the
  // selected ones, whose rows are the window slots [0, min(n_win, len))
  const bool has_win = kWin && chunk == n_chunks - 1;
  const int n_tiles = n_sel_tiles + (has_win ? 1 : 0);
  const int n_win_rows = has_win ? int(min(int64_t(p.n_win), len)) : 0;
  const int32_t* idx = p.idx + int64_t(b) * p.top_k;
  const uint8_t* win_b = has_win ? p.swa + int64_t(b) * p.n_win * kD : nullptr;
  // cache position (selected tiles) or window slot (window tile) of row `row` of tile tt;
  // -1 for none
  auto tile_pos = [&](int tt, int row) -> int32_t {
    if (!kWin || tt < n_sel_tiles) {
      const int je = e_begin + tt * kTile + row;
      return (tt < n_sel_tiles && je < e_end) ? idx[je] : -1;
    }
    return (tt < n_tiles && row < n_win_rows) ? row : -1;
  };

  if (tid == 0) {
    for (int j = 0; j < kChunks; ++j) {
      mbar_init(&bars[B_VREADY + j], kGatherWarps + kSoftWarps);
      mbar_init(&bars[B_VFREE + j], 1);
    }
    mbar_init(&bars[B_SFULL], 1);
    mbar_init(&bars[B_SFREE], kSoftWarps);
    mbar_init(&bars[B_PREADY], kSoftWarps);
    mbar_init(&bars[B_PFREE], 1);
    mbar_init(&bars[B_QREADY], kSoftWarps);
    mbar_init(&bars[B_DONE], 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp >= kSoftWarps && warp < kMmaWarp) {
    // ------------------------------ gather + dequantize ------------------------------
    // Gather warp g loads and dequantizes tile rows 16 g + 8 i + lane / 4 (i = 0, 1); the
    // softmax warps take rows 64 .. 127.
    const int row0 = 16 * (warp - kSoftWarps);
    const int qd = lane >> 2;
    const uint8_t* packed_b = p.packed + int64_t(b) * p.cap * (kD / 2);
    const uint8_t* scales_b = p.scales + int64_t(b) * p.cap * (kD / kGroup);
    griddep_wait();  // the index list comes from the preceding kernel on the stream
    int32_t pos_next[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) pos_next[i] = tile_pos(0, row0 + 8 * i + qd);
    for (int t = 0; t < n_tiles && !*s_abort; ++t) {
      // Tile t's rows are loaded only once the softmax warps have written tile t - 1's
      // probabilities: TMEM and shared-memory accesses queue behind the global loads the
      // SM has in flight, so loads issued earlier would stall the softmax. They overlap
      // the P.V of tile t - 1 instead, which frees the buffers they are needed for.
      if (t > 0 && !gather_wait(&bars[B_PREADY], (t - 1) & 1)) {
        if (lane == 0) fail_wait(p, s_abort);
        break;
      }
      int32_t pos[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        pos[i] = (pos_next[i] >= 0 && pos_next[i] < len) ? pos_next[i] : -1;
        pos_next[i] = tile_pos(t + 1, row0 + 8 * i + qd);  // one tile ahead
      }
      const bool ld_ok = (kWin && t == n_sel_tiles) ? load_dequant_win<2>(smem, bars, win_b, pos, row0, t)
                                                    : load_dequant<2>(smem, bars, packed_b, scales_b, pos, row0, t);
      if (!ld_ok) {
        if (lane == 0) fail_wait(p, s_abort);
        break;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------ MMA issuer ------------------------------
    // The whole warp waits (every lane polls the mbarrier: one lane polling and then
    // broadcasting resumed the warp measurably later); lane 0 issues the MMAs and commits.
    {
      constexpr uint32_t kIdescQK = umma_idesc(0u, 128, kHeadsPerCta, 0u, 0u);
      constexpr uint32_t kIdescPV = umma_idesc(0u, 128, kHeadsPerCta, 1u, 1u);
      constexpr uint32_t kIdescPV2 = umma_idesc(0u, 128, 2 * kHeadsPerCta, 1u, 1u);
      // Descriptors are built once; each MMA adds its operand offset in 16-byte units to the
      // start-address field (shared-memory addresses stay below 2^18 bytes, so the 14-bit
      // field never carries). A single thread issues ~50 cycles apart at best for N = 64,
      // so the issue path is kept to constant adds.
      const uint64_t dq = sw128_kmajor_desc(smem_u32(smem + kOffQ));
      const uint64_t dvk = sw128_kmajor_desc(smem_u32(smem + kOffV));
      const uint64_t dvm = sw128_mnmajor_desc(smem_u32(smem + kOffV), kVChunkBytes);
      const uint64_t dph = sw128_mnmajor_desc(smem_u32(smem + kOffPh), kPBytes);
      const uint64_t dpl = sw128_mnmajor_desc(smem_u32(smem + kOffPl), kPBytes);
      const bool issuer = lane == 0;
      bool ok = __all_sync(0xffffffffu, mbar_wait_timed(&bars[B_QREADY], 0));
      if (!ok && issuer) fail_wait(p, s_abort);
      for (int t = 0; ok && t < n_tiles; ++t) {
        if (__shfl_sync(0xffffffffu, *s_abort, 0)) break;
        if (!__all_sync(0xffffffffu, mbar_wait_timed(&bars[B_SFREE], (t & 1) ^ 1))) {
          if (issuer) fail_wait(p, s_abort);
          break;
        }
        const uint32_t ds = tmem + kColS;
        // (loops kept rolled: their first pass runs from a cold instruction cache)
#pragma unroll 1
        for (int jc = 0; jc < kChunks && ok; ++jc) {
          if (!__all_sync(0xffffffffu, mbar_wait_timed(&bars[B_VREADY + jc], t & 1))) {
            ok = false;
            break;
          }
          if (issuer) {
            tc_fence_after();
            const uint64_t a = dvk + static_cast<uint64_t>((jc * kVChunkBytes) >> 4);
            const uint64_t bq = dq + static_cast<uint64_t>((jc * kQChunkBytes) >> 4);
            umma_f16(ds, a, bq, kIdescQK, jc != 0);  // K steps of 16 elements = 32 bytes
            umma_f16(ds, a + 2, bq + 2, kIdescQK, true);
            umma_f16(ds, a + 4, bq + 4, kIdescQK, true);
            umma_f16(ds, a + 6, bq + 6, kIdescQK, true);
          }
          __syncwarp();
        }
        if (!ok) {
          if (issuer) fail_wait(p, s_abort);
          break;
        }
        if (issuer) umma_commit(&bars[B_SFULL]);
        if (!__all_sync(0xffffffffu, mbar_wait_timed(&bars[B_PREADY], t & 1))) {
          if (issuer) fail_wait(p, s_abort);
          break;
        }
        if (issuer) {
          tc_fence_after();
          const bool acc0 = t > 0;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            const uint32_t d = tmem + o_col(c);
            if (c < kPairTiles) {
              // N = 128: P_hi's 64 heads, then P_lo's (the operand's second 64-element block
              // along N lies kPBytes further, where P_lo is)
#pragma unroll 2
              for (int s = 0; s < kTile / 16; ++s) {  // 16 entries = 2048 bytes of K per step
                const uint64_t a = dvm + static_cast<uint64_t>((2 * c * kVChunkBytes + 2048 * s) >> 4);
                const uint64_t ko = static_cast<uint64_t>((2048 * s) >> 4);
                umma_f16(d, a, dph + ko, kIdescPV2, acc0 || s > 0);
              }
            } else {
#pragma unroll 2
              for (int s = 0; s < kTile / 16; ++s) {
                const uint64_t a = dvm + static_cast<uint64_t>((2 * c * kVChunkBytes + 2048 * s) >> 4);
                const uint64_t ko = static_cast<uint64_t>((2048 * s) >> 4);
                umma_f16(d, a, dph + ko, kIdescPV, acc0 || s > 0);
                umma_f16(d, a, dpl + ko, kIdescPV, true);
              }
            }
            umma_commit(&bars[B_VFREE + 2 * c]);
            umma_commit(&bars[B_VFREE + 2 * c + 1]);
          }
          umma_commit(&bars[B_PFREE]);
        }
        __syncwarp();
      }
      // every MMA issued above completes before TMEM is released
      if (issuer) umma_commit(&bars[B_DONE]);
      if (!__all_sync(0xffffffffu, mbar_wait_timed(&bars[B_DONE], 0)) && issuer) fail_wait(p, s_abort);
    }
    __syncwarp();
  } else {
    // ---------------------- Q conversion, softmax and output (warps 0-7) ----------------------
    // Q: bf16 -> fp16 with a per-head power-of-two scale; K-major 128B-swizzled chunks. Each
    // warp converts heads warp, warp + 8, ...; its eight rows are loaded before any is
    // converted so that the global loads overlap.
    {
      uint4 qv[kHeadsPerCta / kSoftWarps][2];
#pragma unroll
      for (int r = 0; r < kHeadsPerCta / kSoftWarps; ++r) {
        const int hh = warp + kSoftWarps * r;
        qv[r][0] = qv[r][1] = make_uint4(0, 0, 0, 0);
        if (hh < nh) {
          const uint16_t* qr = p.q + (int64_t(b) * p.H + hbase + hh) * kD + 16 * lane;
          qv[r][0] = *reinterpret_cast<const uint4*>(qr);
          qv[r][1] = *reinterpret_cast<const uint4*>(qr + 8);
        }
      }
#pragma unroll
      for (int r = 0; r < kHeadsPerCta / kSoftWarps; ++r) {
        const int hh = warp + kSoftWarps * r;
        const uint32_t wd[8] = {qv[r][0].x, qv[r][0].y, qv[r][0].z, qv[r][0].w,
                                qv[r][1].x, qv[r][1].y, qv[r][1].z, qv[r][1].w};
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = max(m, max(wd[i] & 0x7fffu, (wd[i] >> 16) & 0x7fffu));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        int k = 0;
        if (m != 0) {
          const int ex = int((m >> 7) & 0xff) - 127;  // exponent of max|q|
          k = 14 - (ex < -126 ? -126 : ex);
          if (k > 127) k = 127;
          if (k < -126) k = -126;
        }
        const float up = __uint_as_float(uint32_t(127 + k) << 23);
        uint32_t h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          h[i] = pack_f16x2(bf16_bits_to_f32(wd[i] & 0xffffu) * up, bf16_bits_to_f32(wd[i] >> 16) * up);
        const float c = hh < nh ? p.sm_scale * kLog2e * __uint_as_float(uint32_t(127 - k / 2) << 23) *
                                      __uint_as_float(uint32_t(127 - (k - k / 2)) << 23)
                                : 0.0f;
        // dims [16 lane, 16 lane + 16): chunk lane / 4, 16-byte units 2 (lane % 4) and +1
        uint8_t* qrow = smem + kOffQ + (lane >> 2) * kQChunkBytes + hh * 128;
        const int u0 = 2 * (lane & 3);
        *reinterpret_cast<uint4*>(qrow + ((u0 ^ (hh & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(qrow + (((u0 + 1) ^ (hh & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
        if (lane == 0) {
          sC[hh] = c;
          sM[hh] = -INFINITY;
          sMT[hh] = -INFINITY;
          sM6[hh] = -INFINITY;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_QREADY]);
      softmax_sync();  // sC / sM of every head are visible to all softmax warps
    }

    const int q4 = warp & 3;          // TMEM lane quarter
    const int h0 = 32 * (warp >> 2);  // first of this thread's 32 heads
    const int e = 32 * q4 + lane;     // tile row (entry) / output dim within a dim tile
    const uint32_t lane_addr = uint32_t(32 * q4) << 16;
    griddep_wait();  // the index list comes from the preceding kernel on the stream
    // this warp also loads and dequantizes tile rows 64 + 8 warp + lane / 4 of every tile
    const int drow = 64 + 8 * warp;
    const uint8_t* packed_b = p.packed + int64_t(b) * p.cap * (kD / 2);
    const uint8_t* scales_b = p.scales + int64_t(b) * p.cap * (kD / kGroup);
    auto dq_pos = [&](int tt) -> int32_t { return tile_pos(tt, drow + (lane >> 2)); };
    int32_t dpos_next = dq_pos(0);
    // bit t: this thread's entry of tile t is valid (at most 32 tiles, 33 with the window)
    using VMask = typename std::conditional<kWin, uint64_t, uint32_t>::type;
    VMask vmask = 0;
    for (int t0 = 0; t0 < n_tiles; t0 += 8) {
      int32_t pv[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) pv[k] = tile_pos(t0 + k, e);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (pv[k] >= 0 && pv[k] < len) vmask |= VMask(1) << (t0 + k);
    }
    float lsum[32];  // per-head running row sums over this thread's entries
#pragma unroll
    for (int j = 0; j < 32; ++j) lsum[j] = 0.0f;
    bool fail = false;  // uniform across the softmax warps
    bool dq_fail = false;  // this warp's share of the dequantization timed out
    if (n_tiles > 0) {
      int32_t dp[1] = {(dpos_next >= 0 && dpos_next < len) ? dpos_next : -1};
      dpos_next = dq_pos(1);
      dq_fail = !((kWin && n_sel_tiles == 0) ? load_dequant_win<1>(smem, bars, win_b, dp, drow, 0)
                                              : load_dequant<1>(smem, bars, packed_b, scales_b, dp, drow, 0));
    }
    for (int t = 0; t < n_tiles; ++t) {
      const bool valid = (vmask >> t) & 1u;
      bool f = !softmax_wait(&bars[B_SFULL], t & 1);
      float z[32];
      bool over = false;
      if (!f) {
        tc_fence_after();
        uint32_t r[32];
        tmem_ld32(tmem + lane_addr + kColS + h0, r);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_SFREE]);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          z[j] = valid ? __uint_as_float(r[j]) * sC[h0 + j] : -INFINITY;
          over |= z[j] > sMT[h0 + j];
        }
        // the previous tile's P.V must be complete before P is rewritten or O rescaled
        // (it precedes this tile's S in the tensor pipe, so this wait is normally free)
        f = !softmax_wait(&bars[B_PFREE], (t & 1) ^ 1);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) z[j] = -INFINITY;
      }
      f = f || dq_fail;
      if (softmax_any(over || f)) {
        if (softmax_any(f)) {
          fail = true;
          break;
        }
        tc_fence_after();
        // move the reference of every head with a logit above m + 2^9
        const float tmax = butterfly32<true>(z);  // lane l: head h0 + l over this warp's rows
        sRed[q4 * 64 + h0 + lane] = tmax;
        softmax_sync();
        if (q4 == 0) {
          const int h = h0 + lane;
          const float tm = fmaxf(fmaxf(sRed[h], sRed[64 + h]), fmaxf(sRed[128 + h], sRed[192 + h]));
          const float mo = sM[h];
          float mn = mo, a = 1.0f;
          if (tm > mo + kMoveLog2) {
            mn = tm + kHeadroomLog2;
            a = mo == -INFINITY ? 0.0f : exp2f(mo - mn);
          }
          sM[h] = mn;
          sMT[h] = mn + kMoveLog2;
          sM6[h] = mn - 6.0f;  // (kPScale = 2^6)
          sA[h] = a;
        }
        softmax_sync();
        bool moved = false;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float a = sA[h0 + j];
          lsum[j] *= a;
          moved |= a != 1.0f;
        }
        if (t > 0 && moved) {  // rescale this thread's O^T elements of the moved heads
          // (16 columns at a time: dim tiles 0-2 hold two accumulators, dim tile 3 one)
#pragma unroll 1
          for (int c = 0; c < 2 * (2 * kPairTiles + 1); ++c) {
            uint32_t r[16];
            const int j0 = 16 * (c & 1), blk = c >> 1;
            const uint32_t col = blk < 2 * kPairTiles ? o_col(blk >> 1) + 64u * (blk & 1) : o_col(kPairTiles);
            const uint32_t addr = tmem + lane_addr + col + h0 + j0;
            tmem_ld16(addr, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * sA[h0 + j0 + j]);
            tmem_st16(addr, r);
          }
          tmem_st_wait();
        }
      }
      // probabilities (< 2^9), row sums, and this thread's half of the entry's row of P^T
      uint8_t* prow_h = smem + kOffPh + e * 128;
      uint8_t* prow_l = smem + kOffPl + e * 128;
#pragma unroll
      for (int unit = 0; unit < 4; ++unit) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int j = 8 * unit + 2 * k;
          // p * 2^6 straight from the exponent; the row sums add the same scaled values and
          // are scaled back by the exact 2^-6 at the end
          const float m0 = sM6[h0 + j], m1 = sM6[h0 + j + 1];
          const float a = m0 == -INFINITY ? 0.0f : ex2_approx(z[j] - m0);
          const float c2 = m1 == -INFINITY ? 0.0f : ex2_approx(z[j + 1] - m1);
          lsum[j] += a;
          lsum[j + 1] += c2;
          hi[k] = pack_f16x2(a, c2);
          lo[k] = pack_f16x2(a - f16_lo_to_f32(hi[k]), c2 - f16_hi_to_f32(hi[k]));
        }
        const uint32_t off = uint32_t((((h0 >> 3) + unit) ^ (e & 7)) << 4);
        *reinterpret_cast<uint4*>(prow_h + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(prow_l + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PREADY]);
      if (t + 1 < n_tiles) {  // this warp's rows of the next tile, as P.V(t) frees V_hat
        int32_t dp[1] = {(dpos_next >= 0 && dpos_next < len) ? dpos_next : -1};
        dpos_next = dq_pos(t + 2);
        dq_fail = !((kWin && t + 1 == n_sel_tiles) ? load_dequant_win<1>(smem, bars, win_b, dp, drow, t + 1)
                                                   : load_dequant<1>(smem, bars, packed_b, scales_b, dp, drow, t + 1));
      }
    }
    // ---- the partial O^T leaves for the workspace one dim tile at a time, as soon as the
    // last tile's P.V has finished that dim tile (fp32, unscaled, [64 heads][512 dims]) ----
    {
      const int64_t part0 = (int64_t(b) * gridDim.y + hg) * cluster_nctas();
      float* po = p.part_o + (part0 + cluster_ctarank()) * (kHeadsPerCta * kD);
      bool f_part = false;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        bool have = !fail && !f_part && n_tiles > 0;
        if (have && !softmax_wait(&bars[B_VFREE + 2 * c], (n_tiles - 1) & 1)) {
          f_part = true;  // (this CTA's partial is dropped below)
          have = false;
        }
        if (have) {
          tc_fence_after();
          tmem_ld32(tmem + lane_addr + o_col(c) + h0, r);
          if (c < kPairTiles) {  // the P_lo accumulator of this dim tile
            uint32_t r2[32];
            tmem_ld32(tmem + lane_addr + o_col(c) + 64u + h0, r2);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) + __uint_as_float(r2[k]));
          } else {
            tmem_ld_wait();
          }
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = 0u;
        }
#pragma unroll
        for (int k = 0; k < 32; ++k) __stcg(po + (h0 + k) * kD + 128 * c + e, __uint_as_float(r[k]));
      }
      // ---- wait for the last P.V and reduce the row sums over the CTA ----
      if (!fail && n_tiles > 0) {
        const bool f = f_part || !softmax_wait(&bars[B_PFREE], (n_tiles - 1) & 1);
        fail = softmax_any(f);
      }
    }
    if (fail) {
      if (tid == 0) fail_wait(p, s_abort);
      if (q4 == 0) sL[h0 + lane] = 0.0f;  // this CTA's partial is dropped
    } else {
      tc_fence_after();
      const float lw = butterfly32<false>(lsum);  // lane l: head h0 + l over this warp's rows
      sRed[q4 * 64 + h0 + lane] = lw;
      softmax_sync();
      if (q4 == 0) {
        const int h = h0 + lane;
        sL[h] = (sRed[h] + sRed[64 + h] + sRed[128 + h] + sRed[192 + h]) * (1.0f / kPScale);
      }
    }
    if (tid == 0) *s_fail = fail ? 1u : 0u;
  }

  // ---- combine the chunk CTAs of this (sequence, head group): one cluster ----
  // Each CTA has written its partial O^T to the workspace (it stays in L2); now (m, l) per
  // head (l = 0: the partial is void). One cluster barrier makes every chunk's partial
  // visible to the others; then CTA `rank` sums dims [rank * 512 / C, +512 / C) of every
  // head over the chunks with the log-sum-exp weights 2^(m_c - M) / (2^6 L) (O holds
  // p * 2^6) and writes them.
  __syncthreads();
  const uint32_t C = cluster_nctas(), rank = cluster_ctarank();
  const int64_t part0 = (int64_t(b) * gridDim.y + hg) * C;  // this (sequence, head group)'s first chunk
  {
    if (tid < kHeadsPerCta) {
      const float l = sL[tid];
      float* pml = p.part_ml + ((part0 + rank) * kHeadsPerCta + tid) * 2;
      __stcg(pml, l > 0.0f ? sM[tid] : -INFINITY);
      __stcg(pml + 1, l);
    }
  }
  cluster_sync_all();  // every chunk CTA's partial is in the workspace and visible
  switch (C) {  // (only the instance that runs is ever fetched)
    case 1: combine_slice<1>(p, b, hbase, nh, rank, part0); break;
    case 2: combine_slice<2>(p, b, hbase, nh, rank, part0); break;
    case 4: combine_slice<4>(p, b, hbase, nh, rank, part0); break;
    case 8: combine_slice<8>(p, b, hbase, nh, rank, part0); break;
    default: combine_slice<16>(p, b, hbase, nh, rank, part0); break;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// Chunks of the index list per (sequence, head group), one CTA each, forming one cluster: a
// power of two up to 16 (at most one chunk per 128-entry tile), the grid within about one
// CTA per SM.
int attn_chunks(int B, int H, int top_k, int num_sms) {
  const int n_hg = (H + kHeadsPerCta - 1) / kHeadsPerCta;
  const int tiles = (top_k + kTile - 1) / kTile;
  int c = 1;
  while (c < kMaxCluster && 2 * c <= tiles && int64_t(B) * n_hg * 2 * c <= num_sms) c *= 2;
  return c;
}

namespace {
// per device and cluster size 2^i: how many clusters of the attention can be resident at
// once (0: not asked yet, -1: none)
int g_attn_max_clusters[64][5] = {};

int max_active_clusters(int chunks) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  int li = 0;
  while ((1 << li) < chunks) ++li;
  int& known = g_attn_max_clusters[dev & 63][li];
  if (known == 0) {
    known = -1;
    for (auto kf : {k_sparse_attn_tc<false>, k_sparse_attn_tc<true>}) {
      if (chunks > 8 && cudaFuncSetAttribute(kf, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return known;
      if (cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemAttn)) !=
          cudaSuccess)
        return known;
    }
    cudaLaunchConfig_t q = {};
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = static_cast<unsigned>(chunks);
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.gridDim = dim3(chunks, 1, 1);
    q.blockDim = dim3(kAttnThreads);
    q.dynamicSmemBytes = kSmemAttn;
    q.attrs = qa;
    q.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_sparse_attn_tc<false>, &q) == cudaSuccess && n > 0) known = n;
    (void)cudaGetLastError();
  }
  return known;
}
}  // namespace

cudaError_t launch_sparse_attn(const AttnParams& p, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  if (p.B == 0) return cudaSuccess;
  const int n_hg = (p.H + kHeadsPerCta - 1) / kHeadsPerCta;
  auto kern = p.swa != nullptr ? k_sparse_attn_tc<true> : k_sparse_attn_tc<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemAttn));
  if (e != cudaSuccess) return e;
  int chunks = p.n_chunks;
  if (chunks < 1 || chunks > kMaxCluster || (chunks & (chunks - 1)) != 0) return cudaErrorInvalidValue;
  // fewer chunks per cluster until every (sequence, head group) cluster can be resident at
  // once (a cluster needs all its CTAs, one per SM here, inside one GPC)
  const int64_t want = int64_t(p.B) * n_hg;
  while (chunks > 1) {
    const int n = max_active_clusters(chunks);
    if (n >= want || (n > 0 && chunks <= 4)) break;
    chunks >>= 1;
  }
  AttnParams pc = p;
  pc.n_chunks = chunks;
  // A programmatic dependent of the kernel before it on the stream: its CTAs may be scheduled
  // while that kernel finishes (an SM it has left idle can run the prologue: barriers, TMEM,
  // Q conversion) and wait in griddep_wait() before reading what it produced.
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(chunks);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(chunks, n_hg, p.B);
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = kSmemAttn;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, pc);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4kv
