// Indexer scoring: score[n] = ks[n] * sum_h w[h] * max(0, q[h] . k[n]) for every visible
// entry (Full mode) or for the positions of a candidate pool (Reindex mode).
//
// Method: [PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로 줄이고 …",
//  - section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2": an indexer with 32 query heads of
//    dimension 128 scores the causally visible entries (Full and Reindex rows of the mode
//    table);
//  - section "계층적 희소 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기": the first Full
//    layer also gives every block of 8 positions its largest score (block max), and Reindex
//    layers score only inside the candidate pool.
// The head-combining rule (weighted sum of ReLU dot products) is this library's reading.
//
// Key formats: bf16, FP8 E4M3, or FP4 (E2M1 codes with one E4M3 scale per 16 channels, the
// format the pages give the indexer query and key, here with the main KV's quantizer).
//
// Kernel (persistent, two CTAs per SM for 8- and 4-bit keys, warp-specialised, 6 warps):
//  * warp 0 (one lane): TMA producer. Streams 128-row key tiles (8 KiB of E2M1 + 1 KiB of
//    scales, 16 KiB of E4M3 or 32 KiB of bf16; 64- / 128-byte swizzled) into a shared-memory
//    ring as deep as shared memory allows, and each sequence's query block into one of two
//    query slots. Full mode: one box per tile; Reindex mode: one 8-row box per pool block.
//  * warp 1: allocates TMEM; one lane issues tcgen05.mma (M = 128 entries, N = padded head
//    count, K = 128 dims; kind::mxf4nvf4 with block scales on E2M1, kind::f8f6f4 on E4M3,
//    kind::f16 on bf16) into a ring of fp32 accumulators in TMEM, and commits to the ring's
//    mbarriers. For E2M1 the whole warp first regroups the tile's scale bytes into the
//    32-row x 16-byte blocks that tcgen05.cp replicates into TMEM (row m's four scales of
//    one K step in column m / 32 of lane m % 32), then the lane copies them and issues.
//  * warps 2-5: the epilogue warpgroup. Each thread owns one row
//    (TMEM lane): loads its N head dot products, combines heads, writes the fp32 score, and
//    adds the score's top 12 key bits to its warpgroup's shared-memory histogram, flushed per
//    sequence (first pass of the exact top-K). With a block-max output it reduces each block
//    of 8 rows across 8 lanes and histograms those.
// Every wait is bounded in time; on timeout the kernel sets a status bit and winds down.
#include <cstdio>

#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"
#include "fp4kv_sm100.cuh"

namespace fp4kv {
namespace {

constexpr int kTileRows = 128;
constexpr int kPoolBlock = 8;
constexpr int kEpiGroups = 1;   // epilogue warpgroups (alternating tiles when > 1)
constexpr int kEpiThreads = 128;
constexpr int kThreads = 64 + kEpiGroups * kEpiThreads;  // producer, mma, epilogue groups
constexpr int kAccCols = 256;  // TMEM columns allocated per CTA (ring of accumulators)
constexpr size_t kSmemPerSm = 227 * 1024;

// key / query element types
constexpr int kKeyBf16 = 0, kKeyE4M3 = 1, kKeyE2M1 = 2;

// Two CTAs per SM for 8- and 4-bit keys: each CTA's single MMA-issuing thread serialises
// its wait -> issue -> commit chain per tile, and two independent chains per SM keep the
// stream near the HBM rate where one deep ring could not. The bf16 (small) case keeps one
// CTA per SM so that its 32 KiB stages fit.
template <int KT, int N>
struct ScanCfg {
  static constexpr bool kFp4 = KT == kKeyE2M1;
  static constexpr int kCtasPerSm = KT == kKeyBf16 ? 1 : 2;
  static constexpr size_t kSmemBudget = kSmemPerSm / kCtasPerSm - 1024;
  static constexpr int kRowBytes = KT == kKeyBf16 ? 256 : (KT == kKeyE4M3 ? 128 : 64);
  static constexpr int kKeyBytes = kTileRows * kRowBytes;  // one stage of keys
  // E2M1: each stage also holds the tile's scale bytes as loaded (8 bytes per row; the rows
  // of an 8-row block contiguous, blocks kSfBlkStride apart: 64 B in Full mode, where one
  // box brings the tile's 1 KiB, 128 B in Reindex mode, where each block is its own box and
  // must start 128-byte aligned) and regrouped for tcgen05.cp (two 32 x 16-byte blocks, one
  // per K step of 64)
  static constexpr int kSfTileBytes = kTileRows * 8;
  static constexpr int kSfRaw = kFp4 ? 2 * kSfTileBytes : 0;
  static constexpr int kSfBlk = kFp4 ? 1024 : 0;
  static constexpr int kStageBytes = kKeyBytes + kSfRaw + kSfBlk;
  // one query block (per sequence): codes, then (E2M1) up to 64 x 8 scale bytes as loaded
  // and their two regrouped 512-byte blocks
  static constexpr int kQCodeBytes = N * kRowBytes;
  static constexpr int kQBytes = kQCodeBytes + (kFp4 ? 512 + 1024 : 0);
  static constexpr size_t kHistBytes = size_t(2 * kEpiGroups) * kHistBins * sizeof(uint32_t);
  static constexpr size_t kFixed = 1024 + 2 * size_t(kQBytes) + kHistBytes + 1024;
  static constexpr int kStagesFit = static_cast<int>((kSmemBudget - kFixed) / kStageBytes);
  static constexpr int kStages = kStagesFit > 16 ? 16 : kStagesFit;
  // E2M1: accumulators in TMEM columns [0, 128), scale factors of A (one 8-column slot per
  // accumulator slot) from column 128, of B (one per query slot) from column 192
  static constexpr int kAccSlots = (kFp4 ? 128 : kAccCols) / N;
  static constexpr uint32_t kSfaCol = 128, kSfbCol = 192;
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + 2 * size_t(kQBytes) +
                                  (2 * kStages + 2 * kAccSlots + 4) * sizeof(uint64_t) + kHistBytes + 64;
  static_assert(kStages >= 2, "shared memory budget");
  static_assert(kSmem <= kSmemBudget, "shared memory budget");
  static_assert(kStageBytes % 1024 == 0 && kQBytes % 512 == 0, "swizzle atom alignment");
  static_assert(!kFp4 || kSfaCol + 8 * kAccSlots <= kSfbCol, "TMEM columns");
  static constexpr uint32_t kIdesc = kFp4 ? umma_idesc_nvf4(128, N) : umma_idesc(KT == kKeyE4M3 ? 0u : 1u, 128, N);
};

// E2M1 scale bytes of 32 * 4 rows (8 per row, group order; row r at
// raw + (r / 8) * blk_stride + (r % 8) * 8) regrouped for tcgen05.cp: block k (K step k =
// channels [64k, 64k + 64)) holds, on its 16-byte line l, the four scales of rows l,
// l + 32, l + 64, l + 96 in that order. Rows at or past `rows` get scale 0.
// Warp-collective (lane = line); ends with the async-proxy fence tcgen05.cp needs.
FP4KV_DEV void regroup_scales(const uint8_t* raw, int blk_stride, uint8_t* blocks, int rows, int lane) {
  uint32_t lo[4], hi[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int r = lane + 32 * g;
    uint2 v = make_uint2(0u, 0u);
    if (r < rows) v = *reinterpret_cast<const uint2*>(raw + (r >> 3) * blk_stride + (r & 7) * 8);
    lo[g] = v.x;
    hi[g] = v.y;
  }
  *reinterpret_cast<uint4*>(blocks + 16 * lane) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  *reinterpret_cast<uint4*>(blocks + 512 + 16 * lane) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  fence_proxy_async_smem();
  __syncwarp();
}

// named barrier of one epilogue warpgroup (ids 1 and 2)
FP4KV_DEV void epi_sync(int group) { asm volatile("bar.sync %0, %1;" ::"r"(1 + group), "n"(kEpiThreads)); }

struct Tiles {
  int64_t begin, end, per_seq;
};

// Iterates this CTA's tiles without 64-bit divisions: (b, tis) advance together.
struct TileIter {
  int b;
  int64_t tis, t, end, per_seq;
  FP4KV_DEV void init(const Tiles& T) {
    t = T.begin;
    end = T.end;
    per_seq = T.per_seq;
    b = static_cast<int>(T.begin / T.per_seq);
    tis = T.begin - int64_t(b) * T.per_seq;
  }
  FP4KV_DEV bool done() const { return t >= end; }
  FP4KV_DEV void next() {
    ++t;
    if (++tis == per_seq) {
      tis = 0;
      ++b;
    }
  }
};

FP4KV_DEV int64_t seq_len_of(const IndexScoreParams& p, int b) {
  int64_t len = p.seq_lens[b];
  if (len > p.cap) len = p.cap;
  return len;
}

template <int KT, int N>
__global__ void __launch_bounds__(kThreads, ScanCfg<KT, N>::kCtasPerSm)
    k_index_score_tc(const IndexScoreParams p, const __grid_constant__ CUtensorMap tm_keys,
                     const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ksf,
                     int64_t tiles_per_seq, int64_t total_tiles) {
  using Cfg = ScanCfg<KT, N>;
  constexpr bool FP8 = KT == kKeyE4M3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* qbuf = ring + size_t(Cfg::kStages) * Cfg::kStageBytes;  // 2 query slots
  uint64_t* full = reinterpret_cast<uint64_t*>(qbuf + 2 * size_t(Cfg::kQBytes));
  uint64_t* empty = full + Cfg::kStages;
  uint64_t* tfull = empty + Cfg::kStages;
  uint64_t* tempty = tfull + Cfg::kAccSlots;
  uint64_t* qfull = tempty + Cfg::kAccSlots;  // [2]
  uint64_t* qempty = qfull + 2;               // [2]
  uint32_t* s_hist_all = reinterpret_cast<uint32_t*>(qempty + 2);  // [group][2][bins]
  uint32_t* s_tmem = s_hist_all + 2 * kEpiGroups * kHistBins;
  volatile uint32_t* s_abort = s_tmem + 1;

  // the top-K select that follows may be scheduled as CTAs of this grid finish
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Tiles T;
  T.per_seq = tiles_per_seq;
  T.begin = total_tiles * blockIdx.x / gridDim.x;
  T.end = total_tiles * (blockIdx.x + 1) / gridDim.x;
  const bool pool_mode = p.pool != nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < Cfg::kAccSlots; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per warp of the tile's epilogue warpgroup
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&qfull[j], 1);
      mbar_init(&qempty[j], 1);
    }
    *s_abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_keys);
    prefetch_tmap(&tm_q);
    if constexpr (Cfg::kFp4) prefetch_tmap(&tm_ksf);
  }
  for (int i = threadIdx.x; i < 2 * kEpiGroups * kHistBins; i += blockDim.x) s_hist_all[i] = 0;
  if (warp == 1) {
    tmem_alloc(s_tmem, kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  // launched as a programmatic dependent: the prologue above overlapped the previous kernel
  // on the stream; everything it wrote is visible past this point
  griddep_wait();

  if (warp == 0) {
    // ------------------------------- TMA producer ----------------------------------
    if (lane == 0) {
      const uint64_t stream_pol = l2_evict_first();
      uint32_t it = 0, nq = 0;  // tiles issued, query blocks issued
      int cur_b = -1, q_b = -1;
      int64_t len = 0;
      TileIter ti;
      for (ti.init(T); !ti.done(); ti.next()) {
        if (ti.b != cur_b) {
          cur_b = ti.b;
          len = seq_len_of(p, cur_b);
        }
        const int64_t unit = pool_mode ? ti.tis * (kTileRows / kPoolBlock) : ti.tis * kTileRows;
        if (!pool_mode && unit >= len) continue;
        if (ti.b != q_b) {
          // first active tile of a sequence: its query block into the next slot, once the
          // MMA issuer has released that slot's previous query block
          const int slot = nq & 1;
          if (!mbar_wait_timed(&qempty[slot], ((nq >> 1) & 1) ^ 1)) {
            atomicOr(p.status, kFlagWaitTimeout);
            *s_abort = 1;
            break;
          }
          uint8_t* qdst = qbuf + size_t(slot) * Cfg::kQBytes;
          const int32_t qy = ti.b * p.H_I;
          if constexpr (Cfg::kFp4) {
            // codes through the map; the scale bytes (H_I * 8, a multiple of 16) as one copy
            mbar_arrive_expect_tx(&qfull[slot], Cfg::kQCodeBytes + 8 * p.H_I);
            tma_load_2d(qdst, &tm_q, 0, qy, &qfull[slot]);
            bulk_g2s(qdst + Cfg::kQCodeBytes, p.q_sf + int64_t(qy) * 8, 8 * p.H_I, &qfull[slot]);
          } else if constexpr (FP8) {
            mbar_arrive_expect_tx(&qfull[slot], Cfg::kQBytes);
            tma_load_2d(qdst, &tm_q, 0, qy, &qfull[slot]);
          } else {
            mbar_arrive_expect_tx(&qfull[slot], Cfg::kQBytes);
            tma_load_2d(qdst, &tm_q, 0, qy, &qfull[slot]);
            tma_load_2d(qdst + Cfg::kQBytes / 2, &tm_q, 64, qy, &qfull[slot]);
          }
          q_b = ti.b;
          ++nq;
        }
        const int stage = it % Cfg::kStages;
        const uint32_t ph = (it / Cfg::kStages) & 1;
        ++it;
        if (!mbar_wait_timed(&empty[stage], ph ^ 1)) {
          atomicOr(p.status, kFlagWaitTimeout);
          *s_abort = 1;
          break;
        }
        uint8_t* dst = ring + size_t(stage) * Cfg::kStageBytes;
        const int32_t row_base = static_cast<int32_t>(int64_t(ti.b) * p.cap);
        if (!pool_mode) {
          // a Full scan reads every key once: evict-first keeps the scores it writes (which
          // the select reads next) in L2 while the keys stream through
          mbar_arrive_expect_tx(&full[stage], Cfg::kKeyBytes + (Cfg::kFp4 ? Cfg::kSfTileBytes : 0));
          const int32_t y = row_base + static_cast<int32_t>(unit);
          if constexpr (Cfg::kFp4) {
            // scale plane viewed as [rows / 2][16 bytes]: y is even (cap even, unit % 128 == 0)
            tma_load_2d_hint(dst, &tm_keys, 0, y, &full[stage], stream_pol);
            tma_load_2d_hint(dst + Cfg::kKeyBytes, &tm_ksf, 0, y >> 1, &full[stage], stream_pol);
          } else if constexpr (FP8) {
            tma_load_2d_hint(dst, &tm_keys, 0, y, &full[stage], stream_pol);
          } else {
            tma_load_2d_hint(dst, &tm_keys, 0, y, &full[stage], stream_pol);
            tma_load_2d_hint(dst + Cfg::kKeyBytes / 2, &tm_keys, 64, y, &full[stage], stream_pol);
          }
        } else {
          const int32_t* pl = p.pool + int64_t(ti.b) * p.npb;
          int32_t blk[kTileRows / kPoolBlock];
          uint32_t bytes = 0;
          for (int s2 = 0; s2 < kTileRows / kPoolBlock; ++s2) {
            const int64_t slot = unit + s2;
            int32_t j = slot < p.npb ? pl[slot] : -1;
            if (j < 0 || int64_t(j) * kPoolBlock >= p.cap) j = -1;
            blk[s2] = j;
            if (j >= 0) bytes += kPoolBlock * (Cfg::kRowBytes + (Cfg::kFp4 ? 8 : 0));
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          for (int s2 = 0; s2 < kTileRows / kPoolBlock; ++s2) {
            if (blk[s2] < 0) continue;
            const int32_t y = row_base + blk[s2] * kPoolBlock;
            if constexpr (Cfg::kFp4) {
              // one 8-row swizzle atom of codes (512 B) and its 64 scale bytes
              tma_load_2d(dst + s2 * 512, &tm_keys, 0, y, &full[stage]);
              tma_load_2d(dst + Cfg::kKeyBytes + s2 * 128, &tm_ksf, 0, y >> 1, &full[stage]);
            } else if constexpr (FP8) {
              tma_load_2d(dst + s2 * 1024, &tm_keys, 0, y, &full[stage]);
            } else {
              tma_load_2d(dst + s2 * 1024, &tm_keys, 0, y, &full[stage]);
              tma_load_2d(dst + Cfg::kKeyBytes / 2 + s2 * 1024, &tm_keys, 64, y, &full[stage]);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
   if constexpr (Cfg::kFp4) {
    // ------------------- MMA issuer, E2M1 (whole warp: scale regrouping) -------------
    uint32_t it = 0, nseg = 0;
    int cur_b = -1, qslot = 0;
    int64_t len = 0;
    bool have_q = false;
    TileIter ti;
    for (ti.init(T); !ti.done(); ti.next()) {
      if (ti.b != cur_b) {
        cur_b = ti.b;
        len = seq_len_of(p, cur_b);
        if (have_q && lane == 0) umma_commit(&qempty[qslot]);  // previous query block free
        have_q = false;
      }
      if (!pool_mode && ti.tis * kTileRows >= len) continue;
      if (__shfl_sync(0xffffffffu, *s_abort, 0)) break;
      if (!have_q) {
        qslot = nseg & 1;
        if (!__all_sync(0xffffffffu, mbar_wait_timed(&qfull[qslot], (nseg >> 1) & 1))) {
          if (lane == 0) {
            atomicOr(p.status, kFlagWaitTimeout);
            *s_abort = 1;
          }
          break;
        }
        ++nseg;
        have_q = true;
        uint8_t* qs = qbuf + size_t(qslot) * Cfg::kQBytes + Cfg::kQCodeBytes;
        regroup_scales(qs, 64, qs + 512, p.H_I, lane);
        if (lane == 0) {
          tc_fence_after();
          const uint32_t sfb = tmem_base + Cfg::kSfbCol + 8u * uint32_t(qslot);
          tmem_cp_32x128_x4(sfb, rows16_desc(smem_u32(qs + 512)));
          tmem_cp_32x128_x4(sfb + 4, rows16_desc(smem_u32(qs + 1024)));
        }
      }
      const int stage = it % Cfg::kStages;
      const uint32_t ph = (it / Cfg::kStages) & 1;
      const int acc = it % Cfg::kAccSlots;
      const uint32_t aph = (it / Cfg::kAccSlots) & 1;
      ++it;
      if (!__all_sync(0xffffffffu, mbar_wait_timed(&tempty[acc], aph ^ 1) && mbar_wait_timed(&full[stage], ph))) {
        if (lane == 0) {
          atomicOr(p.status, kFlagWaitTimeout);
          *s_abort = 1;
        }
        break;
      }
      uint8_t* st = ring + size_t(stage) * Cfg::kStageBytes;
      regroup_scales(st + Cfg::kKeyBytes, pool_mode ? 128 : 64, st + Cfg::kKeyBytes + Cfg::kSfRaw, kTileRows,
                     lane);
      if (lane == 0) {
        tc_fence_after();
        const uint32_t sfa = tmem_base + Cfg::kSfaCol + 8u * uint32_t(acc);
        const uint32_t sfb = tmem_base + Cfg::kSfbCol + 8u * uint32_t(qslot);
        const uint32_t blk = smem_u32(st + Cfg::kKeyBytes + Cfg::kSfRaw);
        tmem_cp_32x128_x4(sfa, rows16_desc(blk));
        tmem_cp_32x128_x4(sfa + 4, rows16_desc(blk + 512));
        const uint32_t a0 = smem_u32(st);
        const uint32_t b0 = smem_u32(qbuf + size_t(qslot) * Cfg::kQBytes);
        const uint32_t d = tmem_base + uint32_t(acc * N);
        // two K steps of 64 E2M1 values (32 bytes) within each 64-byte swizzled row
        umma_nvf4(d, sw64_kmajor_desc(a0), sw64_kmajor_desc(b0), Cfg::kIdesc, sfa, sfb, false);
        umma_nvf4(d, sw64_kmajor_desc(a0 + 32), sw64_kmajor_desc(b0 + 32), Cfg::kIdesc, sfa + 4, sfb + 4, true);
        umma_commit(&empty[stage]);
        umma_commit(&tfull[acc]);
      }
      __syncwarp();
    }
    if (have_q && lane == 0) umma_commit(&qempty[qslot]);
   } else {
    // ------------------------------- MMA issuer ------------------------------------
    if (lane == 0) {
      uint32_t it = 0, nseg = 0;
      int cur_b = -1, qslot = 0;
      int64_t len = 0;
      bool have_q = false;
      TileIter ti;
      for (ti.init(T); !ti.done(); ti.next()) {
        if (ti.b != cur_b) {
          cur_b = ti.b;
          len = seq_len_of(p, cur_b);
          if (have_q) umma_commit(&qempty[qslot]);  // previous sequence's query block free
          have_q = false;
        }
        if (!pool_mode && ti.tis * kTileRows >= len) continue;
        if (*s_abort) break;
        if (!have_q) {
          qslot = nseg & 1;
          if (!mbar_wait_timed(&qfull[qslot], (nseg >> 1) & 1)) {
            atomicOr(p.status, kFlagWaitTimeout);
            *s_abort = 1;
            break;
          }
          ++nseg;
          have_q = true;
        }
        const int stage = it % Cfg::kStages;
        const uint32_t ph = (it / Cfg::kStages) & 1;
        const int acc = it % Cfg::kAccSlots;
        const uint32_t aph = (it / Cfg::kAccSlots) & 1;
        ++it;
        if (!mbar_wait_timed(&tempty[acc], aph ^ 1) || !mbar_wait_timed(&full[stage], ph)) {
          atomicOr(p.status, kFlagWaitTimeout);
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(ring + size_t(stage) * Cfg::kStageBytes);
        const uint32_t b0 = smem_u32(qbuf + size_t(qslot) * Cfg::kQBytes);
        const uint32_t d = tmem_base + uint32_t(acc * N);
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // 4 x 32 bytes of K per 128-byte swizzle row
          if constexpr (FP8) {
            umma_f8f6f4(d, sw128_kmajor_desc(a0 + 32 * k), sw128_kmajor_desc(b0 + 32 * k), Cfg::kIdesc, k > 0);
          } else {
            umma_f16(d, sw128_kmajor_desc(a0 + 32 * k), sw128_kmajor_desc(b0 + 32 * k), Cfg::kIdesc, k > 0);
          }
        }
        if constexpr (!FP8) {  // second 64-dim half of the bf16 rows
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_f16(d, sw128_kmajor_desc(a0 + Cfg::kKeyBytes / 2 + 32 * k),
                     sw128_kmajor_desc(b0 + Cfg::kQBytes / 2 + 32 * k), Cfg::kIdesc, true);
        }
        umma_commit(&empty[stage]);
        umma_commit(&tfull[acc]);
      }
      if (have_q) umma_commit(&qempty[qslot]);
    }
   }
  } else {
    // ------------------------------- epilogue (2 warpgroups) -----------------------
    const int group = (warp - 2) >> 2;          // warpgroup: tiles it % kEpiGroups == group
    const int gtid = threadIdx.x - 64 - group * kEpiThreads;
    const int quarter = warp & 3;               // TMEM lanes [32*quarter, +32)
    const int row = 32 * quarter + lane;        // tile row owned by this thread
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    uint32_t* s_hist = s_hist_all + 2 * group * kHistBins;
    uint32_t* s_bhist = s_hist + kHistBins;
    float wv[N];
    int cur_b = -1;
    uint32_t it = 0;
    TileIter ti;
    // adds this CTA's histogram(s) of sequence b to the global ones and clears them: four
    // bins per 16-byte access, atomics only for non-zero bins (the scores of a sequence
    // fall into few bins)
    auto flush_one = [&](uint32_t* sh, uint32_t* gh) {
      for (int i4 = gtid; i4 < kHistBins / 4; i4 += kEpiThreads) {
        uint4* q4 = reinterpret_cast<uint4*>(sh) + i4;
        const uint4 c = *q4;
        if ((c.x | c.y | c.z | c.w) == 0u) continue;
        uint32_t* g = gh + 4 * i4;
        if (c.x) atomicAdd(g, c.x);
        if (c.y) atomicAdd(g + 1, c.y);
        if (c.z) atomicAdd(g + 2, c.z);
        if (c.w) atomicAdd(g + 3, c.w);
        *q4 = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto flush = [&](int b) {
      epi_sync(group);
      flush_one(s_hist, p.hist + int64_t(b) * kHistBins);
      if (p.bmax != nullptr) flush_one(s_bhist, p.bmax_hist + int64_t(b) * kHistBins);
      epi_sync(group);
    };
    int len_b = -1;
    int64_t len = 0;
    for (ti.init(T); !ti.done(); ti.next()) {
      if (ti.b != len_b) {
        len_b = ti.b;
        len = seq_len_of(p, len_b);
      }
      if (!pool_mode && ti.tis * kTileRows >= len) continue;
      const uint32_t my = it++;
      if ((my % kEpiGroups) != static_cast<uint32_t>(group)) continue;
      const int acc = my % Cfg::kAccSlots;
      const uint32_t aph = (my / Cfg::kAccSlots) & 1;
      if (ti.b != cur_b) {
        if (cur_b >= 0 && p.hist != nullptr) flush(cur_b);
        cur_b = ti.b;
#pragma unroll
        for (int h = 0; h < N; ++h) wv[h] = h < p.H_I ? p.w[int64_t(cur_b) * p.H_I + h] : 0.0f;
      }
      // Once a wait has given up (here or in another role) the warp stops waiting and working
      // but keeps walking the same tiles, so every warp of the warpgroup reaches the same
      // histogram flushes (named barriers) and none is left waiting at one alone.
      bool live = __shfl_sync(0xffffffffu, *s_abort, 0) == 0u;
      if (live) {
        // (every lane polls: a wait polled by lane 0 alone and then broadcast resumed the warp
        // measurably later, and the epilogue's wait is on the scan's per-tile path)
        live = __all_sync(0xffffffffu, mbar_wait_timed(&tfull[acc], aph));
        if (!live && lane == 0) {
          atomicOr(p.status, kFlagWaitTimeout);
          *s_abort = 1;
        }
      }
      if (!live) continue;
      tc_fence_after();
      uint32_t r[N];
#pragma unroll
      for (int c0 = 0; c0 < N; c0 += 16)
        tmem_ld16(tmem_base + lane_addr + uint32_t(acc * N + c0),
                  *reinterpret_cast<uint32_t(*)[16]>(&r[c0]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      // four independent FMA chains, combined in a fixed order
      float part[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int h = 0; h < N; ++h) part[h & 3] += wv[h] * fmaxf(__uint_as_float(r[h]), 0.0f);
      float s = (part[0] + part[1]) + (part[2] + part[3]);

      const int64_t seq_base = int64_t(ti.b) * p.cap;
      float* srow = p.scores + int64_t(ti.b) * p.score_stride;
      // the largest key of the warp's 32 consecutive values (value index tile * 128 + row
      // in both modes); 0 when none of them is valid
      uint32_t* gmax_row = p.gmax != nullptr ? p.gmax + int64_t(ti.b) * p.gmax_stride + ti.tis * (kTileRows / 32) + quarter
                                             : nullptr;
      if (!pool_mode) {
        const int64_t pos = ti.tis * kTileRows + row;
        const bool valid = pos < len;
        if (valid) {
          if (p.key_scale != nullptr) s *= p.key_scale[seq_base + pos];
          srow[pos] = s;
          if (p.hist != nullptr) atomicAdd(&s_hist[order_key(s) >> (32 - kHistBits)], 1u);
        }
        if (gmax_row != nullptr) {
          const uint32_t km = __reduce_max_sync(0xffffffffu, valid ? order_key(s) : 0u);
          if (lane == 0) *gmax_row = km;
        }
        if (p.bmax != nullptr) {
          float m = valid ? s : -INFINITY;
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
          if ((lane & 7) == 0 && m > -INFINITY) {
            p.bmax[int64_t(ti.b) * p.bmax_stride + pos / kPoolBlock] = m;
            atomicAdd(&s_bhist[order_key(m) >> (32 - kHistBits)], 1u);
          }
        }
      } else {
        const int64_t slot = ti.tis * (kTileRows / kPoolBlock) + row / kPoolBlock;
        bool valid = false;
        if (slot < p.npb) {
          const int64_t j = p.pool[int64_t(ti.b) * p.npb + slot];
          const int64_t pos = j * kPoolBlock + (row % kPoolBlock);
          valid = j >= 0 && pos < len;
          if (valid && p.key_scale != nullptr) s *= p.key_scale[seq_base + pos];
          srow[slot * kPoolBlock + (row % kPoolBlock)] = valid ? s : -INFINITY;
        }
        if (valid && p.hist != nullptr) atomicAdd(&s_hist[order_key(s) >> (32 - kHistBits)], 1u);
        if (gmax_row != nullptr) {
          const uint32_t km = __reduce_max_sync(0xffffffffu, valid ? order_key(s) : 0u);
          if (lane == 0) *gmax_row = km;
        }
      }
    }
    if (cur_b >= 0 && p.hist != nullptr) flush(cur_b);
  }

  // ------------------------------- teardown --------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kAccCols);
  }
}

// ---------------------------------------------------------------------------------------
// host: tensor maps through the driver entry point (no link against libcuda)
// ---------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map over [rows][row_bytes] of 1- or 2-byte elements, box [box_rows][box_bytes],
// the given swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* base, bool two_byte, uint64_t row_bytes, uint64_t rows,
              uint32_t box_bytes, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t elem = two_byte ? 2 : 1;
  cuuint64_t dims[2] = {row_bytes / elem, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes / elem), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, two_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int KT, int N>
cudaError_t launch_n(const IndexScoreParams& p, int num_sms, cudaStream_t stream) {
  using Cfg = ScanCfg<KT, N>;
  const bool pool_mode = p.pool != nullptr;
  const int64_t tiles_per_seq =
      pool_mode ? (p.npb + kTileRows / kPoolBlock - 1) / (kTileRows / kPoolBlock)
                : (p.cap + kTileRows - 1) / kTileRows;
  const int64_t total = tiles_per_seq * p.B;
  if (total == 0) return cudaSuccess;
  const uint64_t key_rows = uint64_t(p.B) * uint64_t(p.cap);
  const uint32_t box_rows = pool_mode ? kPoolBlock : kTileRows;
  CUtensorMap tk, tq, tsf;
  bool ok;
  if constexpr (Cfg::kFp4) {
    // codes: rows of 64 bytes, 64-byte swizzle; scales: the [rows][8] plane viewed as
    // [rows / 2][16] (cap is even), unswizzled, two key rows per map row
    ok = make_map(&tk, p.keys, false, 64, key_rows, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_64B) &&
         make_map(&tq, p.q, false, 64, uint64_t(p.B) * uint64_t(p.H_I), 64, N, CU_TENSOR_MAP_SWIZZLE_64B) &&
         make_map(&tsf, p.key_sf, false, 16, key_rows / 2, 16, box_rows / 2, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    const bool two = KT == kKeyBf16;
    const uint64_t row_bytes = two ? 2 * kKeyDim : kKeyDim;
    ok = make_map(&tk, p.keys, two, row_bytes, key_rows, 128, box_rows, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_map(&tq, p.q, two, row_bytes, uint64_t(p.B) * uint64_t(p.H_I), 128, N, CU_TENSOR_MAP_SWIZZLE_128B);
    tsf = tk;  // unused
  }
  if (!ok) return cudaErrorInvalidValue;
  int grid = num_sms * Cfg::kCtasPerSm;
  if (total < grid) grid = static_cast<int>(total);
  auto kern = k_index_score_tc<KT, N>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Cfg::kSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, p, tk, tq, tsf, tiles_per_seq, total);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int KT>
cudaError_t launch_dtype(const IndexScoreParams& p, int num_sms, cudaStream_t stream) {
  if (p.H_I <= 16) return launch_n<KT, 16>(p, num_sms, stream);
  if (p.H_I <= 32) return launch_n<KT, 32>(p, num_sms, stream);
  if (p.H_I <= 48) return launch_n<KT, 48>(p, num_sms, stream);
  return launch_n<KT, 64>(p, num_sms, stream);
}

}  // namespace

cudaError_t launch_index_score(const IndexScoreParams& p, int num_sms, cudaStream_t stream) {
  switch (p.key_type) {
    case kKeyBf16: return launch_dtype<kKeyBf16>(p, num_sms, stream);
    case kKeyE4M3: return launch_dtype<kKeyE4M3>(p, num_sms, stream);
    case kKeyE2M1: return launch_dtype<kKeyE2M1>(p, num_sms, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fp4kv
