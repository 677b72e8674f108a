// Indexer scoring: score[n] = ks[n] * sum_h w[h] * max(0, q[h] . k[n]) for every visible
// entry (Full mode) or for the positions of a candidate pool (Reindex mode).
//
// Method: [PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로 줄이고 …",
//  - section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2": indexer with 32 query heads of
//    dimension 128 scoring the causally visible entries (Full and Reindex rows of the mode
//    table);
//  - section "계층적 희소 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기": the first Full
//    layer also gives every block of 8 positions its largest score (block max), and Reindex
//    layers score only inside the candidate pool.
// The head-combining rule (weighted sum of ReLU dot products) is this library's reading.
//
// Kernel design (one persistent CTA per SM):
//  * a producer warp streams 128-row key tiles (16 KiB of FP8 or 32 KiB of bf16) into an
//    8/4-stage shared-memory ring with 1-D bulk async copies completing on mbarriers (Full
//    mode: one copy per tile; Reindex: one 1 KiB copy per pool block of 8 rows);
//  * 8 consumer warps each take 16 rows of a tile and run m16n8k16 tensor-core MMAs with
//    fp32 accumulation. FP8 E4M3 keys and queries are widened to fp16 (exact) in registers;
//    products of E4M3 values are exact in fp16 x fp16 -> fp32. The 128 key dims are visited
//    in a fixed permutation (identical for keys and queries), chosen so that each lane
//    reads 32 contiguous bytes of a row with conflict-free 16-byte shared loads;
//  * the epilogue combines heads, writes the fp32 score, and adds the score's 12-bit
//    radix digit to a shared-memory histogram that is flushed to global memory per
//    sequence (the first pass of the exact top-K select). With a block-max output it also
//    reduces each block of 8 rows (8 lanes) and histograms the block maxima.
#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"

namespace fp4kv {
namespace {

constexpr int kTileRows = 128;
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kPoolBlock = 8;

template <bool FP8>
struct KeyCfg {
  static constexpr int kRowBytes = FP8 ? 128 : 256;
  static constexpr int kTileBytes = kTileRows * kRowBytes;
  static constexpr int kStages = FP8 ? 8 : 4;
  static constexpr size_t kSmem = size_t(kStages) * kTileBytes + 2 * kStages * sizeof(uint64_t) +
                                  2 * kHistBins * sizeof(uint32_t) + 16;
};

FP4KV_DEV void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers)); }

FP4KV_DEV uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

struct TileRef {
  int b;
  int64_t unit;  // Full: first row of the tile; Reindex: first pool slot of the tile
  bool active;
};

FP4KV_DEV TileRef tile_ref(const IndexScoreParams& p, int64_t t, int64_t tiles_per_seq) {
  TileRef r;
  r.b = static_cast<int>(t / tiles_per_seq);
  const int64_t tis = t % tiles_per_seq;
  if (p.pool == nullptr) {
    r.unit = tis * kTileRows;
    int64_t len = p.seq_lens[r.b];
    if (len > p.cap) len = p.cap;
    r.active = r.unit < len;
  } else {
    r.unit = tis * (kTileRows / kPoolBlock);
    r.active = true;
  }
  return r;
}

template <int NT, bool FP8>
__global__ void __launch_bounds__(kThreads, 1) k_index_score(const IndexScoreParams p,
                                                             int64_t tiles_per_seq,
                                                             int64_t total_tiles) {
  using Cfg = KeyCfg<FP8>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(Cfg::kStages) * Cfg::kTileBytes);
  uint64_t* empty = full + Cfg::kStages;
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(empty + Cfg::kStages);
  uint32_t* s_bhist = s_hist + kHistBins;
  volatile uint32_t* s_abort = s_bhist + kHistBins;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t t_begin = total_tiles * blockIdx.x / gridDim.x;
  const int64_t t_end = total_tiles * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * kHistBins; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------ producer warp ------------------------------------
    if (lane == 0) {
      const uint8_t* keys = static_cast<const uint8_t*>(p.keys);
      uint32_t it = 0;
      for (int64_t t = t_begin; t < t_end; ++t) {
        const TileRef tr = tile_ref(p, t, tiles_per_seq);
        if (!tr.active) continue;
        const int stage = it % Cfg::kStages;
        const uint32_t phase = (it / Cfg::kStages) & 1;
        if (!mbar_wait(&empty[stage], phase ^ 1)) {
          atomicOr(p.status, kFlagWaitTimeout);
          *s_abort = 1;
          break;
        }
        uint8_t* dst = ring + size_t(stage) * Cfg::kTileBytes;
        const int64_t seq_base = int64_t(tr.b) * p.cap;
        if (p.pool == nullptr) {
          int64_t rows = p.cap - tr.unit;
          if (rows > kTileRows) rows = kTileRows;
          const uint32_t bytes = uint32_t(rows) * Cfg::kRowBytes;
          mbar_arrive_expect_tx(&full[stage], bytes);
          bulk_g2s(dst, keys + (seq_base + tr.unit) * Cfg::kRowBytes, bytes, &full[stage]);
        } else {
          const int32_t* pl = p.pool + int64_t(tr.b) * p.npb;
          uint32_t total = 0;
          for (int s = 0; s < kTileRows / kPoolBlock; ++s) {
            const int64_t slot = tr.unit + s;
            if (slot >= p.npb) break;
            const int64_t j = pl[slot];
            if (j < 0 || j * kPoolBlock >= p.cap) continue;
            int64_t rows = p.cap - j * kPoolBlock;
            if (rows > kPoolBlock) rows = kPoolBlock;
            total += uint32_t(rows) * Cfg::kRowBytes;
          }
          mbar_arrive_expect_tx(&full[stage], total);
          for (int s = 0; s < kTileRows / kPoolBlock; ++s) {
            const int64_t slot = tr.unit + s;
            if (slot >= p.npb) break;
            const int64_t j = pl[slot];
            if (j < 0 || j * kPoolBlock >= p.cap) continue;
            int64_t rows = p.cap - j * kPoolBlock;
            if (rows > kPoolBlock) rows = kPoolBlock;
            bulk_g2s(dst + s * kPoolBlock * Cfg::kRowBytes,
                     keys + (seq_base + j * kPoolBlock) * Cfg::kRowBytes,
                     uint32_t(rows) * Cfg::kRowBytes, &full[stage]);
          }
        }
        ++it;
      }
    }
    return;
  }

  // ------------------------------ consumer warps -------------------------------------
  const int g = lane >> 2;  // row within the 8-row half of the warp's 16 rows
  const int tq = lane & 3;  // quad lane: owns key dims [32*tq, 32*tq + 32)
  uint32_t bq[NT][8][2];    // query fragments (B operand), per n-tile and k-step
  float wv[NT][2];
  int cur_b = -1;
  uint32_t it = 0;

  auto flush_hist = [&](int b) {
    consumer_sync();
    for (int i = threadIdx.x; i < kHistBins; i += kConsumers) {
      const uint32_t c = s_hist[i];
      if (c) atomicAdd(p.hist + int64_t(b) * kHistBins + i, c);
      s_hist[i] = 0;
      if (p.bmax != nullptr) {
        const uint32_t c2 = s_bhist[i];
        if (c2) atomicAdd(p.bmax_hist + int64_t(b) * kHistBins + i, c2);
        s_bhist[i] = 0;
      }
    }
    consumer_sync();
  };

  auto load_query = [&](int b) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int h = nt * 8 + g;
      if (h < p.H_I) {
        if constexpr (FP8) {
          const uint8_t* qr = static_cast<const uint8_t*>(p.q) + (int64_t(b) * p.H_I + h) * kKeyDim +
                              32 * tq;
          const uint4 c0 = *reinterpret_cast<const uint4*>(qr);
          const uint4 c1 = *reinterpret_cast<const uint4*>(qr + 16);
          const uint32_t wd[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            bq[nt][s][0] = e4m3x2_to_f16x2(static_cast<uint16_t>(wd[s] & 0xffffu));
            bq[nt][s][1] = e4m3x2_to_f16x2(static_cast<uint16_t>(wd[s] >> 16));
          }
        } else {
          const uint16_t* qr = static_cast<const uint16_t*>(p.q) +
                               (int64_t(b) * p.H_I + h) * kKeyDim + 32 * tq;
          uint32_t wd[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(qr + 8 * c);
            wd[4 * c] = v.x; wd[4 * c + 1] = v.y; wd[4 * c + 2] = v.z; wd[4 * c + 3] = v.w;
          }
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            bq[nt][s][0] = wd[2 * s];
            bq[nt][s][1] = wd[2 * s + 1];
          }
        }
      } else {
#pragma unroll
        for (int s = 0; s < 8; ++s) bq[nt][s][0] = bq[nt][s][1] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int hw = nt * 8 + 2 * tq + j;
        wv[nt][j] = hw < p.H_I ? p.w[int64_t(b) * p.H_I + hw] : 0.0f;
      }
    }
  };

  for (int64_t t = t_begin; t < t_end; ++t) {
    const TileRef tr = tile_ref(p, t, tiles_per_seq);
    if (!tr.active) continue;
    if (*s_abort) break;
    const int stage = it % Cfg::kStages;
    const uint32_t phase = (it / Cfg::kStages) & 1;
    ++it;
    if (!mbar_wait(&full[stage], phase)) {
      atomicOr(p.status, kFlagWaitTimeout);
      *s_abort = 1;
      break;
    }
    if (tr.b != cur_b) {
      if (cur_b >= 0 && p.hist != nullptr) flush_hist(cur_b);
      load_query(tr.b);
      cur_b = tr.b;
    }

    // ---- A fragments: rows ra = 16*warp + g and rb = ra + 8 of the tile ----
    const uint8_t* tile = ring + size_t(stage) * Cfg::kTileBytes;
    const int ra = 16 * warp + g;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;

    if constexpr (FP8) {
      // lanes of an 8-lane phase cover rows (2k, 2k+1); odd rows read their two chunks in
      // the opposite order so the phase touches 8 distinct 4-bank groups
      const int c_first = 2 * tq + (g & 1);
      const int c_second = 2 * tq + 1 - (g & 1);
      uint4 a0 = lds128(tile + ra * 128 + c_first * 16);
      uint4 a1 = lds128(tile + ra * 128 + c_second * 16);
      uint4 b0 = lds128(tile + (ra + 8) * 128 + c_first * 16);
      uint4 b1 = lds128(tile + (ra + 8) * 128 + c_second * 16);
      if (g & 1) {
        const uint4 ta = a0; a0 = a1; a1 = ta;
        const uint4 tb = b0; b0 = b1; b1 = tb;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t a[4];
        a[0] = e4m3x2_to_f16x2(static_cast<uint16_t>(wa[s] & 0xffffu));
        a[1] = e4m3x2_to_f16x2(static_cast<uint16_t>(wb[s] & 0xffffu));
        a[2] = e4m3x2_to_f16x2(static_cast<uint16_t>(wa[s] >> 16));
        a[3] = e4m3x2_to_f16x2(static_cast<uint16_t>(wb[s] >> 16));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_f16_16816(acc[nt], a, bq[nt][s][0], bq[nt][s][1]);
      }
    } else {
      uint32_t wa[16], wb[16];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 va = lds128(tile + ra * 256 + 64 * tq + 16 * c);
        const uint4 vb = lds128(tile + (ra + 8) * 256 + 64 * tq + 16 * c);
        wa[4 * c] = va.x; wa[4 * c + 1] = va.y; wa[4 * c + 2] = va.z; wa[4 * c + 3] = va.w;
        wb[4 * c] = vb.x; wb[4 * c + 1] = vb.y; wb[4 * c + 2] = vb.z; wb[4 * c + 3] = vb.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t a[4] = {wa[2 * s], wb[2 * s], wa[2 * s + 1], wb[2 * s + 1]};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt], a, bq[nt][s][0], bq[nt][s][1]);
      }
    }

    // ---- epilogue: combine heads -> score of rows ra, rb ----
    float sa = 0.0f, sb = 0.0f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      sa += wv[nt][0] * fmaxf(acc[nt][0], 0.0f) + wv[nt][1] * fmaxf(acc[nt][1], 0.0f);
      sb += wv[nt][0] * fmaxf(acc[nt][2], 0.0f) + wv[nt][1] * fmaxf(acc[nt][3], 0.0f);
    }
    sa += __shfl_xor_sync(0xffffffffu, sa, 1);
    sb += __shfl_xor_sync(0xffffffffu, sb, 1);
    sa += __shfl_xor_sync(0xffffffffu, sa, 2);
    sb += __shfl_xor_sync(0xffffffffu, sb, 2);

    int64_t len = p.seq_lens[tr.b];
    if (len > p.cap) len = p.cap;
    const int64_t seq_base = int64_t(tr.b) * p.cap;
    if (p.pool == nullptr) {
      const int64_t pa = tr.unit + ra, pb = pa + 8;
      const bool va = pa < len, vb = pb < len;
      if (p.key_scale != nullptr) {
        if (va) sa *= p.key_scale[seq_base + pa];
        if (vb) sb *= p.key_scale[seq_base + pb];
      }
      float* srow = p.scores + int64_t(tr.b) * p.score_stride;
      if (tq == 0 && va) {
        srow[pa] = sa;
        if (p.hist != nullptr) atomicAdd(&s_hist[order_key(sa) >> (32 - kHistBits)], 1u);
      }
      if (tq == 1 && vb) {
        srow[pb] = sb;
        if (p.hist != nullptr) atomicAdd(&s_hist[order_key(sb) >> (32 - kHistBits)], 1u);
      }
      if (p.bmax != nullptr) {
        float ma = va ? sa : -INFINITY, mb = vb ? sb : -INFINITY;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
          mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
        }
        const int64_t blk = (tr.unit + 16 * warp) / kPoolBlock;
        float* brow = p.bmax + int64_t(tr.b) * p.bmax_stride;
        if (lane == 0 && ma > -INFINITY) {
          brow[blk] = ma;
          atomicAdd(&s_bhist[order_key(ma) >> (32 - kHistBits)], 1u);
        }
        if (lane == 1 && mb > -INFINITY) {
          brow[blk + 1] = mb;
          atomicAdd(&s_bhist[order_key(mb) >> (32 - kHistBits)], 1u);
        }
      }
    } else {
      const int32_t* pl = p.pool + int64_t(tr.b) * p.npb;
      const int64_t slot_a = tr.unit + 2 * warp, slot_b = slot_a + 1;
      float* srow = p.scores + int64_t(tr.b) * p.score_stride;
      if (tq <= 1) {
        const int64_t slot = tq == 0 ? slot_a : slot_b;
        float s = tq == 0 ? sa : sb;
        if (slot < p.npb) {
          const int64_t j = pl[slot];
          const int64_t pos = j * kPoolBlock + g;
          const bool valid = j >= 0 && pos < len;
          if (valid && p.key_scale != nullptr) s *= p.key_scale[seq_base + pos];
          srow[slot * kPoolBlock + g] = valid ? s : -INFINITY;
          if (valid && p.hist != nullptr)
            atomicAdd(&s_hist[order_key(s) >> (32 - kHistBits)], 1u);
        }
      }
    }
  }
  if (cur_b >= 0 && p.hist != nullptr) flush_hist(cur_b);
}

template <int NT, bool FP8>
cudaError_t launch_nt(const IndexScoreParams& p, int num_sms, cudaStream_t stream) {
  using Cfg = KeyCfg<FP8>;
  const int64_t tiles_per_seq =
      p.pool == nullptr ? (p.cap + kTileRows - 1) / kTileRows
                        : (p.npb + kTileRows / kPoolBlock - 1) / (kTileRows / kPoolBlock);
  const int64_t total = tiles_per_seq * p.B;
  if (total == 0) return cudaSuccess;
  int grid = num_sms;
  if (total < grid) grid = static_cast<int>(total);
  auto kern = k_index_score<NT, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Cfg::kSmem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, Cfg::kSmem, stream>>>(p, tiles_per_seq, total);
  return cudaGetLastError();
}

template <bool FP8>
cudaError_t launch_dtype(const IndexScoreParams& p, int num_sms, cudaStream_t stream) {
  const int nt = (p.H_I + 7) / 8;
  if (nt <= 1) return launch_nt<1, FP8>(p, num_sms, stream);
  if (nt <= 2) return launch_nt<2, FP8>(p, num_sms, stream);
  if (nt <= 4) return launch_nt<4, FP8>(p, num_sms, stream);
  return launch_nt<8, FP8>(p, num_sms, stream);
}

}  // namespace

cudaError_t launch_index_score(const IndexScoreParams& p, int num_sms, cudaStream_t stream) {
  return p.keys_fp8 ? launch_dtype<true>(p, num_sms, stream)
                    : launch_dtype<false>(p, num_sms, stream);
}

}  // namespace fp4kv
