// kv_quant_fp4: quantize-on-write of bf16 KV rows into packed E2M1 codes + E4M3 scales;
// swa_quant_fp8: the sliding-window KV's write, bf16 rows into E4M3 codes.
//
// Method: [PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로 줄이고 …", section
// "890바이트를 만든 나머지 절반, FP4 KV 캐시와 지속 캐시 재설계": the main KV is kept as E2M1
// values with one E4M3 scale per 16 channels (largest magnitude 448 x 6 = 2688).
//
// Per 16-channel group: S = E4M3_RNE_sat(amax / 6); code = sign(x) | E2M1_RNE_sat(|x| / S).
//
// Exactness argument (the kernel must agree bit for bit with the exact definition):
//  * amax / 6 is computed by an IEEE fp32 division. The exact quotient of a bf16 amax by 6
//    is either an E4M3 rounding midpoint itself (then the division is exact) or lies at a
//    relative distance >= 2^-14.5 from every midpoint, far beyond the 2^-24 error of the
//    division; the hardware cvt then rounds to nearest-even and saturates at 448.
//  * |x| / S is formed as |x| * RN(1/S) + 128 in one fused multiply-add (so the product is
//    rounded once, to a multiple of 2^-16), minus 128. RN(1/S) is within 2^-24 relative of
//    1/S, so for r < 8 an exact tie r = t (t a multiple of 1/4) is within 2^-21 of t and
//    snaps to it exactly, while a non-tie bf16/E4M3 ratio is at least 2^-10 away from every
//    E2M1 midpoint, so the snap cannot move it across one. Ratios >= 8 saturate either way.
//  * cvt.rn.satfinite.e2m1x2.f32 rounds to nearest-even on the code and saturates at 6; it
//    gets the ratio with x's sign bit put back, and rounding is symmetric, so the code is
//    sign | RNE(|x| / S): -0 and negative values rounding to zero give 0x8.
// Memory: at d = 512 (with 16-byte aligned codes) half a warp per row, two groups per lane,
// four rows' loads in flight per warp; otherwise one warp per row, one 16-channel group per
// lane (32 B read, 8 B + 1 B written per lane).
#include "fp4kv_common.cuh"
#include "fp4kv_sm100.cuh"
#include "fp4kv_launch.h"

namespace fp4kv {

namespace {

// RN(a * inv + 128) - 128: the ratio a * inv rounded once to a multiple of 2^-16 (for
// a * inv < 128; larger ratios saturate the code either way)
FP4KV_DEV float snap_ratio(float a, float inv) {
  return __fadd_rn(__fmaf_rn(a, inv, 128.0f), -128.0f);
}

// Quantize one group of 16 bf16 values held as 8 words (2 values per word, low half first).
// Returns the 8 packed bytes (low nibble = even channel) and the scale code.
FP4KV_DEV void quant_group(const uint32_t (&w)[8], uint2& packed, uint32_t& scale_code) {
  uint32_t m2 = 0;  // per-half maxima of the 15-bit magnitudes
#pragma unroll
  for (int i = 0; i < 8; ++i) m2 = __vmaxu2(m2, w[i] & 0x7fff7fffu);
  const uint32_t m = max(m2 & 0xffffu, m2 >> 16);
  const float amax = bf16_bits_to_f32(m);
  const uint32_t sc = f32_to_e4m3_satfinite(__fdiv_rn(amax, 6.0f));
  const float S = f16_lo_to_f32(e4m3x2_to_f16x2(static_cast<uint16_t>(sc)));
  uint32_t bytes[8];
  if (S > 0.0f) {
    const float inv = __frcp_rn(S);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t e = w[i] << 16, o = w[i] & 0xffff0000u;  // the two channels as f32 bits
      const float r0 = snap_ratio(__uint_as_float(e & 0x7fffffffu), inv);
      const float r1 = snap_ratio(__uint_as_float(o & 0x7fffffffu), inv);
      // the sign goes back on before the rounding to E2M1, which is symmetric; a negative
      // value that rounds to zero keeps its sign (code 0x8)
      bytes[i] = f32x2_to_e2m1x2_satfinite(__uint_as_float(__float_as_uint(r0) | (e & 0x80000000u)),
                                           __uint_as_float(__float_as_uint(r1) | (o & 0x80000000u)));
    }
  } else {  // an all-zero group: sign-only codes
#pragma unroll
    for (int i = 0; i < 8; ++i) bytes[i] = ((w[i] >> 12) & 0x8u) | ((w[i] >> 24) & 0x80u);
  }
  packed.x = bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24);
  packed.y = bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24);
  scale_code = sc;
}

__global__ void __launch_bounds__(256) k_kv_quant_fp4(const uint16_t* __restrict__ x,
                                                      int64_t n_rows, int d, int64_t x_stride,
                                                      const int64_t* __restrict__ dst_row,
                                                      uint8_t* __restrict__ packed,
                                                      uint8_t* __restrict__ scales,
                                                      int64_t cap_rows) {
  // the indexer scan that follows on the stream may start its prologue now (it waits for
  // this grid before reading anything)
  griddep_launch_dependents();
  // launched as a programmatic dependent: the kernel before it on the stream (the previous
  // step's attention merge, whose attention may still read these rows) is complete past here
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int groups = d / kGroup;
  for (int64_t r = warp; r < n_rows; r += nwarps) {
    const int64_t dst = dst_row ? dst_row[r] : r;
    if (dst < 0 || dst >= cap_rows) continue;
    const uint16_t* xr = x + r * x_stride;
    uint8_t* pr = packed + dst * (d / 2);
    uint8_t* sr = scales + dst * groups;
    for (int g = lane; g < groups; g += 32) {
      const uint4 v0 = ld_stream_v4(xr + g * kGroup);
      const uint4 v1 = ld_stream_v4(xr + g * kGroup + 8);
      const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint2 pk;
      uint32_t sc;
      quant_group(w, pk, sc);
      *reinterpret_cast<uint2*>(pr + g * 8) = pk;
      sr[g] = static_cast<uint8_t>(sc);
    }
  }
}

// d = 512, the path of the bulk writes: half a warp per row and two 16-channel groups per
// lane (64 B read, one 16-byte packed store and one 2-byte scale store per lane), and the
// loads of kRows rows (kRows / 2 row pairs, 128 B per lane) issued before any is quantized, so
// that enough bytes are in flight to stream at the HBM rate.
constexpr int kRows512 = 4;
__global__ void __launch_bounds__(256) k_kv_quant_fp4_d512(const uint16_t* __restrict__ x, int64_t n_rows,
                                                           int64_t x_stride, const int64_t* __restrict__ dst_row,
                                                           uint8_t* __restrict__ packed,
                                                           uint8_t* __restrict__ scales, int64_t cap_rows) {
  griddep_launch_dependents();
  griddep_wait();  // (as in k_kv_quant_fp4)
  constexpr int kD = 512, kGroups = kD / kGroup;
  const int lane = threadIdx.x & 31, half = lane >> 4, hl = lane & 15;
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r0 = warp * kRows512; r0 < n_rows; r0 += nwarps * kRows512) {
    uint4 v[kRows512 / 2][4];
    int64_t row[kRows512 / 2];
#pragma unroll
    for (int k = 0; k < kRows512 / 2; ++k) {
      row[k] = r0 + 2 * k + half;
      if (row[k] < n_rows) {
        const uint16_t* xr = x + row[k] * x_stride + 2 * kGroup * hl;
#pragma unroll
        for (int j = 0; j < 4; ++j) v[k][j] = ld_stream_v4(xr + 8 * j);
      }
    }
#pragma unroll
    for (int k = 0; k < kRows512 / 2; ++k) {
      if (row[k] >= n_rows) continue;
      const int64_t dst = dst_row ? dst_row[row[k]] : row[k];
      if (dst < 0 || dst >= cap_rows) continue;
      const uint32_t wa[8] = {v[k][0].x, v[k][0].y, v[k][0].z, v[k][0].w, v[k][1].x, v[k][1].y, v[k][1].z, v[k][1].w};
      const uint32_t wb[8] = {v[k][2].x, v[k][2].y, v[k][2].z, v[k][2].w, v[k][3].x, v[k][3].y, v[k][3].z, v[k][3].w};
      uint2 pa, pb;
      uint32_t sa, sb;
      quant_group(wa, pa, sa);
      quant_group(wb, pb, sb);
      *reinterpret_cast<uint4*>(packed + dst * (kD / 2) + 16 * hl) = make_uint4(pa.x, pa.y, pb.x, pb.y);
      *reinterpret_cast<uint16_t*>(scales + dst * kGroups + 2 * hl) = static_cast<uint16_t>(sa | (sb << 8));
    }
  }
}

// SWA KV write: bf16 rows -> E4M3 codes (round to nearest even, saturating at +-448), one
// byte per channel ([PyTorchKR] FP4 KV section: the quantization-sensitive SWA KV stays
// FP8). One warp per row, 16 channels per lane and step: 32 B read, 16 B written per lane.
__global__ void __launch_bounds__(256) k_swa_quant_fp8(const uint16_t* __restrict__ x, int64_t n_rows,
                                                       int d, int64_t x_stride,
                                                       const int64_t* __restrict__ dst_row,
                                                       uint8_t* __restrict__ out, int64_t cap_rows) {
  griddep_launch_dependents();
  griddep_wait();  // (as in k_kv_quant_fp4)
  const int lane = threadIdx.x & 31;
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = warp; r < n_rows; r += nwarps) {
    const int64_t dst = dst_row ? dst_row[r] : r;
    if (dst < 0 || dst >= cap_rows) continue;
    const uint16_t* xr = x + r * x_stride;
    uint8_t* orow = out + dst * d;
    for (int c = 16 * lane; c < d; c += 16 * 32) {
      const uint4 v0 = ld_stream_v4(xr + c);
      const uint4 v1 = ld_stream_v4(xr + c + 8);
      const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint16_t lo, hi;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo)
            : "f"(bf16_bits_to_f32(w[2 * k] >> 16)), "f"(bf16_bits_to_f32(w[2 * k] & 0xffffu)));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi)
            : "f"(bf16_bits_to_f32(w[2 * k + 1] >> 16)), "f"(bf16_bits_to_f32(w[2 * k + 1] & 0xffffu)));
        // the sign of x is kept (a negative value that rounds to zero is 0x80)
        const uint32_t w0 = w[2 * k], w1 = w[2 * k + 1];
        o[k] = (uint32_t(lo) | ((w0 >> 8) & 0x80u) | ((w0 >> 16) & 0x8000u)) |
               ((uint32_t(hi) | ((w1 >> 8) & 0x80u) | ((w1 >> 16) & 0x8000u)) << 16);
      }
      *reinterpret_cast<uint4*>(orow + c) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// A launch that may begin while the kernel before it on the stream finishes (programmatic
// dependent launch); the kernel orders itself with griddep_wait().
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, cudaStream_t stream, Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace

cudaError_t launch_swa_quant_fp8(const uint16_t* x, int64_t n_rows, int d, int64_t x_stride,
                                 const int64_t* dst_row, uint8_t* out, int64_t cap_rows, int num_sms,
                                 cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (n_rows + 7) / 8;
  const int64_t max_blocks = static_cast<int64_t>(num_sms) * 8;
  if (blocks > max_blocks) blocks = max_blocks;
  cudaError_t e = launch_pdl(k_swa_quant_fp8, dim3(static_cast<unsigned>(blocks)), dim3(threads), stream, x, n_rows,
                             d, x_stride, dst_row, out, cap_rows);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_kv_quant_fp4(const uint16_t* x, int64_t n_rows, int d, int64_t x_stride,
                                const int64_t* dst_row, uint8_t* packed, uint8_t* scales,
                                int64_t cap_rows, int num_sms, cudaStream_t stream) {
  if (n_rows == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t max_blocks = static_cast<int64_t>(num_sms) * 8;
  // (x is 16-byte aligned and its stride a multiple of 8 elements, so its rows are too)
  if (d == 512 && (reinterpret_cast<uintptr_t>(packed) & 15u) == 0 && (reinterpret_cast<uintptr_t>(scales) & 1u) == 0) {
    // one resident wave: the grid-stride loop then ends on every SM at about the same time
    static int per_sm = 0;
    if (per_sm == 0 &&
        (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_kv_quant_fp4_d512, threads, 0) != cudaSuccess ||
         per_sm < 1))
      per_sm = 2;
    const int64_t rows_per_block = (threads / 32) * kRows512;
    int64_t blocks = (n_rows + rows_per_block - 1) / rows_per_block;
    if (blocks > int64_t(num_sms) * per_sm) blocks = int64_t(num_sms) * per_sm;
    cudaError_t e = launch_pdl(k_kv_quant_fp4_d512, dim3(static_cast<unsigned>(blocks)), dim3(threads), stream, x,
                               n_rows, x_stride, dst_row, packed, scales, cap_rows);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  const int64_t rows_per_block = threads / 32;
  int64_t blocks = (n_rows + rows_per_block - 1) / rows_per_block;
  if (blocks > max_blocks) blocks = max_blocks;
  cudaError_t e = launch_pdl(k_kv_quant_fp4, dim3(static_cast<unsigned>(blocks)), dim3(threads), stream, x, n_rows,
                             d, x_stride, dst_row, packed, scales, cap_rows);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp4kv
