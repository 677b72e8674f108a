// Device helpers shared by the libfp4kv kernels (sm_100a).
//
// Only thin wrappers around documented PTX instructions live here: mbarriers, bulk
// asynchronous copies, ldmatrix / mma.sync, and the FP4 / FP8 conversion instructions.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#define FP4KV_DEV __device__ __forceinline__

namespace fp4kv {

// ---------------------------------------------------------------------------------------
// Library-wide constants
// ---------------------------------------------------------------------------------------
constexpr int kGroup = 16;          // channels per E4M3 scale
constexpr int kKeyDim = 128;        // indexer head dimension
constexpr int kHistBits = 12;       // first-level radix digit of the top-K select
constexpr int kHistBins = 1 << kHistBits;
constexpr uint32_t kSpinLimit = 1u << 26;  // bounded waits: ~seconds, then give up

// Status word bits written by kernels into the workspace header.
constexpr uint32_t kFlagWaitTimeout = 1u;

// ---------------------------------------------------------------------------------------
// Bit helpers
// ---------------------------------------------------------------------------------------
FP4KV_DEV float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Order-preserving map fp32 -> uint32 (larger float -> larger key). -0.0 is first folded
// into +0.0 so that equal scores compare equal.
FP4KV_DEV uint32_t order_key(float f) {
  f = f + 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
FP4KV_DEV float key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

// ---------------------------------------------------------------------------------------
// FP8 / FP4 conversions (hardware cvt instructions)
// ---------------------------------------------------------------------------------------
// fp32 -> E4M3 code, round-to-nearest-even, saturating to +-448.
FP4KV_DEV uint32_t f32_to_e4m3_satfinite(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xffu;
}
// Two fp32 -> one byte of E2M1 codes, round-to-nearest-even, saturating at +-6 (the sign
// in bits 3 and 7: -0 and negative values that round to zero give 0x8). `lo` lands in
// bits 0..3, `hi` in bits 4..7.
FP4KV_DEV uint32_t f32x2_to_e2m1x2_satfinite(float lo, float hi) {
  uint32_t r;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// One byte of two E2M1 codes -> f16x2 (low nibble in the low half). Exact.
FP4KV_DEV uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}"
      : "=r"(r) : "r"(byte));
  return r;
}
// Two E4M3 codes (low byte, next byte) -> f16x2. Exact.
FP4KV_DEV uint32_t e4m3x2_to_f16x2(uint16_t two) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(two));
  return r;
}
FP4KV_DEV uint32_t hmul2_f16(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
FP4KV_DEV uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
FP4KV_DEV float f16_lo_to_f32(uint32_t h2) {
  float f;
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n cvt.f32.f16 %0, l;\n}" : "=f"(f) : "r"(h2));
  return f;
}
FP4KV_DEV float f16_hi_to_f32(uint32_t h2) {
  float f;
  asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n cvt.f32.f16 %0, h;\n}" : "=f"(f) : "r"(h2));
  return f;
}

// ---------------------------------------------------------------------------------------
// Shared-memory addressing, mbarriers and bulk async copies
// ---------------------------------------------------------------------------------------
FP4KV_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

FP4KV_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
FP4KV_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
FP4KV_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}"
               ::"r"(smem_u32(bar)) : "memory");
}
FP4KV_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
FP4KV_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and the caller must bail out) after kSpinLimit polls.
FP4KV_DEV bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// 1-D bulk copy global -> shared, completing on an mbarrier (transaction bytes).
// dst, src 16-byte aligned; bytes a multiple of 16.
FP4KV_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------------------------------
// Warp-level tensor-core MMA (m16n8k16, fp16 inputs, fp32 accumulate) and ldmatrix
// ---------------------------------------------------------------------------------------
FP4KV_DEV void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
FP4KV_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
FP4KV_DEV void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
FP4KV_DEV void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

FP4KV_DEV uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
// 8 bytes of a randomly addressed 32-byte record: the 64-byte L2 fetch hint halves what a
// miss brings from DRAM (a miss otherwise fills a whole 128-byte line)
FP4KV_DEV uint2 ld_nc_v2_64b(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::64B.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
FP4KV_DEV uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

FP4KV_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
FP4KV_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace fp4kv
