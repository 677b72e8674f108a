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
//  * S = q . v_hat on tensor cores (fp16 x fp16 -> fp32); online softmax in fp32 with exp2.
//  * P is split as P_hi + P_lo, both fp16, after scaling by 2^8 (P_lo stays out of the fp16
//    subnormal range); P.V is two MMAs, so P carries ~22 bits into the product.
//
// Work split: CTA = (chunk of the index list, group of <= 64 heads, sequence); 8 warps.
// Per sub-tile of 64 entries: the warps gather packed rows + scales with coalesced 16-byte
// loads and write fp16 rows into an XOR-swizzled shared buffer (conflict-free for stores and
// for ldmatrix); S = Q V^T (m16n8k16 MMAs), per-head running max / sum, P to shared memory,
// O += P V. Each chunk writes its unnormalised O with (max, sum); a small second kernel
// (k_attn_combine, one warp per head) merges the chunks. No CTA waits on another.
#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"

namespace fp4kv {
namespace {

constexpr int kD = 512;          // latent width the kernel is built for
constexpr int kHeadsPerCta = 64;
constexpr int kSub = 64;         // entries per sub-tile
constexpr int kAttnThreads = 256;
constexpr float kPScale = 256.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr size_t kSmemQ = size_t(kHeadsPerCta) * kD * 2;
constexpr size_t kSmemV = size_t(kSub) * kD * 2;
constexpr size_t kSmemP = size_t(kHeadsPerCta) * kSub * 2;
constexpr size_t kSmemAttn = kSmemQ + kSmemV + 2 * kSmemP + 64 * 4 + 8 * 16 * 4 + 64 * 4 + 16;

// byte offset of 16-byte chunk `c` of row `r` in a buffer of 1 KiB rows (64 chunks)
FP4KV_DEV uint32_t off_wide(int r, int c) { return uint32_t(r) * 1024u + (uint32_t(c ^ (r & 7)) << 4); }
// same for 128-byte rows (8 chunks)
FP4KV_DEV uint32_t off_narrow(int r, int c) { return uint32_t(r) * 128u + (uint32_t(c ^ (r & 7)) << 4); }

FP4KV_DEV void ldmatrix_x2(uint32_t& r0, uint32_t& r1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1) : "r"(addr));
}

template <int MT>
__global__ void __launch_bounds__(kAttnThreads, 1) k_sparse_attn(const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sV = sQ + kSmemQ;
  uint8_t* sPh = sV + kSmemV;
  uint8_t* sPl = sPh + kSmemP;
  float* sC = reinterpret_cast<float*>(sPl + kSmemP);  // [64] log2-domain logit scale
  float* sRed = sC + 64;                                // [8 warps][16 rows]
  int32_t* sIdx = reinterpret_cast<int32_t*>(sRed + 128);  // [64] position or -1

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int chunk = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int n_hg = gridDim.y;
  const int hbase = hg * kHeadsPerCta;
  const int nh = min(kHeadsPerCta, p.H - hbase);
  int64_t len = p.seq_lens[b];
  if (len > p.cap) len = p.cap;

  // ---- Q: bf16 -> fp16 with a per-head power-of-two scale, swizzled rows ----
  for (int hh = warp; hh < kHeadsPerCta; hh += 8) {
    uint4 o0 = make_uint4(0, 0, 0, 0), o1 = o0;
    float c = 0.0f;
    if (hh < nh) {
      const uint16_t* qr = p.q + (int64_t(b) * p.H + hbase + hh) * kD + 16 * lane;
      const uint4 v0 = *reinterpret_cast<const uint4*>(qr);
      const uint4 v1 = *reinterpret_cast<const uint4*>(qr + 8);
      const uint32_t wd[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t m = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = max(m, max(wd[i] & 0x7fffu, (wd[i] >> 16) & 0x7fffu));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      int k = 0;
      if (m != 0) {
        const int e = int((m >> 7) & 0xff) - 127;  // exponent of max|q| (bf16 normal)
        k = 14 - (e < -126 ? -126 : e);
        if (k > 127) k = 127;
        if (k < -126) k = -126;
      }
      const float up = __uint_as_float(uint32_t(127 + k) << 23);
      uint32_t h[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        h[i] = pack_f16x2(bf16_bits_to_f32(wd[i] & 0xffffu) * up, bf16_bits_to_f32(wd[i] >> 16) * up);
      o0 = make_uint4(h[0], h[1], h[2], h[3]);
      o1 = make_uint4(h[4], h[5], h[6], h[7]);
      // 2^-k in two steps so that it never underflows or overflows as a float
      c = p.sm_scale * kLog2e * __uint_as_float(uint32_t(127 - k / 2) << 23) *
          __uint_as_float(uint32_t(127 - (k - k / 2)) << 23);
    }
    *reinterpret_cast<uint4*>(sQ + off_wide(hh, 2 * lane)) = o0;
    *reinterpret_cast<uint4*>(sQ + off_wide(hh, 2 * lane + 1)) = o1;
    if (lane == 0) sC[hh] = c;
  }

  // ---- per-warp roles ----
  const int mt = warp % MT;         // m-tile (16 heads) of this warp in both phases
  const int wi = warp / MT;         // index among the warps sharing the m-tile
  constexpr int kWarpsPerMt = 8 / MT;
  constexpr int kNtS = MT;          // S: n-tiles (8 entries) per warp
  constexpr int kNtO = 8 * MT;      // PV: n-tiles (8 dims) per warp
  const int dim0 = wi * (kD / kWarpsPerMt);

  float o[kNtO][4];
#pragma unroll
  for (int i = 0; i < kNtO; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m_g = -INFINITY, m_g8 = -INFINITY, l_g = 0.0f, l_g8 = 0.0f;

  const int n_chunks = gridDim.x;
  const int e_begin = int(int64_t(p.top_k) * chunk / n_chunks);
  const int e_end = int(int64_t(p.top_k) * (chunk + 1) / n_chunks);
  const int32_t* idx = p.idx + int64_t(b) * p.top_k;
  const uint8_t* packed_b = p.packed + int64_t(b) * p.cap * (kD / 2);
  const uint8_t* scales_b = p.scales + int64_t(b) * p.cap * (kD / kGroup);

  for (int st = e_begin; st < e_end; st += kSub) {
    if (tid < kSub) {
      const int j = st + tid;
      int32_t pos = j < e_end ? idx[j] : -1;
      if (pos < 0 || pos >= len) pos = -1;
      sIdx[tid] = pos;
    }
    __syncthreads();  // sIdx ready; previous sub-tile fully consumed

    // ---- gather + dequantize: warp -> 8 entries, lane -> (entry, quarter) ----
    {
      const int e = 8 * warp + (lane & 7);
      const int qd = lane >> 3;
      const int32_t pos = sIdx[e];
      if (pos >= 0) {
        const uint8_t* prow = packed_b + int64_t(pos) * (kD / 2);
        const uint8_t* srow = scales_b + int64_t(pos) * (kD / kGroup);
        uint4 pk[4];
        uint16_t sp[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int pc = qd + 4 * j;
          pk[j] = ld_nc_v4(prow + 16 * pc);
          sp[j] = __ldg(reinterpret_cast<const unsigned short*>(srow + 2 * pc));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int pc = qd + 4 * j;
          const uint32_t s_lo = e4m3x2_to_f16x2(uint16_t((sp[j] & 0xffu) * 0x101u));
          const uint32_t s_hi = e4m3x2_to_f16x2(uint16_t((sp[j] >> 8) * 0x101u));
          const uint32_t wd[4] = {pk[j].x, pk[j].y, pk[j].z, pk[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t s2 = i < 2 ? s_lo : s_hi;
            uint4 v;
            v.x = hmul2_f16(e2m1x2_to_f16x2(wd[i] & 0xffu), s2);
            v.y = hmul2_f16(e2m1x2_to_f16x2((wd[i] >> 8) & 0xffu), s2);
            v.z = hmul2_f16(e2m1x2_to_f16x2((wd[i] >> 16) & 0xffu), s2);
            v.w = hmul2_f16(e2m1x2_to_f16x2(wd[i] >> 24), s2);
            *reinterpret_cast<uint4*>(sV + off_wide(e, 4 * pc + i)) = v;
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(sV + off_wide(e, 4 * (qd + 4 * j) + i)) = make_uint4(0, 0, 0, 0);
      }
    }
    __syncthreads();

    // ---- S = Q V^T for (m-tile mt, entries [8*kNtS*wi, +8*kNtS)) ----
    float acc[kNtS][4];
#pragma unroll
    for (int j = 0; j < kNtS; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.0f;
    const uint32_t sQ_base = smem_u32(sQ), sV_base = smem_u32(sV);
    const int arow = 16 * mt + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll 4
    for (int ks = 0; ks < kD / 16; ++ks) {
      uint32_t a[4];
      ldmatrix_x4(a, sQ_base + off_wide(arow, 2 * ks + (lane >> 4)));
      if constexpr (kNtS == 1) {
        uint32_t b0, b1;
        const int ent = 8 * wi + (lane & 7);
        ldmatrix_x2(b0, b1, sV_base + off_wide(ent, 2 * ks + ((lane >> 3) & 1)));
        mma_f16_16816(acc[0], a, b0, b1);
      } else {
#pragma unroll
        for (int jj = 0; jj < kNtS; jj += 2) {
          uint32_t bb[4];
          const int ent = 8 * (wi * kNtS + jj + (lane >> 4)) + (lane & 7);
          ldmatrix_x4(bb, sV_base + off_wide(ent, 2 * ks + ((lane >> 3) & 1)));
          mma_f16_16816(acc[jj], a, bb[0], bb[1]);
          mma_f16_16816(acc[jj + 1], a, bb[2], bb[3]);
        }
      }
    }

    // ---- online softmax (log2 domain) ----
    const float cg = sC[16 * mt + g], cg8 = sC[16 * mt + g + 8];
    float mx = -INFINITY, mx8 = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kNtS; ++jj) {
      const int e0 = 8 * (wi * kNtS + jj) + 2 * tq;
      const bool v0 = sIdx[e0] >= 0, v1 = sIdx[e0 + 1] >= 0;
      acc[jj][0] = v0 ? acc[jj][0] * cg : -INFINITY;
      acc[jj][1] = v1 ? acc[jj][1] * cg : -INFINITY;
      acc[jj][2] = v0 ? acc[jj][2] * cg8 : -INFINITY;
      acc[jj][3] = v1 ? acc[jj][3] * cg8 : -INFINITY;
      mx = fmaxf(mx, fmaxf(acc[jj][0], acc[jj][1]));
      mx8 = fmaxf(mx8, fmaxf(acc[jj][2], acc[jj][3]));
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx8 = fmaxf(mx8, __shfl_xor_sync(0xffffffffu, mx8, 1));
    mx8 = fmaxf(mx8, __shfl_xor_sync(0xffffffffu, mx8, 2));
    if (tq == 0) {
      sRed[warp * 16 + g] = mx;
      sRed[warp * 16 + g + 8] = mx8;
    }
    __syncthreads();
    float tmax = -INFINITY, tmax8 = -INFINITY;
#pragma unroll
    for (int k = 0; k < kWarpsPerMt; ++k) {
      tmax = fmaxf(tmax, sRed[(k * MT + mt) * 16 + g]);
      tmax8 = fmaxf(tmax8, sRed[(k * MT + mt) * 16 + g + 8]);
    }
    const float mn = fmaxf(m_g, tmax), mn8 = fmaxf(m_g8, tmax8);
    const float al = mn == -INFINITY ? 1.0f : exp2f(m_g - mn);
    const float al8 = mn8 == -INFINITY ? 1.0f : exp2f(m_g8 - mn8);
    m_g = mn;
    m_g8 = mn8;
    float ps = 0.0f, ps8 = 0.0f;
#pragma unroll
    for (int jj = 0; jj < kNtS; ++jj) {
      const float p0 = mn == -INFINITY ? 0.0f : exp2f(acc[jj][0] - mn);
      const float p1 = mn == -INFINITY ? 0.0f : exp2f(acc[jj][1] - mn);
      const float p2 = mn8 == -INFINITY ? 0.0f : exp2f(acc[jj][2] - mn8);
      const float p3 = mn8 == -INFINITY ? 0.0f : exp2f(acc[jj][3] - mn8);
      ps += p0 + p1;
      ps8 += p2 + p3;
      const int e0 = 8 * (wi * kNtS + jj) + 2 * tq;
      const float s0 = p0 * kPScale, s1 = p1 * kPScale, s2 = p2 * kPScale, s3 = p3 * kPScale;
      const uint32_t h01 = pack_f16x2(s0, s1), h23 = pack_f16x2(s2, s3);
      const uint32_t l01 = pack_f16x2(s0 - f16_lo_to_f32(h01), s1 - f16_hi_to_f32(h01));
      const uint32_t l23 = pack_f16x2(s2 - f16_lo_to_f32(h23), s3 - f16_hi_to_f32(h23));
      const int r0 = 16 * mt + g, r8 = r0 + 8, cc = e0 >> 3, within = (e0 & 7) * 2;
      *reinterpret_cast<uint32_t*>(sPh + off_narrow(r0, cc) + within) = h01;
      *reinterpret_cast<uint32_t*>(sPh + off_narrow(r8, cc) + within) = h23;
      *reinterpret_cast<uint32_t*>(sPl + off_narrow(r0, cc) + within) = l01;
      *reinterpret_cast<uint32_t*>(sPl + off_narrow(r8, cc) + within) = l23;
    }
    l_g = l_g * al + ps;
    l_g8 = l_g8 * al8 + ps8;
#pragma unroll
    for (int i = 0; i < kNtO; ++i) {
      o[i][0] *= al;
      o[i][1] *= al;
      o[i][2] *= al8;
      o[i][3] *= al8;
    }
    __syncthreads();  // P complete

    // ---- O += P V for (m-tile mt, dims [dim0, dim0 + 8*kNtO)) ----
    const uint32_t sPh_base = smem_u32(sPh), sPl_base = smem_u32(sPl);
#pragma unroll
    for (int ks = 0; ks < kSub / 16; ++ks) {
      uint32_t ah[4], alo[4];
      ldmatrix_x4(ah, sPh_base + off_narrow(arow, 2 * ks + (lane >> 4)));
      ldmatrix_x4(alo, sPl_base + off_narrow(arow, 2 * ks + (lane >> 4)));
      const int ent = 16 * ks + 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
      for (int np = 0; np < kNtO / 2; ++np) {
        uint32_t bb[4];
        ldmatrix_x4_trans(bb, sV_base + off_wide(ent, (dim0 >> 3) + 2 * np + (lane >> 4)));
        mma_f16_16816(o[2 * np], ah, bb[0], bb[1]);
        mma_f16_16816(o[2 * np], alo, bb[0], bb[1]);
        mma_f16_16816(o[2 * np + 1], ah, bb[2], bb[3]);
        mma_f16_16816(o[2 * np + 1], alo, bb[2], bb[3]);
      }
    }
  }

  // ---- per-head sums across the warps of an m-tile ----
  l_g += __shfl_xor_sync(0xffffffffu, l_g, 1);
  l_g += __shfl_xor_sync(0xffffffffu, l_g, 2);
  l_g8 += __shfl_xor_sync(0xffffffffu, l_g8, 1);
  l_g8 += __shfl_xor_sync(0xffffffffu, l_g8, 2);
  __syncthreads();
  if (tq == 0) {
    sRed[warp * 16 + g] = l_g;
    sRed[warp * 16 + g + 8] = l_g8;
  }
  __syncthreads();
  float L = 0.0f, L8 = 0.0f;
#pragma unroll
  for (int k = 0; k < kWarpsPerMt; ++k) {
    L += sRed[(k * MT + mt) * 16 + g];
    L8 += sRed[(k * MT + mt) * 16 + g + 8];
  }
  const int h0 = 16 * mt + g, h8 = h0 + 8;

  if (n_chunks == 1) {
    const float inv = L > 0.0f ? 1.0f / (kPScale * L) : 0.0f;
    const float inv8 = L8 > 0.0f ? 1.0f / (kPScale * L8) : 0.0f;
#pragma unroll
    for (int i = 0; i < kNtO; ++i) {
      const int dim = dim0 + 8 * i + 2 * tq;
      if (h0 < nh)
        *reinterpret_cast<float2*>(p.out + (int64_t(b) * p.H + hbase + h0) * kD + dim) =
            make_float2(o[i][0] * inv, o[i][1] * inv);
      if (h8 < nh)
        *reinterpret_cast<float2*>(p.out + (int64_t(b) * p.H + hbase + h8) * kD + dim) =
            make_float2(o[i][2] * inv8, o[i][3] * inv8);
    }
    if (p.lse != nullptr && wi == 0 && tq == 0) {
      if (h0 < nh) p.lse[int64_t(b) * p.H + hbase + h0] = L > 0.0f ? m_g * kLn2 + logf(L) : -INFINITY;
      if (h8 < nh) p.lse[int64_t(b) * p.H + hbase + h8] = L8 > 0.0f ? m_g8 * kLn2 + logf(L8) : -INFINITY;
    }
    return;
  }

  // ---- split: write this chunk's unnormalised partial; k_attn_combine merges them ----
  const int64_t part = (int64_t(b) * n_hg + hg) * n_chunks + chunk;
  float* po = p.part_o + part * kHeadsPerCta * kD;
  float* pml = p.part_ml + part * kHeadsPerCta * 2;
#pragma unroll
  for (int i = 0; i < kNtO; ++i) {
    const int dim = dim0 + 8 * i + 2 * tq;
    *reinterpret_cast<float2*>(po + h0 * kD + dim) = make_float2(o[i][0], o[i][1]);
    *reinterpret_cast<float2*>(po + h8 * kD + dim) = make_float2(o[i][2], o[i][3]);
  }
  if (wi == 0 && tq == 0) {
    pml[2 * h0] = m_g;
    pml[2 * h0 + 1] = L;
    pml[2 * h8] = m_g8;
    pml[2 * h8 + 1] = L8;
  }
}

// Merge of the chunk partials (log-sum-exp combine): grid (8 head blocks, head groups, B),
// one warp per head, each lane 16 of the 512 dims.
__global__ void __launch_bounds__(256) k_attn_combine(const AttnParams p, int n_hg) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hg = blockIdx.y, b = blockIdx.z;
  const int hh = blockIdx.x * 8 + warp;
  const int nh = min(kHeadsPerCta, p.H - hg * kHeadsPerCta);
  if (hh >= nh) return;
  const int n_chunks = p.n_chunks;
  const float* pml0 = p.part_ml + (int64_t(b) * n_hg + hg) * n_chunks * kHeadsPerCta * 2;
  const float* po0 = p.part_o + (int64_t(b) * n_hg + hg) * n_chunks * kHeadsPerCta * kD;
  float M = -INFINITY;
  for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, pml0[(int64_t(c) * kHeadsPerCta + hh) * 2]);
  float Lt = 0.0f;
  float4 acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c = 0; c < n_chunks; ++c) {
    const float mc = pml0[(int64_t(c) * kHeadsPerCta + hh) * 2];
    const float lc = pml0[(int64_t(c) * kHeadsPerCta + hh) * 2 + 1];
    if (!(lc > 0.0f)) continue;
    const float wgt = exp2f(mc - M);
    Lt += lc * wgt;
    const float4* src = reinterpret_cast<const float4*>(po0 + (int64_t(c) * kHeadsPerCta + hh) * kD) + 4 * lane;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 v = src[u];
      acc[u].x += wgt * v.x; acc[u].y += wgt * v.y; acc[u].z += wgt * v.z; acc[u].w += wgt * v.w;
    }
  }
  const float inv = Lt > 0.0f ? 1.0f / (kPScale * Lt) : 0.0f;
  float4* dst = reinterpret_cast<float4*>(p.out + (int64_t(b) * p.H + hg * kHeadsPerCta + hh) * kD) + 4 * lane;
#pragma unroll
  for (int u = 0; u < 4; ++u)
    dst[u] = make_float4(acc[u].x * inv, acc[u].y * inv, acc[u].z * inv, acc[u].w * inv);
  if (p.lse != nullptr && lane == 0)
    p.lse[int64_t(b) * p.H + hg * kHeadsPerCta + hh] = Lt > 0.0f ? M * kLn2 + logf(Lt) : -INFINITY;
}

template <int MT>
cudaError_t launch_mt(const AttnParams& p, int n_hg, cudaStream_t stream) {
  auto kern = k_sparse_attn<MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemAttn));
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_chunks, n_hg, p.B);
  kern<<<grid, kAttnThreads, kSmemAttn, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.n_chunks == 1) return e;
  k_attn_combine<<<dim3(kHeadsPerCta / 8, n_hg, p.B), 256, 0, stream>>>(p, n_hg);
  return cudaGetLastError();
}

}  // namespace

int attn_chunks(int B, int H, int top_k, int num_sms) {
  const int n_hg = (H + kHeadsPerCta - 1) / kHeadsPerCta;
  int c = num_sms / (B * n_hg);
  const int max_c = top_k / 128;
  if (c > max_c) c = max_c;
  if (c < 1) c = 1;
  return c;
}

cudaError_t launch_sparse_attn(const AttnParams& p, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  if (p.B == 0) return cudaSuccess;
  const int n_hg = (p.H + kHeadsPerCta - 1) / kHeadsPerCta;
  const int heads = p.H < kHeadsPerCta ? p.H : kHeadsPerCta;
  if (heads <= 16) return launch_mt<1>(p, n_hg, stream);
  if (heads <= 32) return launch_mt<2>(p, n_hg, stream);
  return launch_mt<4>(p, n_hg, stream);
}

}  // namespace fp4kv
