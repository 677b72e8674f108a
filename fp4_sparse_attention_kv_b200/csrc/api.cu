// C ABI of libfp4kv: argument validation, workspace layout and kernel dispatch.
// The declarations, argument meaning, layouts and error behaviour are documented in
// include/fp4kv.h. Nothing here allocates device memory or synchronises (except
// fp4kv_workspace_status, a diagnostic call documented as synchronising).
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "fp4kv.h"
#include "fp4kv_common.cuh"
#include "fp4kv_launch.h"
#include "fp4kv_sm100.cuh"

namespace {

thread_local std::string g_last_error;

fp4kv_status fail(fp4kv_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

fp4kv_status ok() {
  g_last_error.clear();
  return FP4KV_OK;
}

fp4kv_status cuda_fail(cudaError_t e, const char* where) {
  return fail(FP4KV_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// ---------------------------------------------------------------------------------------
// Optional per-kernel timing for benchmarks: launches bracketed by CUDA events.
// ---------------------------------------------------------------------------------------
namespace prof {
constexpr int kKinds = 4;  // 0 kv_quant, 1 indexer scoring, 2 top-K select, 3 sparse attention
struct Rec {
  int kind;
  cudaEvent_t a, b;
};
std::mutex mu;
bool enabled = false;
std::vector<Rec> recs;
std::vector<cudaEvent_t> pool;

cudaEvent_t take() {
  if (!pool.empty()) {
    cudaEvent_t e = pool.back();
    pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

struct Scope {
  int kind;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  Scope(int k, cudaStream_t st) : kind(k), s(st) {
    std::lock_guard<std::mutex> g(mu);
    if (!enabled) return;
    a = take();
    if (a) cudaEventRecord(a, s);
  }
  ~Scope() {
    if (!a) return;
    std::lock_guard<std::mutex> g(mu);
    cudaEvent_t b = take();
    if (!b) return;
    cudaEventRecord(b, s);
    recs.push_back({kind, a, b});
  }
};
}  // namespace prof

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ---------------------------------------------------------------------------------------
// Workspace layouts
// ---------------------------------------------------------------------------------------
struct IndexerLayout {
  size_t status = 0, scores = 0, gmax = 0, bmax = 0, hist = 0, hist_end = 0, list = 0;
  size_t total = 0;
  int64_t score_stride = 0, gmax_stride = 0, bmax_stride = 0;
  int n_probs = 0;
  int64_t k[2] = {0, 0};
  int64_t vstride[2] = {0, 0};
};

// kind: 0 flat top-K, 1 reindex top-K, 2 hierarchical (top-K + pool), 3 scores only
IndexerLayout indexer_layout(int kind, int64_t B, int64_t cap, int64_t top_k, int64_t npb) {
  IndexerLayout L;
  size_t off = kAlign;  // status header
  L.score_stride = (kind == 1) ? npb * 8 : (cap + 7) / 8 * 8;
  L.scores = off;
  off += up(sizeof(float) * B * L.score_stride);
  if (kind != 3) {  // the largest key of every 32 scores
    L.gmax_stride = ((L.score_stride + 31) / 32 + 7) / 8 * 8;
    L.gmax = off;
    off += up(sizeof(uint32_t) * B * L.gmax_stride);
  }
  if (kind == 2) {
    L.bmax_stride = ((cap + 7) / 8 + 7) / 8 * 8;
    L.bmax = off;
    off += up(sizeof(float) * B * L.bmax_stride);
  }
  if (kind == 3) {
    L.n_probs = 0;
    L.total = kAlign;  // status word only; the scores go to the caller's buffer
    return L;
  }
  L.n_probs = kind == 2 ? 2 : 1;
  L.k[0] = top_k;
  L.vstride[0] = L.score_stride;
  if (kind == 2) {
    L.k[1] = npb;
    L.vstride[1] = L.bmax_stride;
  }
  // the first-digit histograms: the region that must start at zero (the select leaves it so)
  L.hist = off;
  off += up(sizeof(uint32_t) * L.n_probs * B * fp4kv::kHistBins);
  L.hist_end = off;
  L.list = off;
  for (int i = 0; i < L.n_probs; ++i) off += up(sizeof(uint64_t) * B * L.vstride[i]);
  L.total = off;
  return L;
}

struct AttnLayout {
  size_t part_ml = 0, part_o = 0, total = 0;
  int n_chunks = 1, n_hg = 1;
};

// The chunk partials the attention's CTAs exchange (sized for the largest chunk count the
// launch may use for these sizes; it never uses more).
AttnLayout attn_layout(int64_t B, int64_t H, int64_t top_k, int sms) {
  AttnLayout L;
  L.n_hg = static_cast<int>((H + 63) / 64);
  L.n_chunks = fp4kv::attn_chunks(static_cast<int>(B), static_cast<int>(H), static_cast<int>(top_k), sms);
  size_t off = kAlign;
  L.part_ml = off;
  off += up(sizeof(float) * B * L.n_hg * L.n_chunks * 64 * 2);
  L.part_o = off;
  off += up(sizeof(float) * B * L.n_hg * L.n_chunks * 64 * 512);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------------------------------
// Shared validation of the indexer query / key arguments
// ---------------------------------------------------------------------------------------
fp4kv_status check_indexer_args(const void* q, const float* w, int32_t H_I, const void* keys,
                                int32_t key_dtype, int64_t cap, const int32_t* seq_lens,
                                int32_t B) {
  if (!q || !w || !keys || !seq_lens) return fail(FP4KV_ERR_INVALID_ARG, "null q, w, keys or seq_lens");
  if (B < 1 || B > 65535) return fail(FP4KV_ERR_UNSUPPORTED, "B=%d outside [1, 65535]", B);
  if (H_I < 1 || H_I > 64) return fail(FP4KV_ERR_UNSUPPORTED, "H_I=%d outside [1, 64]", H_I);
  if (cap < 1 || cap > (int64_t(1) << 31) - 8)
    return fail(FP4KV_ERR_UNSUPPORTED, "cap=%lld outside [1, 2^31 - 8]", (long long)cap);
  if (int64_t(B) * cap > (int64_t(1) << 31) - 256)
    return fail(FP4KV_ERR_UNSUPPORTED, "B*cap=%lld must stay below 2^31 rows", (long long)(int64_t(B) * cap));
  if (key_dtype != FP4KV_KEY_BF16 && key_dtype != FP4KV_KEY_E4M3 && key_dtype != FP4KV_KEY_E2M1)
    return fail(FP4KV_ERR_UNSUPPORTED, "key_dtype=%d", key_dtype);
  if (key_dtype == FP4KV_KEY_E2M1 && ((H_I & 1) || (cap & 1)))
    return fail(FP4KV_ERR_UNSUPPORTED, "E2M1 keys need an even H_I and cap (H_I=%d, cap=%lld)", H_I,
                (long long)cap);
  if (!aligned(q, 16) || !aligned(keys, 16) || !aligned(w, 4))
    return fail(FP4KV_ERR_INVALID_ARG, "q and keys must be 16-byte aligned");
  return FP4KV_OK;
}

fp4kv::IndexScoreParams score_params(const void* q, const float* w, int32_t H_I, const void* keys,
                                     int32_t key_dtype, const float* key_scale, int64_t cap,
                                     const int32_t* seq_lens, int32_t B, uint32_t* status) {
  fp4kv::IndexScoreParams p{};
  p.q = q;
  p.w = w;
  p.H_I = H_I;
  p.keys = keys;
  p.key_type = key_dtype;  // the kernel's numbering follows fp4kv_key_dtype
  if (key_dtype == FP4KV_KEY_E2M1) {
    // two planes back to back: codes [rows][64], then scales [rows][8]
    p.key_sf = static_cast<const uint8_t*>(keys) + int64_t(B) * cap * 64;
    p.q_sf = static_cast<const uint8_t*>(q) + int64_t(B) * H_I * 64;
  }
  p.key_scale = key_scale;
  p.cap = cap;
  p.seq_lens = seq_lens;
  p.B = B;
  p.status = status;
  return p;
}

}  // namespace

// Test hook: waits on an mbarrier that nothing ever signals, bounded by limit_ns, then
// reports the timeout in the status word exactly as the library's kernels do.
__global__ void k_selftest_wait(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    fp4kv::mbar_init(&bar, 1);
    fp4kv::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = fp4kv::globaltimer_ns();
    bool done = false;
    while (!(done = fp4kv::mbar_try_wait(&bar, 0)) && fp4kv::globaltimer_ns() - t0 <= limit_ns) {
    }
    if (!done) atomicOr(status, fp4kv::kFlagWaitTimeout);
  }
}

extern "C" {

const char* fp4kv_last_error(void) { return g_last_error.c_str(); }

const char* fp4kv_version(void) { return "libfp4kv 0.1 (sm_100a)"; }

size_t fp4kv_workspace_bytes(int32_t op, int32_t B, int64_t cap, int32_t heads, int32_t top_k,
                             int32_t n_pool_blocks) {
  if (B < 1 || cap < 1) return 0;
  switch (op) {
    case FP4KV_OP_KV_QUANT:
      return 0;
    case FP4KV_OP_INDEXER_TOPK:
      return indexer_layout(0, B, cap, top_k, n_pool_blocks).total;
    case FP4KV_OP_REINDEX_TOPK:
      return indexer_layout(1, B, cap, top_k, n_pool_blocks).total;
    case FP4KV_OP_HIER_POOL_SELECT:
      return indexer_layout(2, B, cap, top_k, n_pool_blocks).total;
    case FP4KV_OP_SPARSE_ATTN:
      if (heads < 1 || top_k < 1) return 0;
      return attn_layout(B, heads, top_k, num_sms()).total;
    case FP4KV_OP_INDEXER_SCORES:
      return indexer_layout(3, B, cap, top_k, n_pool_blocks).total;
    default:
      return 0;
  }
}

fp4kv_status fp4kv_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws && ws_bytes) return fail(FP4KV_ERR_INVALID_ARG, "null workspace");
  if (ws_bytes == 0) return ok();
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "workspace_init");
  return ok();
}

fp4kv_status fp4kv_selftest_wait_timeout(int32_t limit_us, void* ws, size_t ws_bytes, void* stream) {
  if (!ws) return fail(FP4KV_ERR_INVALID_ARG, "null workspace");
  if (ws_bytes < kAlign) return fail(FP4KV_ERR_INVALID_ARG, "ws_bytes %zu < %zu", ws_bytes, kAlign);
  if (limit_us < 1 || limit_us > 1000000)
    return fail(FP4KV_ERR_INVALID_ARG, "limit_us=%d outside [1, 1000000]", limit_us);
  k_selftest_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(ws),
                                                                    uint64_t(limit_us) * 1000u);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest_wait_timeout");
  return ok();
}

fp4kv_status fp4kv_workspace_status(void* ws, uint32_t* host_status, void* stream) {
  if (!ws || !host_status) return fail(FP4KV_ERR_INVALID_ARG, "null workspace or host_status");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(host_status, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "workspace_status");
  return *host_status ? fail(FP4KV_ERR_DEVICE_FLAG, "device status word 0x%x", *host_status) : ok();
}

fp4kv_status fp4kv_kv_quant_fp4(const uint16_t* x, int64_t n_rows, int32_t d, int64_t x_row_stride,
                                const int64_t* dst_row, uint8_t* packed, uint8_t* scales,
                                int64_t cap_rows, void* stream) {
  if (n_rows < 0 || cap_rows < 0) return fail(FP4KV_ERR_INVALID_ARG, "negative n_rows or cap_rows");
  if (d % 32 != 0 || d < 32 || d > 1024) return fail(FP4KV_ERR_UNSUPPORTED, "d=%d must be a multiple of 32 in [32, 1024]", d);
  if (n_rows == 0) return ok();
  if (!x || !packed || !scales) return fail(FP4KV_ERR_INVALID_ARG, "null x, packed or scales");
  if (x_row_stride < d || x_row_stride % 8 != 0)
    return fail(FP4KV_ERR_INVALID_ARG, "x_row_stride=%lld must be >= d and a multiple of 8", (long long)x_row_stride);
  if (!aligned(x, 16) || !aligned(packed, 8))
    return fail(FP4KV_ERR_INVALID_ARG, "x must be 16-byte and packed 8-byte aligned");
  if (!dst_row && n_rows > cap_rows) return fail(FP4KV_ERR_INVALID_ARG, "n_rows > cap_rows with dst_row == NULL");
  cudaError_t e;
  {
    prof::Scope ps(0, static_cast<cudaStream_t>(stream));
    e = fp4kv::launch_kv_quant_fp4(x, n_rows, d, x_row_stride, dst_row, packed, scales, cap_rows,
                                   num_sms(), static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "kv_quant_fp4");
  return ok();
}

fp4kv_status fp4kv_topk_merge(const float* cand_score, const int32_t* cand_idx, int32_t n_parts, int32_t k_part,
                              int32_t B, const int32_t* part_base, int32_t top_k, int32_t local_lo,
                              int32_t local_hi, int32_t* out_idx, int32_t* out_local, float* out_score,
                              void* stream) {
  if (!cand_score || !cand_idx || !part_base || !out_idx)
    return fail(FP4KV_ERR_INVALID_ARG, "null cand_score, cand_idx, part_base or out_idx");
  if (B < 1 || B > 65535) return fail(FP4KV_ERR_UNSUPPORTED, "B=%d outside [1, 65535]", B);
  if (n_parts < 1 || n_parts > fp4kv::kMaxShardParts)
    return fail(FP4KV_ERR_UNSUPPORTED, "n_parts=%d outside [1, %d]", n_parts, fp4kv::kMaxShardParts);
  if (k_part < 1 || int64_t(n_parts) * k_part > 16384)
    return fail(FP4KV_ERR_UNSUPPORTED, "n_parts * k_part = %lld outside [1, 16384]", (long long)n_parts * k_part);
  if (top_k < 1 || top_k > 4096) return fail(FP4KV_ERR_UNSUPPORTED, "top_k=%d outside [1, 4096]", top_k);
  if (k_part < top_k)
    return fail(FP4KV_ERR_UNSUPPORTED,
                "k_part=%d < top_k=%d: each part must keep top_k candidates for the merge to be exact",
                k_part, top_k);
  for (int r = 0; r < n_parts; ++r)
    if (part_base[r] < 0) return fail(FP4KV_ERR_INVALID_ARG, "part_base[%d] = %d < 0", r, part_base[r]);
  if (!aligned(cand_score, 4) || !aligned(cand_idx, 4) || !aligned(out_idx, 4) || !aligned(out_local, 4) ||
      !aligned(out_score, 4))
    return fail(FP4KV_ERR_INVALID_ARG, "misaligned argument (4 B)");
  cudaError_t e;
  {
    prof::Scope ps(2, static_cast<cudaStream_t>(stream));
    e = fp4kv::launch_topk_merge(cand_score, cand_idx, n_parts, k_part, part_base, B, top_k, local_lo, local_hi,
                                 out_idx, out_local, out_score, static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "topk_merge");
  return ok();
}

fp4kv_status fp4kv_lse_combine(const float* part_out, const float* part_lse, int32_t n_parts, int32_t B, int32_t H,
                               int32_t d, float* out, float* lse, void* stream) {
  if (!part_out || !part_lse || !out) return fail(FP4KV_ERR_INVALID_ARG, "null part_out, part_lse or out");
  if (n_parts < 1 || n_parts > 1024) return fail(FP4KV_ERR_UNSUPPORTED, "n_parts=%d outside [1, 1024]", n_parts);
  if (B < 1 || B > 65535 || H < 1 || H > 128 || d < 1 || d > 1024)
    return fail(FP4KV_ERR_UNSUPPORTED, "B=%d, H=%d or d=%d outside the supported range", B, H, d);
  if (!aligned(part_out, 4) || !aligned(part_lse, 4) || !aligned(out, 4) || !aligned(lse, 4))
    return fail(FP4KV_ERR_INVALID_ARG, "misaligned argument (4 B)");
  cudaError_t e;
  {
    prof::Scope ps(3, static_cast<cudaStream_t>(stream));
    e = fp4kv::launch_lse_combine(part_out, part_lse, n_parts, int64_t(B) * H, d, out, lse,
                                  static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "lse_combine");
  return ok();
}

fp4kv_status fp4kv_swa_quant_fp8(const uint16_t* x, int64_t n_rows, int32_t d, int64_t x_row_stride,
                                 const int64_t* dst_row, uint8_t* out, int64_t cap_rows, void* stream) {
  if (n_rows < 0 || cap_rows < 0) return fail(FP4KV_ERR_INVALID_ARG, "negative n_rows or cap_rows");
  if (d % 16 != 0 || d < 16 || d > 1024) return fail(FP4KV_ERR_UNSUPPORTED, "d=%d must be a multiple of 16 in [16, 1024]", d);
  if (n_rows == 0) return ok();
  if (!x || !out) return fail(FP4KV_ERR_INVALID_ARG, "null x or out");
  if (x_row_stride < d || x_row_stride % 8 != 0)
    return fail(FP4KV_ERR_INVALID_ARG, "x_row_stride=%lld must be >= d and a multiple of 8", (long long)x_row_stride);
  if (!aligned(x, 16) || !aligned(out, 16))
    return fail(FP4KV_ERR_INVALID_ARG, "x and out must be 16-byte aligned");
  if (!dst_row && n_rows > cap_rows) return fail(FP4KV_ERR_INVALID_ARG, "n_rows > cap_rows with dst_row == NULL");
  cudaError_t e;
  {
    prof::Scope ps(0, static_cast<cudaStream_t>(stream));
    e = fp4kv::launch_swa_quant_fp8(x, n_rows, d, x_row_stride, dst_row, out, cap_rows, num_sms(),
                                    static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "swa_quant_fp8");
  return ok();
}

fp4kv_status fp4kv_indexer_scores(const void* q, const float* w, int32_t H_I, const void* keys,
                                  int32_t key_dtype, const float* key_scale, int64_t cap,
                                  const int32_t* seq_lens, int32_t B, float* out_score,
                                  void* ws, size_t ws_bytes, void* stream) {
  fp4kv_status st = check_indexer_args(q, w, H_I, keys, key_dtype, cap, seq_lens, B);
  if (st != FP4KV_OK) return st;
  if (!out_score || !ws) return fail(FP4KV_ERR_INVALID_ARG, "null out_score or ws");
  const IndexerLayout L = indexer_layout(3, B, cap, 0, 0);
  if (ws_bytes < L.total) return fail(FP4KV_ERR_WORKSPACE_TOO_SMALL, "ws_bytes %zu < %zu", ws_bytes, L.total);
  uint8_t* base = static_cast<uint8_t*>(ws);
  fp4kv::IndexScoreParams p = score_params(q, w, H_I, keys, key_dtype, key_scale, cap, seq_lens, B,
                                           reinterpret_cast<uint32_t*>(base));
  p.scores = out_score;
  p.score_stride = cap;
  cudaError_t e;
  {
    prof::Scope ps(1, static_cast<cudaStream_t>(stream));
    e = fp4kv::launch_index_score(p, num_sms(), static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "indexer_scores");
  return ok();
}

static fp4kv_status run_indexer(int kind, const void* q, const float* w, int32_t H_I,
                                const void* keys, int32_t key_dtype, const float* key_scale,
                                int64_t cap, const int32_t* seq_lens, int32_t B,
                                const int32_t* pool, int32_t n_pool_blocks, int32_t top_k,
                                int32_t* out_idx, int32_t* out_pool, float* out_score,
                                void* ws, size_t ws_bytes, cudaStream_t stream) {
  const IndexerLayout L = indexer_layout(kind, B, cap, top_k, n_pool_blocks);
  if (!ws) return fail(FP4KV_ERR_INVALID_ARG, "null workspace");
  if (ws_bytes < L.total) return fail(FP4KV_ERR_WORKSPACE_TOO_SMALL, "ws_bytes %zu < %zu", ws_bytes, L.total);
  if (!aligned(ws, kAlign)) return fail(FP4KV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int sms = num_sms();
  fp4kv::IndexScoreParams p = score_params(q, w, H_I, keys, key_dtype, key_scale, cap, seq_lens, B,
                                           reinterpret_cast<uint32_t*>(base));
  p.scores = reinterpret_cast<float*>(base + L.scores);
  p.score_stride = L.score_stride;
  p.hist = reinterpret_cast<uint32_t*>(base + L.hist);
  p.gmax = reinterpret_cast<uint32_t*>(base + L.gmax);
  p.gmax_stride = L.gmax_stride;
  if (kind == 1) {
    p.pool = pool;
    p.npb = n_pool_blocks;
  }
  if (kind == 2) {
    p.bmax = reinterpret_cast<float*>(base + L.bmax);
    p.bmax_stride = L.bmax_stride;
    p.bmax_hist = p.hist + int64_t(B) * fp4kv::kHistBins;
  }
  cudaError_t e;
  {
    prof::Scope ps(1, stream);
    e = fp4kv::launch_index_score(p, sms, stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, "indexer scoring");

  fp4kv::SelectProblem probs[2];
  size_t list_off = L.list;
  for (int i = 0; i < L.n_probs; ++i) {
    fp4kv::SelectProblem& P = probs[i];
    P = fp4kv::SelectProblem{};
    P.values = (i == 0) ? p.scores : p.bmax;
    P.vstride = L.vstride[i];
    P.seq_lens = seq_lens;
    P.mode = (kind == 1) ? 2 : (i == 0 ? 0 : 1);
    P.pool = pool;
    P.npb = n_pool_blocks;
    P.k = static_cast<int>(L.k[i]);
    P.gmax = (i == 0) ? p.gmax : nullptr;
    P.gstride = L.gmax_stride;
    P.hist = p.hist + int64_t(i) * B * fp4kv::kHistBins;
    P.list = reinterpret_cast<uint64_t*>(base + list_off);
    list_off += up(sizeof(uint64_t) * B * L.vstride[i]);
    P.out_idx = (i == 0) ? out_idx : out_pool;
    P.out_score = (i == 0) ? out_score : nullptr;
    P.status = p.status;
  }
  {
    prof::Scope ps(2, stream);
    e = fp4kv::launch_topk_select(probs, L.n_probs, B, sms, stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, "top-k select");
  return ok();
}

fp4kv_status fp4kv_indexer_topk(const void* q, const float* w, int32_t H_I, const void* keys,
                                int32_t key_dtype, const float* key_scale, int64_t cap,
                                const int32_t* seq_lens, int32_t B, const int32_t* pool,
                                int32_t n_pool_blocks, int32_t block_size, int32_t top_k,
                                int32_t* out_idx, float* out_score, void* ws, size_t ws_bytes,
                                void* stream) {
  fp4kv_status st = check_indexer_args(q, w, H_I, keys, key_dtype, cap, seq_lens, B);
  if (st != FP4KV_OK) return st;
  if (!out_idx) return fail(FP4KV_ERR_INVALID_ARG, "null out_idx");
  if (top_k < 1 || top_k > 4096) return fail(FP4KV_ERR_UNSUPPORTED, "top_k=%d outside [1, 4096]", top_k);
  if (pool) {
    if (block_size != 8) return fail(FP4KV_ERR_UNSUPPORTED, "block_size=%d (only 8)", block_size);
    if (n_pool_blocks < 1 || n_pool_blocks > 4096)
      return fail(FP4KV_ERR_UNSUPPORTED, "n_pool_blocks=%d outside [1, 4096]", n_pool_blocks);
  }
  return run_indexer(pool ? 1 : 0, q, w, H_I, keys, key_dtype, key_scale, cap, seq_lens, B, pool,
                     pool ? n_pool_blocks : 0, top_k, out_idx, nullptr, out_score, ws, ws_bytes,
                     static_cast<cudaStream_t>(stream));
}

fp4kv_status fp4kv_hier_pool_select(const void* q, const float* w, int32_t H_I, const void* keys,
                                    int32_t key_dtype, const float* key_scale, int64_t cap,
                                    const int32_t* seq_lens, int32_t B, int32_t top_k,
                                    int32_t block_size, int32_t n_pool_blocks, int32_t* out_idx,
                                    int32_t* out_pool, float* out_score, void* ws,
                                    size_t ws_bytes, void* stream) {
  fp4kv_status st = check_indexer_args(q, w, H_I, keys, key_dtype, cap, seq_lens, B);
  if (st != FP4KV_OK) return st;
  if (!out_idx || !out_pool) return fail(FP4KV_ERR_INVALID_ARG, "null out_idx or out_pool");
  if (top_k < 1 || top_k > 4096) return fail(FP4KV_ERR_UNSUPPORTED, "top_k=%d outside [1, 4096]", top_k);
  if (block_size != 8) return fail(FP4KV_ERR_UNSUPPORTED, "block_size=%d (only 8)", block_size);
  if (n_pool_blocks < 1 || n_pool_blocks > 4096)
    return fail(FP4KV_ERR_UNSUPPORTED, "n_pool_blocks=%d outside [1, 4096]", n_pool_blocks);
  return run_indexer(2, q, w, H_I, keys, key_dtype, key_scale, cap, seq_lens, B, nullptr,
                     n_pool_blocks, top_k, out_idx, out_pool, out_score, ws, ws_bytes,
                     static_cast<cudaStream_t>(stream));
}

static fp4kv_status run_attn(const uint16_t* q, int32_t B, int32_t H, int32_t d, const uint8_t* packed,
                             const uint8_t* scales, int64_t cap, const int32_t* seq_lens,
                             const int32_t* idx, int32_t top_k, const uint8_t* swa, int32_t n_win,
                             float sm_scale, float* out, float* lse, void* ws, size_t ws_bytes,
                             void* stream) {
  if (!q || !packed || !scales || !seq_lens || !idx || !out || !ws)
    return fail(FP4KV_ERR_INVALID_ARG, "null pointer argument");
  if (B < 1 || B > 65535) return fail(FP4KV_ERR_UNSUPPORTED, "B=%d outside [1, 65535]", B);
  if (H < 1 || H > 128) return fail(FP4KV_ERR_UNSUPPORTED, "H=%d outside [1, 128]", H);
  if (d != 512) return fail(FP4KV_ERR_UNSUPPORTED, "d=%d (attention is built for d=512)", d);
  if (top_k < 1 || top_k > 4096) return fail(FP4KV_ERR_UNSUPPORTED, "top_k=%d outside [1, 4096]", top_k);
  if (cap < 1 || cap > (int64_t(1) << 31) - 8)
    return fail(FP4KV_ERR_UNSUPPORTED, "cap=%lld outside [1, 2^31 - 8]", (long long)cap);
  if (!aligned(q, 16) || !aligned(packed, 16) || !aligned(scales, 16) || !aligned(out, 8) ||
      !aligned(ws, kAlign))
    return fail(FP4KV_ERR_INVALID_ARG, "misaligned q/packed/scales (16 B), out (8 B) or ws (256 B)");
  const int sms = num_sms();
  const AttnLayout L = attn_layout(B, H, top_k, sms);
  if (ws_bytes < L.total) return fail(FP4KV_ERR_WORKSPACE_TOO_SMALL, "ws_bytes %zu < %zu", ws_bytes, L.total);
  uint8_t* base = static_cast<uint8_t*>(ws);
  fp4kv::AttnParams p{};
  p.q = q;
  p.B = B;
  p.H = H;
  p.d = d;
  p.packed = packed;
  p.scales = scales;
  p.cap = cap;
  p.seq_lens = seq_lens;
  p.idx = idx;
  p.top_k = top_k;
  p.swa = swa;
  p.n_win = n_win;
  p.sm_scale = sm_scale;
  p.out = out;
  p.lse = lse;
  p.n_chunks = L.n_chunks;
  p.part_ml = reinterpret_cast<float*>(base + L.part_ml);
  p.part_o = reinterpret_cast<float*>(base + L.part_o);
  p.status = reinterpret_cast<uint32_t*>(base);
  cudaError_t e;
  {
    prof::Scope ps(3, static_cast<cudaStream_t>(stream));
    e = fp4kv::launch_sparse_attn(p, sms, static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "sparse_attn_decode");
  return ok();
}

fp4kv_status fp4kv_sparse_attn_decode(const uint16_t* q, int32_t B, int32_t H, int32_t d,
                                      const uint8_t* packed, const uint8_t* scales, int64_t cap,
                                      const int32_t* seq_lens, const int32_t* idx, int32_t top_k,
                                      float sm_scale, float* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream) {
  return run_attn(q, B, H, d, packed, scales, cap, seq_lens, idx, top_k, nullptr, 0, sm_scale, out, lse,
                  ws, ws_bytes, stream);
}

fp4kv_status fp4kv_sparse_swa_attn_decode(const uint16_t* q, int32_t B, int32_t H, int32_t d,
                                          const uint8_t* packed, const uint8_t* scales, int64_t cap,
                                          const int32_t* seq_lens, const int32_t* idx, int32_t top_k,
                                          const uint8_t* swa, int32_t n_win, float sm_scale, float* out,
                                          float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!swa) return fail(FP4KV_ERR_INVALID_ARG, "null swa");
  if (n_win < 1 || n_win > 128) return fail(FP4KV_ERR_UNSUPPORTED, "n_win=%d outside [1, 128]", n_win);
  if (!aligned(swa, 16)) return fail(FP4KV_ERR_INVALID_ARG, "swa must be 16-byte aligned");
  return run_attn(q, B, H, d, packed, scales, cap, seq_lens, idx, top_k, swa, n_win, sm_scale, out, lse,
                  ws, ws_bytes, stream);
}

// ---------------------------------------------------------------------------------------
// Allocation-free variant of fp4kv_indexer_topk.
//
// Some callers cannot allocate device memory at all: code embedded in a host runtime that
// owns every byte of device memory (a serving engine with a fixed, pre-reserved pool, or a
// plugin interface that hands out no allocator), and latency-critical decode loops where
// cudaMalloc's implicit device-wide synchronisation is not acceptable. For them the
// scratch of the indexer top-K lives in this file-scope device array instead of a
// caller-provided workspace. Every GPU that loads the library holds these bytes until the
// process exits.
// ---------------------------------------------------------------------------------------
constexpr size_t kNoAllocBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_noalloc_ws[kNoAllocBytes];

namespace {
std::mutex g_noalloc_mu;
// per device ordinal: the context the address was looked up in, and the address
struct NoallocSlot {
  void* ctx = nullptr;
  void* ptr = nullptr;
};
NoallocSlot g_noalloc_slot[256];

// The driver's cuCtxGetCurrent through the runtime's entry-point query (no link against
// libcuda). The cached address of the scratch is only valid in the context it was looked
// up in: after a device reset the primary context is a new one and the lookup is redone.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_noalloc_ws on the current device, looked up with that device current
// on the first call in each context and cached. In host code the array's name is only a
// host-side stand-in, never a device address.
fp4kv_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_topk_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= 256) return fail(FP4KV_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  void* ctx = current_context();
  if (!slot.ptr || ctx == nullptr || ctx != slot.ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_ws);
    if (e != cudaSuccess || p == nullptr)
      return cuda_fail(e == cudaSuccess ? cudaErrorInvalidSymbol : e,
                       "indexer_topk_noalloc: cudaGetSymbolAddress");
    slot.ptr = p;
    slot.ctx = current_context();  // the lookup has made the device's context current
  }
  *out = slot.ptr;
  return FP4KV_OK;
}
}  // namespace

fp4kv_status fp4kv_indexer_topk_noalloc(const void* q, const float* w, int32_t H_I,
                                        const void* keys, int32_t key_dtype,
                                        const float* key_scale, int64_t cap,
                                        const int32_t* seq_lens, int32_t B, const int32_t* pool,
                                        int32_t n_pool_blocks, int32_t block_size, int32_t top_k,
                                        int32_t* out_idx, float* out_score, void* stream) {
  fp4kv_status st = check_indexer_args(q, w, H_I, keys, key_dtype, cap, seq_lens, B);
  if (st != FP4KV_OK) return st;
  if (!out_idx) return fail(FP4KV_ERR_INVALID_ARG, "null out_idx");
  if (top_k < 1 || top_k > 4096) return fail(FP4KV_ERR_UNSUPPORTED, "top_k=%d outside [1, 4096]", top_k);
  if (pool) {
    if (block_size != 8) return fail(FP4KV_ERR_UNSUPPORTED, "block_size=%d (only 8)", block_size);
    if (n_pool_blocks < 1 || n_pool_blocks > 4096)
      return fail(FP4KV_ERR_UNSUPPORTED, "n_pool_blocks=%d outside [1, 4096]", n_pool_blocks);
  }
  const int kind = pool ? 1 : 0;
  const IndexerLayout L = indexer_layout(kind, B, cap, top_k, pool ? n_pool_blocks : 0);
  if (L.total > kNoAllocBytes)
    return fail(FP4KV_ERR_UNSUPPORTED,
                "indexer_topk_noalloc: these sizes need %zu bytes of scratch, above the built-in "
                "maximum of %zu (use fp4kv_indexer_topk with a caller workspace)",
                L.total, kNoAllocBytes);
  void* ws = nullptr;
  st = noalloc_scratch(&ws);
  if (st != FP4KV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the histograms must start at zero. The status word at the head is left
  // as it is: a bounded wait that gave up in an earlier call stays visible until
  // fp4kv_noalloc_status reads (and clears) it.
  cudaError_t e = cudaMemsetAsync(static_cast<uint8_t*>(ws) + L.hist, 0, L.hist_end - L.hist, s);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_topk_noalloc: clearing scratch");
  return run_indexer(kind, q, w, H_I, keys, key_dtype, key_scale, cap, seq_lens, B, pool,
                     pool ? n_pool_blocks : 0, top_k, out_idx, nullptr, out_score, ws, L.total, s);
}

fp4kv_status fp4kv_noalloc_status(uint32_t* host_status, void* stream) {
  if (!host_status) return fail(FP4KV_ERR_INVALID_ARG, "null host_status");
  void* ws = nullptr;
  fp4kv_status st = noalloc_scratch(&ws);
  if (st != FP4KV_OK) return st;
  return fp4kv_workspace_status(ws, host_status, stream);
}

fp4kv_status fp4kv_selftest_wait_timeout_noalloc(int32_t limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000)
    return fail(FP4KV_ERR_INVALID_ARG, "limit_us=%d outside [1, 1000000]", limit_us);
  void* ws = nullptr;
  fp4kv_status st = noalloc_scratch(&ws);
  if (st != FP4KV_OK) return st;
  return fp4kv_selftest_wait_timeout(limit_us, ws, kNoAllocBytes, stream);
}

fp4kv_status fp4kv_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> g(prof::mu);
  prof::enabled = on != 0;
  return ok();
}

fp4kv_status fp4kv_profile_read(int32_t* launches, float* total_ms) {
  if (!launches || !total_ms) return fail(FP4KV_ERR_INVALID_ARG, "null output arrays");
  std::vector<prof::Rec> recs;
  {
    std::lock_guard<std::mutex> g(prof::mu);
    recs.swap(prof::recs);
  }
  for (int k = 0; k < prof::kKinds; ++k) {
    launches[k] = 0;
    total_ms[k] = 0.0f;
  }
  cudaError_t err = cudaSuccess;
  for (const prof::Rec& r : recs) {
    float ms = 0.0f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) {
      err = e;
    } else if (r.kind >= 0 && r.kind < prof::kKinds) {
      launches[r.kind] += 1;
      total_ms[r.kind] += ms;
    }
  }
  {
    std::lock_guard<std::mutex> g(prof::mu);
    for (const prof::Rec& r : recs) {
      prof::pool.push_back(r.a);
      prof::pool.push_back(r.b);
    }
  }
  if (err != cudaSuccess) return cuda_fail(err, "profile_read");
  return ok();
}

}  // extern "C"
