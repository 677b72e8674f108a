/*
 * libfp4kv -- decode-time sparse attention over a global KV cache stored as FP4.
 *
 * C ABI of the library. Every call takes plain pointers and sizes; no call allocates device
 * memory, synchronises, or aborts. Kernels are enqueued on the caller's CUDA stream
 * (`stream` is a cudaStream_t; NULL means the legacy default stream). All tensor pointers
 * are DEVICE pointers owned by the caller unless a comment says otherwise; the library keeps
 * no pointer after a call returns.
 *
 * Method sources (web pages about DeepSeek-V4.1-Flash):
 *  [PyTorchKR]  discuss.pytorch.kr, "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로
 *               줄이고 플래그십 V4-Pro를 대체하는 552B 규모의 MoE 모델"
 *               - section "890바이트를 만든 나머지 절반, FP4 KV 캐시와 지속 캐시 재설계":
 *                 main KV stored as E2M1 values with one E4M3 scale per 16 channels (NVFP4
 *                 without its second-level global scale), largest magnitude 448 x 6 = 2688,
 *                 used for storage only and dequantized before attention;
 *               - section "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2": the Full / Reindex /
 *                 Reuse mode table (who computes the main KV, the indexer K and the top-K
 *                 indices), 32 indexer query heads of dimension 128, attention top-K;
 *               - section "계층적 희소 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기": the
 *                 first Full decoder layer scores every visible position, gives each block of
 *                 8 positions its largest score and keeps the best blocks as a candidate
 *                 pool; later Reindex layers score only inside the pool.
 *  [ingu627]    ingu627 blog on DeepSeek V4.1-Flash-1017, section "3. KV 캐시 압축: HBM
 *               890바이트와 SSD 8분의 1 바운디드 리플레이" (FP4 KV quantization,
 *               index_topk) and section "MoE 라우팅과 하드웨어 병목의 분리 매칭" (64 query
 *               heads sharing a single KV head).
 *
 * Readings where the pages are silent (fixed by this library):
 *  - scale S = E4M3(amax / 6) with round-to-nearest-even, saturating at 448; codes
 *    E2M1(|x| / S) round-to-nearest-even, saturating at 6, with the sign bit of x kept
 *    (a negative value rounding to zero is stored as 0x8); an all-zero group has S = 0;
 *  - two codes per byte, even channel in the low nibble; one scale byte per 16 channels;
 *  - indexer score[n] = ks[n] * sum_h w[h] * max(0, q[h] . k[n]) in fp32 (ks = 1 when no
 *    key scale is given);
 *  - top-K by (score descending, position ascending); indices are written in ascending
 *    position order and padded with -1;
 *  - attention: o[h] = sum_j softmax_j(sm_scale * q[h] . v_j) v_j with v_j the dequantized
 *    row (one latent row is both key and value); lse[h] = natural log of the softmax
 *    denominator plus the max logit.
 *
 * Cache layout (batch-major, two planes, rows padded to the capacity `cap`):
 *    packed [B][cap][d/2]   uint8, E2M1 codes
 *    scales [B][cap][d/16]  uint8, E4M3 codes
 *    keys   [B][cap][128]   uint8 E4M3 codes, or uint16 bf16 bits
 * Position n of sequence b is row b*cap + n. Positions n >= seq_lens[b] are not visible.
 *
 * Inputs must be finite. NaN or Inf in any input gives undefined (but memory-safe)
 * results.
 */
#ifndef FP4KV_H_
#define FP4KV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP4KV_OK = 0,
  FP4KV_ERR_INVALID_ARG = 1,         /* null pointer, negative size, misaligned pointer  */
  FP4KV_ERR_UNSUPPORTED = 2,         /* a size outside the supported range                */
  FP4KV_ERR_CUDA = 3,                /* a launch or runtime call failed (see last_error) */
  FP4KV_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below fp4kv_workspace_bytes(...)         */
  FP4KV_ERR_DEVICE_FLAG = 5          /* a kernel reported a timed-out wait (status word)  */
} fp4kv_status;

/* Indexer query / key formats. FP4KV_KEY_E2M1 is the FP4 indexer format ([PyTorchKR] FP4
 * KV section: the indexer query and key were already FP4): each 128-dim vector is 64
 * bytes of E2M1 codes (two per byte, even dim in the low nibble) plus 8 E4M3 scales (one
 * per 16 dims), as fp4kv_kv_quant_fp4 with d = 128 writes them. The q and keys buffers
 * each hold two planes back to back: all codes [B][rows][64], then all scales
 * [B][rows][8] (rows = H_I for q, cap for keys). Needs an even H_I and an even cap. */
typedef enum { FP4KV_KEY_BF16 = 0, FP4KV_KEY_E4M3 = 1, FP4KV_KEY_E2M1 = 2 } fp4kv_key_dtype;

typedef enum {
  FP4KV_OP_KV_QUANT = 0,
  FP4KV_OP_INDEXER_TOPK = 1,     /* flat (pool == NULL) */
  FP4KV_OP_REINDEX_TOPK = 2,     /* fp4kv_indexer_topk with a pool */
  FP4KV_OP_HIER_POOL_SELECT = 3,
  FP4KV_OP_SPARSE_ATTN = 4,
  FP4KV_OP_INDEXER_SCORES = 5
} fp4kv_op;

/* Supported ranges (anything else returns FP4KV_ERR_UNSUPPORTED):
 *   d % 32 == 0 and 32 <= d <= 1024 (attention: d == 512);   indexer key dim == 128;
 *   1 <= H_I <= 64;   1 <= top_k <= 4096;   1 <= H <= 128;   1 <= block_size, and
 *   block_size == 8 for the pool;   1 <= n_pool_blocks <= 4096;   1 <= B <= 65535.       */

/* Text of the last error raised on the calling thread ("" after a successful call). */
const char* fp4kv_last_error(void);
/* Library version string (static storage). */
const char* fp4kv_version(void);

/* Bytes of scratch `ws` that an op needs for the given sizes. `heads` is H for
 * FP4KV_OP_SPARSE_ATTN and H_I for the indexer ops; unused arguments are ignored.
 * Returns 0 for ops that need no workspace or for unsupported sizes. */
size_t fp4kv_workspace_bytes(int32_t op, int32_t B, int64_t cap, int32_t heads, int32_t top_k,
                             int32_t n_pool_blocks);

/* Zero a workspace before its first use (enqueued on `stream`). Kernels leave the
 * workspace zeroed again when they finish, so it can be reused by later calls on the same
 * stream and captured in CUDA graphs; calls that share one workspace must not overlap. */
fp4kv_status fp4kv_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Device status word of a workspace: bit 0 set if a kernel gave up on a bounded wait.
 * Enqueues an async copy of the word into *host_status (pinned or pageable host memory)
 * and synchronises `stream`; then clears the word. For tests and diagnostics. */
fp4kv_status fp4kv_workspace_status(void* ws, uint32_t* host_status, void* stream);

/* selftest_wait_timeout -- (The pages have no counterpart: a test hook.) Launches one
 * small kernel that waits on an mbarrier nothing ever signals, bounded by limit_us
 * microseconds (1 .. 1,000,000), so that the bounded-wait error path every kernel of the
 * library uses can be exercised without faulting the device: when the bound runs out the
 * kernel sets bit 0 of the workspace status word and returns, leaving the context usable.
 * Read the word with fp4kv_workspace_status (which then returns FP4KV_ERR_DEVICE_FLAG).
 * ws: any workspace of at least 256 bytes (only its status word is touched).
 * INVALID_ARG for a null ws, a smaller ws_bytes or limit_us outside the range. */
fp4kv_status fp4kv_selftest_wait_timeout(int32_t limit_us, void* ws, size_t ws_bytes, void* stream);

/* kv_quant_fp4 -- quantize-on-write ([PyTorchKR] FP4 KV section).
 * x        : bf16 rows [n_rows][x_row_stride] (uint16 bits); d channels used per row.
 *            16-byte aligned, x_row_stride a multiple of 8.
 * dst_row  : nullable int64 [n_rows]; input row i is written to cache row dst_row[i]
 *            (e.g. b*cap + position). NULL writes row i to row i. Entries outside
 *            [0, cap_rows) are skipped.
 * packed   : [cap_rows][d/2] uint8, 16-byte aligned.   scales : [cap_rows][d/16] uint8.
 * Per group of 16 channels: S = E4M3_RNE_sat(amax/6); codes = sign | E2M1_RNE_sat(|x|/S). */
fp4kv_status fp4kv_kv_quant_fp4(const uint16_t* x, int64_t n_rows, int32_t d, int64_t x_row_stride,
                                const int64_t* dst_row, uint8_t* packed, uint8_t* scales,
                                int64_t cap_rows, void* stream);

/* indexer_scores -- Full-mode scoring of every visible entry, no selection
 * ([PyTorchKR] CSA2 section: the indexer scores all causally visible positions).
 * q         : [B][H_I][128] E4M3 codes (key_dtype E4M3) or bf16 bits (key_dtype BF16), or
 *             the two E2M1 planes (key_dtype E2M1, see fp4kv_key_dtype).
 * w         : fp32 [B][H_I] head weights (any query scale folded in).
 * keys      : [B][cap][128], same dtype as q (E2M1: the two planes). 16-byte aligned.
 * key_scale : nullable fp32 [B][cap] per-entry key scale ks.
 * seq_lens  : int32 [B] (device); seq_lens[b] <= cap. Entries n >= seq_lens[b] are not
 *             scored and out_score[b][n] is left unwritten for them.
 * out_score : fp32 [B][cap].
 * ws        : at least fp4kv_workspace_bytes(FP4KV_OP_INDEXER_SCORES, ...) (a status word). */
fp4kv_status fp4kv_indexer_scores(const void* q, const float* w, int32_t H_I, const void* keys,
                                  int32_t key_dtype, const float* key_scale, int64_t cap,
                                  const int32_t* seq_lens, int32_t B, float* out_score,
                                  void* ws, size_t ws_bytes, void* stream);

/* indexer_topk -- Full mode (pool == NULL): exact top-K over every visible entry.
 * Reindex mode (pool != NULL): score only the positions of the pool's blocks
 * (block j covers positions [j*block_size, (j+1)*block_size) clipped to seq_len; ids < 0
 * are skipped; ids must be distinct) with this layer's own query, then top-K among them
 * ([PyTorchKR] CSA2 mode table, Reindex row; hierarchical indexer section).
 * pool      : nullable int32 [B][n_pool_blocks].
 * out_idx   : int32 [B][top_k], positions in ascending order, padded with -1.
 * out_score : nullable fp32 [B][top_k], the score of each chosen position (-inf for pads).
 * ws        : at least fp4kv_workspace_bytes(FP4KV_OP_INDEXER_TOPK or _REINDEX_TOPK, ...),
 *             zeroed once by fp4kv_workspace_init. */
fp4kv_status fp4kv_indexer_topk(const void* q, const float* w, int32_t H_I, const void* keys,
                                int32_t key_dtype, const float* key_scale, int64_t cap,
                                const int32_t* seq_lens, int32_t B, const int32_t* pool,
                                int32_t n_pool_blocks, int32_t block_size, int32_t top_k,
                                int32_t* out_idx, float* out_score, void* ws, size_t ws_bytes,
                                void* stream);

/* hier_pool_select -- the first Full-mode decoder layer of the hierarchical sparse indexer
 * ([PyTorchKR] hierarchical indexer section): one scan that yields the flat top-K AND the
 * candidate pool, i.e. the n_pool_blocks blocks of block_size positions with the largest
 * block max score (ties: lower block id), as block ids in ascending order padded with -1.
 * out_pool : int32 [B][n_pool_blocks]. Other arguments as fp4kv_indexer_topk. */
fp4kv_status fp4kv_hier_pool_select(const void* q, const float* w, int32_t H_I, const void* keys,
                                    int32_t key_dtype, const float* key_scale, int64_t cap,
                                    const int32_t* seq_lens, int32_t B, int32_t top_k,
                                    int32_t block_size, int32_t n_pool_blocks, int32_t* out_idx,
                                    int32_t* out_pool, float* out_score, void* ws,
                                    size_t ws_bytes, void* stream);

/* sparse_attn_decode -- gather the selected rows, dequantize them (E2M1 x E4M3, exact) and
 * run softmax attention for every query head ([PyTorchKR] FP4 KV section: dequantized
 * before attention; [ingu627]: 64 query heads over one shared KV head).
 * Reuse mode is this call with the previous layer's idx ([PyTorchKR] CSA2 mode table).
 * q        : bf16 bits [B][H][d], 16-byte aligned.   d == 512.
 * packed, scales : the cache planes (see layout above), both 16-byte aligned here.
 * idx      : int32 [B][top_k]; entries < 0 or >= seq_lens[b] are skipped; duplicates count.
 * out      : fp32 [B][H][d].   lse : nullable fp32 [B][H] (-inf when no entry is valid,
 *            in which case out is 0).
 * ws       : at least fp4kv_workspace_bytes(FP4KV_OP_SPARSE_ATTN, B, cap, H, top_k, 0),
 *            zeroed once by fp4kv_workspace_init. */
fp4kv_status fp4kv_sparse_attn_decode(const uint16_t* q, int32_t B, int32_t H, int32_t d,
                                      const uint8_t* packed, const uint8_t* scales, int64_t cap,
                                      const int32_t* seq_lens, const int32_t* idx, int32_t top_k,
                                      float sm_scale, float* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream);

/* sparse_swa_attn_decode -- fp4kv_sparse_attn_decode plus the sliding-window branch
 * ([PyTorchKR] "왜 KV 캐시가 에이전트 시대의 병목이 되었나": a global branch over the main KV
 * and a sliding-window (SWA) branch over a local KV of the last n_win tokens; FP4 KV
 * section: the SWA KV stays FP8). The window's rows join the selected rows in ONE softmax
 * (this library's reading of how the two branches combine): out = sum over the selected
 * entries and the window rows of softmax(sm_scale * q . v) * v, lse over both sets.
 * swa   : E4M3 codes [B][n_win][d] (fp4kv_swa_quant_fp8 writes them), 16-byte aligned; a ring
 *         buffer: position pos lives in slot pos % n_win, and slots [0, min(n_win,
 *         seq_lens[b])) are the window of sequence b (the caller keeps them current).
 * n_win : 1 .. 128. Other arguments and the workspace as fp4kv_sparse_attn_decode.
 * Positions that are both selected and in the window count twice. */
fp4kv_status fp4kv_sparse_swa_attn_decode(const uint16_t* q, int32_t B, int32_t H, int32_t d,
                                          const uint8_t* packed, const uint8_t* scales, int64_t cap,
                                          const int32_t* seq_lens, const int32_t* idx, int32_t top_k,
                                          const uint8_t* swa, int32_t n_win, float sm_scale, float* out,
                                          float* lse, void* ws, size_t ws_bytes, void* stream);

/* topk_merge -- context-sharded decode (no counterpart on the pages: several GPUs split every
 * sequence's positions into contiguous ranges; part r holds positions [part_base[r], ...) and
 * runs fp4kv_indexer_topk over its own range with out_score). This call merges the gathered
 * per-part lists exactly: out_idx[b] = the top_k of the union of the candidates by score
 * descending, then position ascending, as global positions in ascending order, padded with
 * -1. The union contains the global top-K (a position among the best K of the whole context
 * is among the best K of its range, ties being broken by position in both), so the result
 * equals the indexer top-K of the whole context.
 * cand_score fp32 / cand_idx int32 [n_parts][B][k_part]: each part's out_score / out_idx
 *            (range-local positions, -1 absent), as an all-gather lays them out;
 * part_base  HOST int32 [n_parts], >= 0;   1 <= n_parts <= 64, n_parts * k_part <= 16384;
 *            k_part >= top_k (each part keeps top_k candidates, padded with -1 when its
 *            range is shorter; fewer could drop a global winner, so k_part < top_k is
 *            rejected with FP4KV_ERR_UNSUPPORTED);
 * out_local  nullable int32 [B][top_k]: the selection as positions local to
 *            [local_lo, local_hi), -1 elsewhere (what this part's attention needs);
 * out_score  nullable fp32 [B][top_k] (-inf for pads). 1 <= top_k <= 4096. */
fp4kv_status fp4kv_topk_merge(const float* cand_score, const int32_t* cand_idx, int32_t n_parts, int32_t k_part,
                              int32_t B, const int32_t* part_base, int32_t top_k, int32_t local_lo,
                              int32_t local_hi, int32_t* out_idx, int32_t* out_local, float* out_score,
                              void* stream);

/* lse_combine -- context-sharded decode: joins attention partials computed over disjoint
 * row sets (each range's fp4kv_sparse_attn_decode over the selected positions it holds).
 * part_out fp32 [n_parts][B][H][d], part_lse fp32 [n_parts][B][H] (-inf: the part had no
 * row). out[b][h] = sum_r w_r part_out[r][b][h] / sum_r w_r with w_r = e^(lse_r - max_r lse_r);
 * lse (nullable) = max + ln(sum w_r), -inf (and out = 0) when every part is empty.
 * 1 <= n_parts <= 1024, H <= 128, d <= 1024. */
fp4kv_status fp4kv_lse_combine(const float* part_out, const float* part_lse, int32_t n_parts, int32_t B, int32_t H,
                               int32_t d, float* out, float* lse, void* stream);

/* swa_quant_fp8 -- the SWA KV's write: bf16 rows x [n_rows][d] (row stride x_row_stride
 * elements, a multiple of 8) to E4M3 codes, round to nearest even, saturating at +-448
 * ([PyTorchKR] FP4 KV section: the quantization-sensitive SWA KV stays FP8; a direct cast
 * without a scale is this library's reading). out: [cap_rows][d] bytes; row i goes to
 * dst_row[i] (nullable: i), rows outside [0, cap_rows) are skipped. d % 16 == 0, d <= 1024;
 * x and out 16-byte aligned. */
fp4kv_status fp4kv_swa_quant_fp8(const uint16_t* x, int64_t n_rows, int32_t d, int64_t x_row_stride,
                                 const int64_t* dst_row, uint8_t* out, int64_t cap_rows, void* stream);

/* indexer_topk_noalloc -- fp4kv_indexer_topk without a caller workspace. (The pages have
 * no counterpart: this is an integration aid.) For callers that cannot allocate device
 * memory: code inside a host runtime that owns all device memory (a serving engine with a
 * fixed pre-reserved pool, a plugin interface without an allocator), or latency-critical
 * decode loops that cannot afford cudaMalloc's implicit device-wide synchronisation.
 * Arguments and results are those of fp4kv_indexer_topk minus ws / ws_bytes. The scratch is
 * a file-scope device array of 8 MiB that every GPU loading the library keeps until the
 * process exits; sizes whose workspace (fp4kv_workspace_bytes of the same op) exceeds 8 MiB
 * return FP4KV_ERR_UNSUPPORTED with an explanatory message. The call allocates nothing: it
 * clears the scratch's counters with cudaMemsetAsync on `stream` and launches the same
 * kernels as fp4kv_indexer_topk. The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current) and caches it for the device's
 * current context (a device reset makes a new context, and the next call looks it up again);
 * make that first call before any stream capture. All calls on a device share the one
 * array, so calls whose kernels overlap on the GPU (different streams, or different host
 * threads) race and give wrong results: serialise them. A kernel whose bounded wait gave up
 * sets bit 0 of the scratch's status word; the word keeps it across later calls until
 * fp4kv_noalloc_status reads it. */
fp4kv_status fp4kv_indexer_topk_noalloc(const void* q, const float* w, int32_t H_I,
                                        const void* keys, int32_t key_dtype,
                                        const float* key_scale, int64_t cap,
                                        const int32_t* seq_lens, int32_t B, const int32_t* pool,
                                        int32_t n_pool_blocks, int32_t block_size, int32_t top_k,
                                        int32_t* out_idx, float* out_score, void* stream);

/* noalloc_status -- the status word of the scratch that fp4kv_indexer_topk_noalloc uses on
 * the current device (no counterpart on the pages; the allocation-free counterpart of
 * fp4kv_workspace_status): copies it into *host_status, waits for `stream`, then clears it.
 * Returns FP4KV_ERR_DEVICE_FLAG if it was non-zero (bit 0: a kernel's bounded wait gave up,
 * so the results of the calls since the last read are not to be trusted). Synchronising
 * diagnostic; allocates nothing. */
fp4kv_status fp4kv_noalloc_status(uint32_t* host_status, void* stream);

/* selftest_wait_timeout_noalloc -- fp4kv_selftest_wait_timeout on the scratch of
 * fp4kv_indexer_topk_noalloc (a test hook, no counterpart on the pages): the status bit
 * lands in the word that fp4kv_noalloc_status reads. */
fp4kv_status fp4kv_selftest_wait_timeout_noalloc(int32_t limit_us, void* stream);

/* Benchmark support (no counterpart on the pages). While enabled, every kernel the library
 * launches is bracketed by two CUDA events recorded on the launch stream (do not enable
 * during CUDA-graph capture). fp4kv_profile_read waits for the recorded events and returns,
 * per kernel kind [0 kv_quant, 1 indexer scoring, 2 top-K select, 3 sparse attention], the
 * number of launches and their summed device time in milliseconds (host arrays of 4), then
 * clears the records. */
fp4kv_status fp4kv_profile_enable(int32_t on);
fp4kv_status fp4kv_profile_read(int32_t* launches, float* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* FP4KV_H_ */
