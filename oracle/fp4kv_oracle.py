"""Plain CPU oracle for decode-time sparse attention over an FP4 KV cache.

TEST INFRASTRUCTURE ONLY. This module is the slow, obviously correct statement of what the
GPU library computes. Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it. The product path (the ``libfp4kv`` shared library and
its Python binding) never imports, links or calls anything here, and this module shares no
code, table or helper with the CUDA sources.

Arithmetic is fp64 unless a step is defined in another precision (the indexer score and
the top-K ordering are fp32 by definition). Rounding decisions are taken by enumerating
the representable values of the target format, so each step can be checked by eye.

Sources (web pages about DeepSeek-V4.1-Flash):

* [PyTorchKR] "DeepSeek-V4.1-Flash, KV 캐시를 토큰당 890바이트로 줄이고 플래그십 V4-Pro를
  대체하는 552B 규모의 MoE 모델" (discuss.pytorch.kr), sections
    - "레이어 사이에서 캐시와 인덱스를 돌려 쓰는 CSA2" (CSA2: the Full / Reindex / Reuse
      mode table, the indexer shape of 32 query heads x 128 dims, attention top-K),
    - "계층적 희소 인덱서로 인덱싱 비용을 컨텍스트 길이에서 분리하기" (hierarchical sparse
      indexer: block max over 8 positions, candidate pool, Reindex inside the pool),
    - "890바이트를 만든 나머지 절반, FP4 KV 캐시와 지속 캐시 재설계" (FP4 main-KV: E2M1
      values with one E4M3 scale per 16 channels, max 448 x 6 = 2688, dequantized
      before attention).
* [ingu627] DeepSeek V4.1-Flash-1017 blog post (ingu627), section "3. KV 캐시 압축: HBM
  890바이트와 SSD 8분의 1 바운디드 리플레이" (FP4 KV quantization, index_topk) and section
  "MoE 라우팅과 하드웨어 병목의 분리 매칭" (64 attention heads sharing one KV head).

Readings where the pages are silent (each is listed in the design notes):

* scale = E4M3(amax / 6), round-to-nearest-even on the code, saturating at 448;
* E2M1 codes round-to-nearest-even on the code, saturating at 6; the sign of x is kept,
  so a negative value that rounds to zero is stored as 0x8;
* two codes per byte, the even channel in the low nibble; scales one byte per group;
* indexer score = ks[n] * sum_h w_h * max(0, q_h . k_n), rounded to fp32; with FP4
  indexer operands, q and k are first stored with the main KV's quantizer;
* top-K by (fp32 score descending, index ascending), output in ascending index order,
  padded with -1;
* attention: softmax(sm_scale * q . v_hat) . v_hat, one latent row serving as K and V.
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------------------
# Number formats  ([PyTorchKR] FP4 main-KV section: E2M1 values + one E4M3 scale per 16
# channels; the format's largest magnitude is 448 * 6 = 2688).
# ----------------------------------------------------------------------------------------

GROUP = 16  # channels per E4M3 scale


def e4m3_decode(code) -> np.ndarray:
    """E4M3 ("FN" flavour: no infinities, 0x7F/0xFF are NaN) code -> value, fp64.

    Bit layout s eeee mmm, exponent bias 7. Exponent field 0 is subnormal: m/8 * 2^-6.
    Otherwise (1 + m/8) * 2^(e-7). The largest finite value is 0x7E = 448.
    """
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


# Non-negative finite E4M3 values, indexed by code 0..126 (monotone increasing).
E4M3_POS_VALUES = e4m3_decode(np.arange(127))
E4M3_MAX = float(E4M3_POS_VALUES[126])  # 448

# E2M1 magnitudes, indexed by the 3-bit magnitude code; bit 3 of a nibble is the sign.
E2M1_POS_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MAX = 6.0


def e2m1_decode(code) -> np.ndarray:
    """4-bit E2M1 code -> value (fp64). Bit 3 is the sign, bits 0..2 index the magnitudes."""
    c = np.asarray(code, dtype=np.int64)
    mag = E2M1_POS_VALUES[c & 7]
    return np.where((c >> 3) & 1 == 1, -mag, mag)


def _nearest_code_even_ties(v: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to each v >= 0; a tie goes to the even index.

    ``grid`` is increasing, and consecutive indices are consecutive codes of the format, so
    "even index" is "even code" (round-to-nearest-even). Values beyond the last grid point
    map to the last index (saturation), since the last point is then the nearest.
    """
    v = np.asarray(v, dtype=np.float64)
    flat = v.reshape(-1)
    out = np.empty(flat.shape, dtype=np.int64)
    chunk = max(1, (1 << 22) // len(grid))
    for s in range(0, flat.size, chunk):
        # beyond the last grid point the last point is the nearest (saturation); clamping
        # first keeps |x - grid| meaningful for huge x
        x = np.minimum(flat[s:s + chunk], grid[-1])
        d = np.abs(x[:, None] - grid[None, :])
        first = np.argmin(d, axis=1)  # lowest index among the minima
        dmin = d[np.arange(x.size), first]
        nxt = np.minimum(first + 1, len(grid) - 1)
        tie = (nxt != first) & (d[np.arange(x.size), nxt] == dmin)
        out[s:s + chunk] = np.where(tie & (first % 2 == 1), nxt, first)
    return out.reshape(v.shape)


def e4m3_round_sat(v) -> np.ndarray:
    """Non-negative value -> E4M3 code: nearest representable, ties to the even code, and
    anything above 448 becomes 448 (code 0x7E)."""
    v = np.asarray(v, dtype=np.float64)
    assert np.all(v >= 0), "scale rounding is only defined for non-negative values"
    return _nearest_code_even_ties(v, E4M3_POS_VALUES)


def e2m1_mag_round_sat(r) -> np.ndarray:
    """Non-negative ratio r = |x| / S -> 3-bit E2M1 magnitude code: nearest grid value,
    ties to the even code, r > 6 -> 6."""
    return _nearest_code_even_ties(np.asarray(r, dtype=np.float64), E2M1_POS_VALUES)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------------------
# Quantize-on-write and dequantize  ([PyTorchKR] FP4 main-KV section; [ingu627] section 3,
# "FP4 KV 양자화": keys/values stored as E2M1 with one E4M3 scale per 16 channels).
# ----------------------------------------------------------------------------------------

def kv_quant_fp4(x) -> tuple[np.ndarray, np.ndarray]:
    """Quantize rows x [R, d] (exact bf16 values, given as fp64) into
    packed [R, d/2] uint8 (two E2M1 codes per byte, even channel in the low nibble) and
    scales [R, d/16] uint8 (E4M3 codes, one per 16-channel group, channel order).

    Per group: amax = max |x|; S = E4M3_RNE_sat(amax / 6); for each x,
    code = signbit(x) << 3 | E2M1_RNE_sat(|x| / S), or just the sign bit when S == 0.
    """
    x = np.asarray(x, dtype=np.float64)
    R, d = x.shape
    assert d % GROUP == 0 and d % 2 == 0
    g = x.reshape(R, d // GROUP, GROUP)
    amax = np.abs(g).max(axis=2)
    s_code = e4m3_round_sat(amax / 6.0)
    S = E4M3_POS_VALUES[s_code]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(S[..., None] > 0, np.abs(g) / np.where(S > 0, S, 1.0)[..., None], 0.0)
    mag = e2m1_mag_round_sat(r)
    mag = np.where(S[..., None] > 0, mag, 0)
    sign = np.signbit(g).astype(np.int64)
    codes = (sign << 3) | mag
    codes = codes.reshape(R, d)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, s_code.astype(np.uint8)


def kv_dequant_fp4(packed, scales) -> np.ndarray:
    """packed [R, d/2] + scales [R, d/16] -> v_hat [R, d] fp64, v_hat = e2m1(code) * e4m3(S).
    ([PyTorchKR] FP4 main-KV section: the cache is dequantized before attention.)"""
    packed = np.asarray(packed, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    R, half = packed.shape
    d = 2 * half
    codes = np.empty((R, d), dtype=np.int64)
    codes[:, 0::2] = packed & 0xF
    codes[:, 1::2] = packed >> 4
    vals = e2m1_decode(codes)
    S = e4m3_decode(scales)
    return (vals.reshape(R, d // GROUP, GROUP) * S[..., None]).reshape(R, d)


def packed_row_bytes(d: int) -> int:
    """Bytes one cached row of d channels occupies: d/2 bytes of codes + d/16 scale bytes."""
    return d // 2 + d // GROUP


# ----------------------------------------------------------------------------------------
# Indexer and top-K  ([PyTorchKR] CSA2 section: indexer query heads 32 x head dim 128,
# attention top-K; the indexer K is projected from the main KV).
# ----------------------------------------------------------------------------------------

def indexer_scores(q, w, keys, key_scale=None) -> np.ndarray:
    """score[n] = fp32( ks[n] * sum_h w[h] * max(0, sum_c q[h, c] * keys[n, c]) ).

    q [H_I, Dk], w [H_I], keys [N, Dk] are exact values (decoded FP8 / bf16) as fp64; the
    sum is evaluated in fp64 and rounded once to fp32.
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    dots = keys @ q.T  # [N, H_I]
    s = np.maximum(dots, 0.0) @ w
    if key_scale is not None:
        s = s * np.asarray(key_scale, dtype=np.float64)
    return s.astype(np.float32)


def indexer_fp4_values(x) -> np.ndarray:
    """FP4 indexer operand ([PyTorchKR] FP4 main-KV section: DeepSeek-V4 already kept the
    indexer query and key in FP4): the values 128-dim query or key rows x [R, 128] (exact
    bf16 values as fp64) hold once stored as E2M1 codes with one E4M3 scale per 16 dims,
    quantized exactly as the main KV is. Scores of FP4 operands are indexer_scores of these
    values."""
    return kv_dequant_fp4(*kv_quant_fp4(x))


def topk_positions(scores, positions, top_k: int) -> np.ndarray:
    """Exact top-K of (scores[i], positions[i]) by score descending, position ascending on
    equal scores. Returns the chosen positions in ascending order, padded with -1 to
    top_k. Scores are compared as fp32 (-0.0 equals +0.0)."""
    s = np.asarray(scores, dtype=np.float32).astype(np.float64)
    p = np.asarray(positions, dtype=np.int64)
    order = np.lexsort((p, -s))  # primary: -score ascending; secondary: position ascending
    take = np.sort(p[order[:min(top_k, p.size)]])
    out = np.full(top_k, -1, dtype=np.int64)
    out[:take.size] = take
    return out


def indexer_topk(q, w, keys, seq_len: int, top_k: int, key_scale=None):
    """Full mode: score every causally visible entry n < seq_len and keep the top-K.
    Returns (idx [top_k] ascending padded -1, scores [seq_len] fp32)."""
    ks = None if key_scale is None else np.asarray(key_scale)[:seq_len]
    sc = indexer_scores(q, w, np.asarray(keys)[:seq_len], ks)
    return topk_positions(sc, np.arange(seq_len), top_k), sc


def block_max(scores, seq_len: int, block_size: int) -> np.ndarray:
    """Bmax[j] = max fp32 score over positions [j*bs, (j+1)*bs) that are < seq_len.
    ([PyTorchKR] hierarchical indexer section: each block gets its largest index score.)"""
    s = np.asarray(scores, dtype=np.float32)[:seq_len]
    nb = -(-seq_len // block_size)
    pad = np.full(nb * block_size, -np.inf, dtype=np.float32)
    pad[:seq_len] = s
    return pad.reshape(nb, block_size).max(axis=1)


def pool_select(scores, seq_len: int, block_size: int, n_pool_blocks: int) -> np.ndarray:
    """Candidate pool: the n_pool_blocks blocks with the largest Bmax (ties: lower block
    id), as block ids in ascending order, padded with -1."""
    bm = block_max(scores, seq_len, block_size)
    return topk_positions(bm, np.arange(bm.size), n_pool_blocks)


def hier_pool_select(q, w, keys, seq_len: int, top_k: int, block_size: int,
                     n_pool_blocks: int, key_scale=None):
    """First Full-mode decoder layer: flat top-K over all entries AND the block pool.
    Returns (idx [top_k], pool [n_pool_blocks], scores [seq_len])."""
    idx, sc = indexer_topk(q, w, keys, seq_len, top_k, key_scale)
    return idx, pool_select(sc, seq_len, block_size, n_pool_blocks), sc


def pool_positions(pool, seq_len: int, block_size: int) -> np.ndarray:
    """Positions covered by the pool's blocks (ids < 0 skipped), clipped to seq_len,
    in the order the blocks are listed."""
    out = []
    for j in np.asarray(pool, dtype=np.int64):
        if j < 0:
            continue
        lo, hi = int(j) * block_size, min((int(j) + 1) * block_size, seq_len)
        out.extend(range(lo, hi))
    return np.asarray(out, dtype=np.int64)


def reindex_topk(q, w, keys, seq_len: int, pool, block_size: int, top_k: int,
                 key_scale=None):
    """Reindex mode: score only the pool's positions with this layer's own query and keep
    the top-K among them ([PyTorchKR] CSA2 mode table, Reindex row; hierarchical indexer
    section). Returns (idx [top_k] ascending padded -1, positions, scores at positions)."""
    pos = pool_positions(pool, seq_len, block_size)
    keys = np.asarray(keys)
    ks = None if key_scale is None else np.asarray(key_scale)[pos]
    sc = indexer_scores(q, w, keys[pos], ks) if pos.size else np.zeros(0, np.float32)
    return topk_positions(sc, pos, top_k), pos, sc


# ----------------------------------------------------------------------------------------
# Sparse attention over the selected rows  ([PyTorchKR] FP4 main-KV section: dequantize
# then attend; [ingu627] "MoE 라우팅과 하드웨어 병목의 분리 매칭": 64 query heads, 1 KV head).
# ----------------------------------------------------------------------------------------

def sparse_attn_decode(q, packed, scales, idx, seq_len: int, sm_scale: float):
    """One sequence. q [H, d] exact (bf16 values as fp64); packed [cap, d/2]; scales
    [cap, d/16]; idx [K] (entries < 0 or >= seq_len skipped, duplicates counted).

    For each head: z_j = sm_scale * q . v_hat_j, m = max z, o = sum e^(z-m) v_hat / sum
    e^(z-m), lse = m + ln sum e^(z-m). No valid entry: o = 0, lse = -inf.
    Returns (out [H, d] fp64, lse [H] fp64).
    """
    q = np.asarray(q, dtype=np.float64)
    H, d = q.shape
    idx = np.asarray(idx, dtype=np.int64)
    sel = idx[(idx >= 0) & (idx < seq_len)]
    if sel.size == 0:
        return np.zeros((H, d)), np.full(H, -np.inf)
    v = kv_dequant_fp4(np.asarray(packed)[sel], np.asarray(scales)[sel])  # [J, d]
    return sparse_attn_decode_rows(q, v, sm_scale)


def sparse_attn_decode_rows(q, v_hat, sm_scale: float):
    """Softmax attention of every head of q [H, d] over already dequantized rows v_hat
    [J, d] (J >= 1, fp64): z = sm_scale * q . v_hat_j, m = max_j z, o = sum e^(z-m) v_hat /
    sum e^(z-m), lse = m + ln sum e^(z-m). ``sparse_attn_decode`` calls this after it has
    gathered and dequantized the selected rows. Returns (out [H, d], lse [H])."""
    q = np.asarray(q, dtype=np.float64)
    v = np.asarray(v_hat, dtype=np.float64)
    z = sm_scale * (q @ v.T)  # [H, J]
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    den = e.sum(axis=1, keepdims=True)
    return (e @ v) / den, m[:, 0] + np.log(den[:, 0])


def swa_quant_fp8(x) -> np.ndarray:
    """The sliding-window KV's storage ([PyTorchKR] FP4 KV section: the SWA KV stays FP8):
    each value as an E4M3 code, nearest value with ties to the even code, saturating at
    448, the sign of x kept (a negative value that rounds to zero is 0x80). x: exact bf16
    values as fp64, any shape; returns uint8 codes of the same shape."""
    x = np.asarray(x, dtype=np.float64)
    mag = e4m3_round_sat(np.abs(x))
    return ((np.signbit(x).astype(np.int64) << 7) | mag).astype(np.uint8)


def sparse_swa_attn_decode_rows(q, v_sel, v_win, sm_scale: float):
    """Attention of the sparse branch and the sliding-window branch in one softmax: the
    selected rows v_sel [J, d] and the window rows v_win [W, d] (dequantized values) are
    attended together, as one set of J + W rows. Returns (o [H, d], lse [H])."""
    v_sel = np.asarray(v_sel, dtype=np.float64).reshape(-1, np.asarray(q).shape[-1])
    v_win = np.asarray(v_win, dtype=np.float64).reshape(-1, np.asarray(q).shape[-1])
    return sparse_attn_decode_rows(q, np.concatenate([v_sel, v_win], axis=0), sm_scale)


def attn_lse_merge(outs, lses):
    """Attention over the union of disjoint row sets from the attentions over each set:
    outs [R, H, d], lses [R, H] (-inf for an empty set). out = sum_r e^(lse_r - M) out_r /
    sum_r e^(lse_r - M), lse = M + ln(sum); (0, -inf) when every set is empty. (Follows from
    writing each set's softmax numerator and denominator with its lse.)"""
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    m = lses.max(axis=0)
    with np.errstate(invalid="ignore"):
        wts = np.where(np.isneginf(lses), 0.0, np.exp(lses - np.where(np.isneginf(m), 0.0, m)))
    den = wts.sum(axis=0)
    out = np.where(den[:, None] > 0, (wts[..., None] * outs).sum(axis=0) / np.where(den > 0, den, 1.0)[:, None], 0.0)
    lse = np.where(den > 0, m + np.log(np.where(den > 0, den, 1.0)), -np.inf)
    return out, lse


def fp8_e4m3_to_f64(codes) -> np.ndarray:
    """FP8 E4M3 indexer keys / queries (uint8 codes) -> exact fp64 values."""
    return e4m3_decode(np.asarray(codes, dtype=np.uint8))


def global_kv_bytes_per_token(entries_per_token: float, d: int, indexer_key_bytes: int) -> float:
    """Bytes of global KV per token for a cache holding ``entries_per_token`` compressed
    entries per token, each one FP4 row of d channels plus one indexer key."""
    return entries_per_token * (packed_row_bytes(d) + indexer_key_bytes)


__all__ = [name for name in dir() if not name.startswith("_") and name not in ("math", "np")]
del math
