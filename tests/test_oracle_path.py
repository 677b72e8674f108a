"""Pins for the oracle's indexer, top-K, candidate pool and sparse attention (CPU only).

Checked against brute force written as plain Python loops on tiny inputs, against dense
softmax attention, and against invariants the method fixes (pool = all blocks makes
Reindex the flat top-K; K = 1 returns the selected row; equal logits average the rows).
"""
import math

import numpy as np
import pytest

from oracle import fp4kv_oracle as O


def _brute_scores(q, w, keys, ks=None):
    out = []
    for n in range(len(keys)):
        tot = 0.0
        for h in range(len(q)):
            dot = math.fsum(float(q[h][c]) * float(keys[n][c]) for c in range(len(keys[n])))
            tot += float(w[h]) * max(0.0, dot)
        if ks is not None:
            tot *= float(ks[n])
        out.append(np.float32(tot))
    return np.array(out, dtype=np.float32)


def _brute_topk(scores, positions, k):
    """Repeatedly take the best remaining (largest score; lowest position on ties)."""
    left = list(zip([float(s) for s in scores], [int(p) for p in positions]))
    chosen = []
    for _ in range(min(k, len(left))):
        best = None
        for i, (s, p) in enumerate(left):
            if best is None or s > left[best][0] or (s == left[best][0] and p < left[best][1]):
                best = i
        chosen.append(left.pop(best)[1])
    chosen.sort()
    return chosen + [-1] * (k - len(chosen))


def test_indexer_single_head_is_a_dot_product():
    rng = np.random.default_rng(3)
    keys = np.abs(rng.standard_normal((20, 128)))
    q = np.abs(rng.standard_normal((1, 128)))
    s = O.indexer_scores(q, np.ones(1), keys)
    ref = [np.float32(math.fsum(q[0] * keys[n])) for n in range(20)]
    assert np.array_equal(s, np.array(ref, dtype=np.float32))


def test_indexer_matches_brute_force_nonsquare():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((3, 8))
    w = rng.uniform(-1, 2, 3)
    keys = rng.standard_normal((37, 8))
    ks = rng.uniform(0.5, 2, 37)
    assert np.array_equal(O.indexer_scores(q, w, keys, ks), _brute_scores(q, w, keys, ks))
    assert np.array_equal(O.indexer_scores(q, w, keys), _brute_scores(q, w, keys))


@pytest.mark.parametrize("k", [1, 5, 16, 40])
def test_topk_matches_brute_force_with_ties(k):
    rng = np.random.default_rng(5 + k)
    s = rng.integers(0, 6, 33).astype(np.float32)  # many equal scores
    s[3] = -0.0
    s[4] = 0.0
    pos = np.arange(33)
    assert O.topk_positions(s, pos, k).tolist() == _brute_topk(s, pos, k)
    perm = rng.permutation(200)[:33]  # arbitrary positions
    assert O.topk_positions(s, perm, k).tolist() == _brute_topk(s, perm, k)


def test_indexer_topk_end_to_end_brute_force():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((4, 16))
    w = rng.uniform(0.5, 1.5, 4) / 4
    keys = rng.standard_normal((50, 16))
    idx, sc = O.indexer_topk(q, w, keys, seq_len=45, top_k=12)
    assert sc.shape == (45,)
    assert idx.tolist() == _brute_topk(_brute_scores(q, w, keys[:45]), range(45), 12)
    idx2, _ = O.indexer_topk(q, w, keys, seq_len=7, top_k=12)  # seq_len < K: pad with -1
    assert idx2.tolist() == list(range(7)) + [-1] * 5


def test_block_max_and_pool_brute_force():
    rng = np.random.default_rng(7)
    s = rng.integers(0, 20, 43).astype(np.float32)  # ragged: 43 = 5 * 8 + 3
    bm = O.block_max(s, 43, 8)
    assert bm.tolist() == [max(s[j * 8:min(j * 8 + 8, 43)]) for j in range(6)]
    pool = O.pool_select(s, 43, 8, 4)
    assert pool.tolist() == _brute_topk(bm, range(6), 4)
    assert O.pool_select(s, 43, 8, 9).tolist() == list(range(6)) + [-1] * 3


def test_reindex_with_pool_of_all_blocks_is_flat_topk():
    rng = np.random.default_rng(8)
    for seq_len in (64, 61, 5):
        q = rng.standard_normal((5, 16))
        w = rng.uniform(0.5, 1.5, 5)
        keys = rng.standard_normal((64, 16))
        flat, _ = O.indexer_topk(q, w, keys, seq_len, 10)
        allblocks = np.arange(-(-seq_len // 8))
        re, pos, _ = O.reindex_topk(q, w, keys, seq_len, allblocks, 8, 10)
        assert re.tolist() == flat.tolist()
        assert pos.tolist() == list(range(seq_len))


def test_flat_topk_lies_inside_a_pool_of_at_least_k_blocks():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((4, 16))
    w = rng.uniform(0.5, 1.5, 4)
    keys = rng.standard_normal((400, 16))
    idx, pool, _ = O.hier_pool_select(q, w, keys, 397, top_k=12, block_size=8, n_pool_blocks=12)
    assert set((idx[idx >= 0] // 8).tolist()) <= set(pool[pool >= 0].tolist())
    # and the same layer re-indexing inside its own pool reproduces its flat top-K
    re, _, _ = O.reindex_topk(q, w, keys, 397, pool, 8, 12)
    assert re.tolist() == idx.tolist()


def test_reindex_brute_force_on_a_partial_pool():
    rng = np.random.default_rng(10)
    q = rng.standard_normal((2, 8))
    w = np.array([0.7, 0.3])
    keys = rng.standard_normal((70, 8))
    pool = np.array([1, 4, 8, -1])  # block 8 covers 64..69 only (seq_len 70)
    idx, pos, sc = O.reindex_topk(q, w, keys, 70, pool, 8, 9)
    want_pos = list(range(8, 16)) + list(range(32, 40)) + list(range(64, 70))
    assert pos.tolist() == want_pos
    assert idx.tolist() == _brute_topk(_brute_scores(q, w, keys[want_pos]), want_pos, 9)


def _rows(rng, n, d):
    x = rng.standard_normal((n, d)) * 2
    return O.kv_quant_fp4(x)


def _brute_attn(q, vh, sm):
    H, J = len(q), len(vh)
    out, lse = [], []
    for h in range(H):
        z = [sm * math.fsum(q[h] * vh[j]) for j in range(J)]
        m = max(z)
        e = [math.exp(t - m) for t in z]
        den = math.fsum(e)
        out.append([math.fsum(e[j] * vh[j][c] for j in range(J)) / den for c in range(len(q[h]))])
        lse.append(m + math.log(den))
    return np.array(out), np.array(lse)


def test_attention_with_all_rows_equals_dense_softmax():
    rng = np.random.default_rng(11)
    packed, scales = _rows(rng, 24, 32)
    q = rng.standard_normal((3, 32)) * 0.3
    idx = rng.permutation(24)
    out, lse = O.sparse_attn_decode(q, packed, scales, idx, 24, 0.7)
    ref_out, ref_lse = _brute_attn(q, O.kv_dequant_fp4(packed, scales), 0.7)
    assert np.allclose(out, ref_out, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_k1_returns_the_row_and_equal_logits_average():
    rng = np.random.default_rng(12)
    packed, scales = _rows(rng, 10, 32)
    vh = O.kv_dequant_fp4(packed, scales)
    q = rng.standard_normal((2, 32))
    out, lse = O.sparse_attn_decode(q, packed, scales, np.array([6, -1, 99]), 10, 1.0)
    assert np.array_equal(out, np.stack([vh[6], vh[6]]))
    assert np.allclose(lse, q @ vh[6])
    out0, lse0 = O.sparse_attn_decode(np.zeros((1, 32)), packed, scales, np.array([1, 2, 5]), 10, 1.0)
    assert np.allclose(out0[0], vh[[1, 2, 5]].mean(axis=0), rtol=0, atol=1e-12)
    assert np.isclose(lse0[0], math.log(3))


def test_attention_duplicates_count_and_invalid_entries_skip():
    rng = np.random.default_rng(13)
    packed, scales = _rows(rng, 12, 32)
    vh = O.kv_dequant_fp4(packed, scales)
    q = rng.standard_normal((2, 32)) * 0.5
    out, lse = O.sparse_attn_decode(q, packed, scales, np.array([3, 3, 7, -1, 12, 11]), 12, 1.0)
    ref_out, ref_lse = _brute_attn(q, vh[[3, 3, 7, 11]], 1.0)
    assert np.allclose(out, ref_out, atol=1e-12) and np.allclose(lse, ref_lse, atol=1e-12)
    # seq_len bounds the valid rows even when the cache holds more
    out2, _ = O.sparse_attn_decode(q, packed, scales, np.array([3, 11]), 10, 1.0)
    assert np.allclose(out2, O.sparse_attn_decode(q, packed, scales, np.array([3]), 10, 1.0)[0])


def test_attention_rows_helper_matches_brute_force_scaled_with_duplicates():
    """The helper every GPU parity test compares against, pinned on its own: plain-loop
    softmax attention at sm_scale != 1 over rows with duplicates and large logits (a
    dropped sm_scale, a missing max shift or a wrong lse term fails here)."""
    rng = np.random.default_rng(15)
    packed, scales = _rows(rng, 9, 32)
    vh = O.kv_dequant_fp4(packed, scales)
    sel = vh[[4, 1, 4, 8, 0, 4]]
    q = rng.standard_normal((3, 32)) * 4.0  # logits of tens: the max shift matters
    for sm in (0.75, 1.0, 2.5):
        out, lse = O.sparse_attn_decode_rows(q, sel, sm)
        ref_out, ref_lse = _brute_attn(q, sel, sm)
        assert np.allclose(out, ref_out, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)
    # and through the gathering entry point, which must agree with the helper exactly
    out_g, lse_g = O.sparse_attn_decode(q, packed, scales, np.array([4, 1, 4, 8, 0, 4]), 9, 0.75)
    ref_out, ref_lse = _brute_attn(q, sel, 0.75)
    assert np.allclose(out_g, ref_out, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse_g, ref_lse, rtol=1e-12, atol=1e-12)


def test_attention_with_no_valid_entry():
    rng = np.random.default_rng(14)
    packed, scales = _rows(rng, 4, 32)
    out, lse = O.sparse_attn_decode(np.ones((2, 32)), packed, scales, np.array([-1, 9]), 4, 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ----------------------------------------------------------------------------------------
# FP4 indexer operands
# ----------------------------------------------------------------------------------------

def test_fp4_indexer_values_leave_fp4_grid_rows_unchanged():
    """Rows already on the FP4 grid, with each 16-dim group's largest magnitude equal to
    6 * S for an E4M3 value S, are stored without loss: the FP4 scores equal the plain
    scores of the same values."""
    rng = np.random.default_rng(3)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    e4m3_normals = O.e4m3_decode(np.arange(0x08, 0x7F))  # normal E4M3 values

    def grid_rows(n):
        mags = grid[rng.integers(0, 8, size=(n, 8, 16))]
        mags[:, :, 0] = 6.0  # the group's amax is 6 * S exactly
        sign = np.where(rng.random((n, 8, 16)) < 0.5, -1.0, 1.0)
        S = e4m3_normals[rng.integers(0, e4m3_normals.size, size=(n, 8, 1))]
        S = np.minimum(S, 2.0)  # keep products well inside the bf16 and fp32 ranges
        return (sign * mags * S).reshape(n, 128)

    q, keys = grid_rows(4), grid_rows(50)
    assert np.array_equal(O.indexer_fp4_values(q), q)
    assert np.array_equal(O.indexer_fp4_values(keys), keys)
    w = rng.uniform(0.5, 1.5, size=4)
    assert np.array_equal(O.indexer_scores(O.indexer_fp4_values(q), w, O.indexer_fp4_values(keys)),
                          O.indexer_scores(q, w, keys))


def test_fp4_indexer_one_nonzero_dim_closed_form():
    """A query and a key with one non-zero dim c: each group holding it quantizes to
    6 * E4M3(|x| / 6) with x's sign, so the single-head score is
    w * max(0, sign * 36 * E4M3(|q_c| / 6) * E4M3(|k_c| / 6))."""
    qs = [0.3, -1.7, 2.5, 0.01171875, 100.0]
    ks = [1.0, 0.4, -3.3, 7.0, 0.05]
    for i, (qv, kv) in enumerate(zip(qs, ks)):
        c = (5 * i + 3) % 128
        q = np.zeros((1, 128))
        k = np.zeros((1, 128))
        q[0, c], k[0, c] = qv, kv
        want = 0.75 * max(0.0, np.sign(qv * kv) * 36.0 * O.e4m3_decode(O.e4m3_round_sat(abs(qv) / 6.0))
                          * O.e4m3_decode(O.e4m3_round_sat(abs(kv) / 6.0)))
        got = O.indexer_scores(O.indexer_fp4_values(q), [0.75], O.indexer_fp4_values(k))
        assert got[0] == np.float32(want), (qv, kv, got[0], want)


# ----------------------------------------------------------------------------------------
# Sliding-window branch (FP8 rows in the same softmax as the selected rows)
# ----------------------------------------------------------------------------------------

def test_swa_quant_fp8_sign_saturation_and_brute_force():
    """Codes are the nearest E4M3 value (ties to the even code, |x| > 448 -> 448) with the
    sign of x, checked against a plain search over all 127 non-negative values."""
    vals = [float(O.e4m3_decode(c)) for c in range(127)]
    rng = np.random.default_rng(7)
    xs = np.concatenate([rng.normal(0, 3, 400), rng.normal(0, 300, 100), [0.0, -0.0, 1e-9, -1e-9, 448, 449, 1e4, -1e4],
                         [(vals[i] + vals[i + 1]) / 2 for i in range(126)]])  # every midpoint
    for x in xs:
        a = abs(float(x))
        if a >= 448:
            want = 0x7E
        else:
            d = [abs(a - v) for v in vals]
            best = min(d)
            ties = [c for c in range(127) if d[c] == best]
            want = ties[0] if len(ties) == 1 else next(c for c in ties if c % 2 == 0)
        want |= 0x80 if math.copysign(1.0, float(x)) < 0 else 0
        assert int(O.swa_quant_fp8(np.float64(x))) == want, x


def _lse_merge(o1, l1, o2, l2):
    m = np.maximum(l1, l2)
    w1, w2 = np.exp(l1 - m), np.exp(l2 - m)
    return (w1[:, None] * o1 + w2[:, None] * o2) / (w1 + w2)[:, None], m + np.log(w1 + w2)


def test_swa_one_softmax_equals_the_lse_merge_of_the_two_branches():
    rng = np.random.default_rng(8)
    q = rng.normal(0, 0.05, (6, 64))
    sel = rng.normal(0, 1, (20, 64))
    win = rng.normal(0, 1, (9, 64))
    o, lse = O.sparse_swa_attn_decode_rows(q, sel, win, 1.3)
    o1, l1 = O.sparse_attn_decode_rows(q, sel, 1.3)
    o2, l2 = O.sparse_attn_decode_rows(q, win, 1.3)
    om, lm = _lse_merge(o1, l1, o2, l2)
    assert np.allclose(o, om, rtol=1e-12, atol=1e-12) and np.allclose(lse, lm, rtol=1e-12, atol=1e-12)
    # an empty selection leaves the window's dense attention, an empty window the sparse one
    ow, lw = O.sparse_swa_attn_decode_rows(q, np.zeros((0, 64)), win, 1.3)
    assert np.allclose(ow, o2) and np.allclose(lw, l2)
    os_, ls = O.sparse_swa_attn_decode_rows(q, sel, np.zeros((0, 64)), 1.3)
    assert np.allclose(os_, o1) and np.allclose(ls, l1)


def test_attn_lse_merge_equals_attention_over_the_union():
    """Context sharding: attention over disjoint row sets merged by their lse equals the
    attention over all rows (brute force), empty sets included."""
    rng = np.random.default_rng(9)
    q = rng.normal(0, 0.05, (5, 32))
    sets = [rng.normal(0, 1, (7, 32)), np.zeros((0, 32)), rng.normal(0, 1, (12, 32)), rng.normal(0, 2, (1, 32))]
    outs, lses = [], []
    for rows in sets:
        if rows.shape[0]:
            o, l = O.sparse_attn_decode_rows(q, rows, 0.7)
        else:
            o, l = np.zeros((5, 32)), np.full(5, -np.inf)
        outs.append(o)
        lses.append(l)
    om, lm = O.attn_lse_merge(np.stack(outs), np.stack(lses))
    ow, lw = O.sparse_attn_decode_rows(q, np.concatenate(sets), 0.7)
    assert np.allclose(om, ow, rtol=1e-12, atol=1e-12) and np.allclose(lm, lw, rtol=1e-12, atol=1e-12)
    oe, le = O.attn_lse_merge(np.zeros((2, 5, 32)), np.full((2, 5), -np.inf))
    assert np.all(oe == 0) and np.all(np.isneginf(le))
