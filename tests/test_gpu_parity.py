"""GPU parity: every call of the C ABI against the CPU oracle on the same seeded inputs.

Sizes span several tiles with ragged tails; the full-size configurations have their own
file. All calls go through the C ABI (``fp4_sparse_attention_kv_b200.binding``).
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import fp4kv_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fk(cuda_lib):
    import fp4_sparse_attention_kv_b200 as fk
    return fk


def _bf16_from_f64(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


# ----------------------------------------------------------------------------------------
# kv_quant_fp4
# ----------------------------------------------------------------------------------------

def _quant_gpu(fk, x_bf16: torch.Tensor):
    n, d = x_bf16.shape
    xd = x_bf16.to(DEV)
    packed = torch.empty((n, d // 2), dtype=torch.uint8, device=DEV)
    scales = torch.empty((n, d // 16), dtype=torch.uint8, device=DEV)
    fk.kv_quant_fp4(xd, packed, scales)
    return packed.cpu().numpy(), scales.cpu().numpy()


def _exhaustive_groups():
    """Groups [A, x1..x15]: for every E4M3 scale code s, A is the largest bf16 value whose
    scale is s, and x runs over every finite bf16 value (both signs) with |x| <= A; plus one
    group per non-negative finite bf16 amax."""
    bits = np.arange(0, 0x7F80, dtype=np.uint16)
    v = O.bf16_bits_to_f64(bits)
    s_of = O.e4m3_round_sat(v / 6.0)
    groups = []
    for s in range(0, 127):
        cand = v[s_of == s]
        if cand.size == 0:
            continue
        A = cand.max()
        xs = v[v <= A]
        xs = np.concatenate([xs, -xs])
        pad = (-xs.size) % 15
        xs = np.concatenate([xs, np.zeros(pad)]).reshape(-1, 15)
        groups.append(np.concatenate([np.full((xs.shape[0], 1), A), xs], axis=1))
    # every amax value once (scale coverage), sign of the max alternating
    am = np.zeros((v.size, 16))
    am[:, 0] = np.where(np.arange(v.size) % 2 == 0, v, -v)
    am[:, 5] = v / 3.0  # arbitrary second element below the max (bf16-rounded below)
    groups.append(am)
    g = np.concatenate(groups, axis=0)
    pad = (-g.shape[0]) % 32
    g = np.concatenate([g, np.zeros((pad, 16))], axis=0)
    return g.reshape(-1, 512)


def test_quant_exhaustive_bf16_values_by_scale(fk):
    x = _exhaustive_groups()
    xb = _bf16_from_f64(x)
    xv = P.to_f64(xb)  # exact bf16 values given to both sides
    gp, gs = _quant_gpu(fk, xb)
    op, os_ = O.kv_quant_fp4(xv)
    assert np.array_equal(gs, os_), f"scale bytes differ in {np.sum(gs != os_)} groups"
    assert np.array_equal(gp, op), f"packed bytes differ in {np.sum(gp != op)} places"


def test_quant_golden_example(fk):
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "quant_example.json")))
    x = np.array(g["rows"], dtype=np.float64)
    x[0, 7] = -0.0
    x[1, 3] = -0.0
    x = np.concatenate([x, np.zeros((2, 32))], axis=1)  # d = 64 (library needs d % 32 == 0)
    gp, gs = _quant_gpu(fk, _bf16_from_f64(x))
    assert [bytes(r[:16]).hex().upper() for r in gp] == g["packed_hex"]
    assert gs[:, :2].tolist() == g["scales"]


@pytest.mark.parametrize("d", [512, 64, 1024])
def test_quant_synthetic_rows_with_saturation(fk, d):
    rows = torch.arange(3000, dtype=torch.int64)
    xb = synth.kv_rows(1, 3, 0, rows, d, heavy_frac=0.01)
    gp, gs = _quant_gpu(fk, xb)
    op, os_ = O.kv_quant_fp4(P.to_f64(xb))
    assert np.array_equal(gs, os_) and np.array_equal(gp, op)
    assert (gs == 0x7E).any()  # some rows saturate the scale at 448


def test_quant_scatter_rows_and_stride(fk):
    d = 512
    src = synth.kv_rows(2, 0, 0, torch.arange(64), 1024)[:, :d]  # row stride 1024 > d
    xd = synth.kv_rows(2, 0, 0, torch.arange(64), 1024).to(DEV)[:, :d]
    cap = 200
    packed = torch.full((cap, d // 2), 0xAB, dtype=torch.uint8, device=DEV)
    scales = torch.full((cap, d // 16), 0xCD, dtype=torch.uint8, device=DEV)
    dst = torch.tensor([3 * i + 1 for i in range(60)] + [-1, cap, 10 ** 9, 0], dtype=torch.int64)
    fk.kv_quant_fp4(xd, packed, scales, dst_row=dst.to(DEV))
    op, os_ = O.kv_quant_fp4(P.to_f64(src))
    pk, sc = packed.cpu().numpy(), scales.cpu().numpy()
    for i, r in enumerate(dst.tolist()):
        if 0 <= r < cap:
            assert np.array_equal(pk[r], op[i]) and np.array_equal(sc[r], os_[i])
    untouched = sorted(set(range(cap)) - {r for r in dst.tolist() if 0 <= r < cap})
    assert np.all(pk[untouched] == 0xAB) and np.all(sc[untouched] == 0xCD)


# ----------------------------------------------------------------------------------------
# indexer scores / top-K / pool / reindex
# ----------------------------------------------------------------------------------------

def _indexer_inputs(seed, B, cap, H_I, fp8):
    q, w = synth.indexer_query(seed, 0, B, H_I, fp8=fp8, device=DEV)
    keys = P.keys_dev(seed, B, cap, fp8, DEV)
    return q, w, keys


def test_generator_is_identical_on_host_and_device():
    rows = torch.arange(0, 5000, 7, dtype=torch.int64)
    for fp8 in (True, False):
        a = synth.indexer_keys(3, 1, rows, 128, fp8)
        b = synth.indexer_keys(3, 1, rows.to(DEV), 128, fp8).cpu()
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    a = synth.kv_rows(4, 2, 1, rows, 512, heavy_frac=0.01)
    b = synth.kv_rows(4, 2, 1, rows.to(DEV), 512, heavy_frac=0.01).cpu()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    qa, wa = synth.indexer_query(5, 1, 3, 32)
    qb, wb = synth.indexer_query(5, 1, 3, 32, device=DEV)
    assert torch.equal(qa, qb.cpu()) and torch.equal(wa, wb.cpu())
    assert torch.equal(synth.attn_query(6, 0, 2, 16, 512).view(torch.int16),
                       synth.attn_query(6, 0, 2, 16, 512, device=DEV).cpu().view(torch.int16))


@pytest.mark.parametrize("fp8,H_I", [(True, 32), (False, 32), (True, 1), (True, 20), (True, 64)])
def test_indexer_scores_match_oracle(fk, fp8, H_I):
    B, cap = 2, 1000
    q, w, keys = _indexer_inputs(7, B, cap, H_I, fp8)
    lens = torch.tensor([1000, 613], dtype=torch.int32, device=DEV)
    ks = torch.rand((B, cap), generator=torch.Generator().manual_seed(1)).to(DEV) + 0.5
    for key_scale in (None, ks):
        got = fk.indexer_scores(q, w, keys, lens, key_scale=key_scale).cpu().numpy()
        for b in range(B):
            L = int(lens[b])
            ref = P.oracle_scores_seq(q[b], w[b], keys[b], L, None if key_scale is None else ks[b])
            err = np.abs(got[b, :L].astype(np.float64) - ref) / np.maximum(np.abs(ref), 1e-3)
            assert err.max() <= 2e-6, err.max()
            assert np.all(np.isneginf(got[b, L:]))


@pytest.mark.parametrize("case", [
    dict(seed=0, B=1, cap=4096, lens=[4096], H_I=32, fp8=False, k=256),     # the tiny config
    dict(seed=1, B=3, cap=5000, lens=[5000, 4093, 77], H_I=32, fp8=True, k=300),
    dict(seed=2, B=2, cap=70000, lens=[70000, 65536], H_I=32, fp8=True, k=2048),
    dict(seed=3, B=2, cap=3000, lens=[3000, 2999], H_I=8, fp8=True, k=1),
    dict(seed=4, B=1, cap=9000, lens=[9000], H_I=64, fp8=True, k=4096),
])
def test_indexer_topk_matches_oracle(fk, case):
    q, w, keys = _indexer_inputs(case["seed"], case["B"], case["cap"], case["H_I"], case["fp8"])
    lens = torch.tensor(case["lens"], dtype=torch.int32, device=DEV)
    k = case["k"]
    score = torch.empty((case["B"], k), dtype=torch.float32, device=DEV)
    idx = fk.indexer_topk(q, w, keys, lens, k, out_score=score).cpu().numpy()
    score = score.cpu().numpy()
    for b in range(case["B"]):
        L = case["lens"][b]
        ref = P.oracle_scores_seq(q[b], w[b], keys[b], L)
        P.check_topk(idx[b], ref, np.arange(L), k, f"b={b}")
        m = min(k, L)
        assert np.all(np.isneginf(score[b, m:]))
        err = np.abs(score[b, :m].astype(np.float64) - ref[idx[b, :m]]) / np.maximum(ref[idx[b, :m]], 1e-3)
        assert err.max() <= 2e-6


def test_indexer_topk_ties_go_to_the_lowest_positions(fk):
    B, cap, k = 2, 3000, 100
    q, w, _ = _indexer_inputs(9, B, cap, 32, True)
    row = synth.indexer_keys(9, 0, torch.arange(1, dtype=torch.int64), 128, True)
    keys = row.repeat(cap, 1).reshape(1, cap, 128).repeat(B, 1, 1).to(DEV).contiguous()
    keys[1, 2000:2050] = 0  # lower scores in the middle of sequence 1
    lens = torch.tensor([3000, 2500], dtype=torch.int32, device=DEV)
    idx = fk.indexer_topk(q, w, keys, lens, k).cpu().numpy()
    assert idx[0].tolist() == list(range(k))
    assert idx[1].tolist() == list(range(k))
    # all scores equal -> every position is a candidate; K larger than one radix bucket
    idx2 = fk.indexer_topk(q, w, keys, lens, 4096).cpu().numpy()
    assert idx2[0].tolist() == list(range(3000)) + [-1] * 1096


def test_indexer_topk_all_equal_scores_beyond_the_staging_buffer(fk):
    # 20000 equal scores: every entry survives both radix digits and the last 8 key bits,
    # so the selection is decided by the position histograms alone, over more kept entries
    # than the warps hold in shared memory (the rest overflow to the workspace)
    cap = 20000
    q, w, _ = _indexer_inputs(9, 1, cap, 32, True)
    row = synth.indexer_keys(9, 0, torch.arange(1, dtype=torch.int64), 128, True)
    keys = row.repeat(cap, 1).reshape(1, cap, 128).to(DEV).contiguous()
    lens = torch.tensor([cap], dtype=torch.int32, device=DEV)
    for k in (1, 100, 4096):
        idx = fk.indexer_topk(q, w, keys, lens, k).cpu().numpy()
        assert idx[0].tolist() == list(range(k)), k


@pytest.mark.parametrize("n_equal", [40, 64, 65, 200])
def test_indexer_topk_equal_top_keys_spread_over_the_cluster(fk, n_equal):
    # n_equal copies of the best-scoring key row at random positions of a 200,000-entry
    # sequence (the select's cluster splits it over several CTAs): the K-th key lies inside
    # a bin of n_equal equal keys, which is ranked directly up to 64 keys and by the last-8-bit
    # and position histograms beyond; either way the lowest K positions of the copies win
    cap, k = 200000, 30
    q, w, keys = _indexer_inputs(21, 1, cap, 32, True)
    lens = torch.tensor([cap], dtype=torch.int32, device=DEV)
    ref = P.oracle_scores_seq(q[0], w[0], keys[0], cap)
    top = int(np.argmax(ref))
    rng = np.random.default_rng(21 + n_equal)
    others = rng.choice(np.setdiff1d(np.arange(cap), [top]), size=n_equal - 1, replace=False)
    pos = np.sort(np.concatenate([[top], others]))
    keys[0, torch.from_numpy(others).to(DEV)] = keys[0, top].clone()
    score = torch.empty((1, k), dtype=torch.float32, device=DEV)
    idx = fk.indexer_topk(q, w, keys, lens, k, out_score=score).cpu().numpy()
    assert idx[0].tolist() == pos[:k].tolist()
    assert np.all(score.cpu().numpy()[0] == np.float32(score.cpu().numpy()[0, 0]))


def test_reindex_with_a_pool_in_arbitrary_order(fk):
    # pool blocks listed out of position order: the output is still ascending positions
    B, cap, k, npb = 2, 20000, 300, 96
    q, w, keys = _indexer_inputs(14, B, cap, 32, True)
    lens = torch.tensor([20000, 15000], dtype=torch.int32, device=DEV)
    rng = np.random.default_rng(14)
    pools = [rng.permutation(int(lens[b]) // 8)[:npb].astype(np.int32) for b in range(B)]
    pool = torch.tensor(np.stack(pools), dtype=torch.int32, device=DEV)
    idx = fk.indexer_topk(q, w, keys, lens, k, pool=pool).cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        pos = O.pool_positions(pools[b], L, 8)
        ref = P.oracle_scores_seq(q[b], w[b], keys[b], L)[pos]
        P.check_topk(idx[b], ref, pos, k, f"unordered pool b={b}")


def test_hier_pool_select_matches_oracle(fk):
    B, cap, k, npb = 2, 20000, 256, 64
    q, w, keys = _indexer_inputs(11, B, cap, 32, True)
    lens = torch.tensor([20000, 12345], dtype=torch.int32, device=DEV)
    idx, pool = fk.hier_pool_select(q, w, keys, lens, k, npb)
    idx, pool = idx.cpu().numpy(), pool.cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        ref = P.oracle_scores_seq(q[b], w[b], keys[b], L)
        P.check_topk(idx[b], ref, np.arange(L), k, f"idx b={b}")
        bm = O.block_max(ref, L, 8)
        P.check_topk(pool[b], bm, np.arange(bm.size), npb, f"pool b={b}")


def test_decoder_sizes_topk_512_pool_2048(fk):
    # the pages' decoder sizes: top-K 512 and a pool of up to 2048 blocks; sequence 1 has
    # fewer blocks (1126) than the pool holds, so its pool is every block plus -1 padding
    B, cap, k, npb = 2, 40000, 512, 2048
    q, w, keys = _indexer_inputs(15, B, cap, 32, True)
    q2, w2 = synth.indexer_query(15, 4, B, 32, device=DEV)
    lens = torch.tensor([40000, 9001], dtype=torch.int32, device=DEV)
    idx, pool = fk.hier_pool_select(q, w, keys, lens, k, npb)
    idx, pool_np = idx.cpu().numpy(), pool.cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        ref = P.oracle_scores_seq(q[b], w[b], keys[b], L)
        P.check_topk(idx[b], ref, np.arange(L), k, f"idx b={b}")
        P.check_topk(pool_np[b], O.block_max(ref, L, 8), np.arange((L + 7) // 8), npb, f"pool b={b}")
    assert pool_np[1].tolist() == list(range(1126)) + [-1] * (npb - 1126)
    idx2 = fk.indexer_topk(q2, w2, keys, lens, k, pool=pool).cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        pos = O.pool_positions(pool_np[b], L, 8)
        ref = P.oracle_scores_seq(q2[b], w2[b], keys[b], L)[pos]
        P.check_topk(idx2[b], ref, pos, k, f"reindex b={b}")


def test_reindex_matches_oracle_and_full_pool_is_flat(fk):
    B, cap, k, npb = 2, 20000, 256, 64
    q, w, keys = _indexer_inputs(12, B, cap, 32, True)
    q2, w2 = synth.indexer_query(12, 1, B, 32, device=DEV)  # this layer's own query
    lens = torch.tensor([20000, 9999], dtype=torch.int32, device=DEV)
    pools = []
    for b in range(B):
        L = int(lens[b])
        ref = P.oracle_scores_seq(q[b], w[b], keys[b], L)
        pl = O.pool_select(ref, L, 8, npb)
        pl[5] = -1  # a hole in the pool
        pools.append(pl)
    pool = torch.tensor(np.stack(pools), dtype=torch.int32, device=DEV)
    idx = fk.indexer_topk(q2, w2, keys, lens, k, pool=pool).cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        pos = O.pool_positions(pools[b], L, 8)
        ref = P.oracle_scores_seq(q2[b], w2[b], keys[b], L)[pos] if pos.size else np.zeros(0)
        P.check_topk(idx[b], ref, pos, k, f"reindex b={b}")
    # pool = every block of a short sequence: Reindex equals the flat top-K
    L = 1000
    lens_s = torch.tensor([L, L], dtype=torch.int32, device=DEV)
    allb = torch.arange(125, dtype=torch.int32, device=DEV).repeat(B, 1).contiguous()
    re = fk.indexer_topk(q2, w2, keys, lens_s, 200, pool=allb).cpu().numpy()
    fl = fk.indexer_topk(q2, w2, keys, lens_s, 200).cpu().numpy()
    assert np.array_equal(re, fl)


# ----------------------------------------------------------------------------------------
# sparse attention
# ----------------------------------------------------------------------------------------

def _attn_case(fk, seed, B, cap, H, lens, idx_np, layer=0, sm_scale=1.0):
    d = 512
    x = P.kv_rows_dev(seed, layer, B, cap, d, DEV)
    packed = torch.empty((B, cap, d // 2), dtype=torch.uint8, device=DEV)
    scales = torch.empty((B, cap, d // 16), dtype=torch.uint8, device=DEV)
    fk.kv_quant_fp4(x.view(B * cap, d), packed.view(B * cap, d // 2), scales.view(B * cap, d // 16))
    del x
    q = synth.attn_query(seed, layer, B, H, d, device=DEV)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    idx = torch.tensor(idx_np, dtype=torch.int32, device=DEV)
    out, lse = fk.sparse_attn_decode(q, packed, scales, lens_t, idx, sm_scale)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    qh = P.to_f64(q.cpu())
    for b in range(B):
        sel = np.asarray(idx_np[b])
        valid = sel[(sel >= 0) & (sel < lens[b])]
        if valid.size:
            rows = P.kv_rows_host(seed, layer, b, valid, d)
            pk, sc = O.kv_quant_fp4(rows)  # the oracle's own quantization
            ro, rl = O.sparse_attn_decode_rows(qh[b], O.kv_dequant_fp4(pk, sc), sm_scale)
        else:
            ro, rl = np.zeros((H, d)), np.full(H, -np.inf)
        P.check_attn(out[b], lse[b], ro, rl, f"b={b}")
    return out, lse


def test_attention_tiny_config_end_to_end(fk):
    # quantize -> oracle top-K of the bf16 indexer -> attention, 16 heads, K = 256
    cap, k = 4096, 256
    q8, w = synth.indexer_query(0, 0, 1, 32, fp8=False)
    keys = synth.indexer_keys(0, 0, torch.arange(cap), 128, fp8=False)
    ref = O.indexer_scores(P.to_f64(q8[0]), w[0].double().numpy(), P.to_f64(keys))
    idx = O.topk_positions(ref, np.arange(cap), k)[None, :]
    _attn_case(fk, 0, 1, cap, 16, [cap], idx)


def test_tiny_config_chained_on_the_gpu(fk):
    """The tiny configuration as the bench runs it, every step on the GPU: the library's
    quantize writes the cache and the new row, its indexer top-K (bf16 keys) selects from
    the written cache, and its attention reads those rows and that selection. The oracle
    runs the same chain from the generator's bf16 inputs on its own: its own quantizer,
    its own top-K (the GPU's selection must match it up to the tie band) and its own
    attention over its own selection."""
    import bench
    cfg = bench.CONFIGS["tiny"]
    wl = bench.DecodeWorkload(cfg, fk, torch.device(DEV))
    wl.step()
    torch.cuda.synchronize()
    cap, K, seed = wl.cap, wl.K, cfg["seed"]
    sc = P.oracle_scores_seq(wl.qi[0], wl.w[0], wl.keys[0], cap)
    idx = wl.idx[0].cpu().numpy()
    P.check_topk(idx, sc, np.arange(cap), K, "tiny top-K")
    want = O.topk_positions(sc, np.arange(cap), K)
    if not np.array_equal(idx, want):  # a swap inside the tie band: attend over the GPU's set
        want = idx
    rows = P.kv_rows_host(seed, 0, 0, want[want >= 0], 512)
    rows[want[want >= 0] == cap - 1] = P.to_f64(wl.x_new[0:1].cpu())[0]
    pk, s8 = O.kv_quant_fp4(rows)
    ro, rl = O.sparse_attn_decode_rows(P.to_f64(wl.q[0].cpu()), O.kv_dequant_fp4(pk, s8), 1.0)
    P.check_attn(wl.out[0].cpu().numpy(), wl.lse[0].cpu().numpy(), ro, rl, "tiny chained attention")
    # the row the step wrote, bit-exact
    pk1, s1 = O.kv_quant_fp4(P.to_f64(wl.x_new[0:1].cpu()))
    assert np.array_equal(wl.packed[0, cap - 1].cpu().numpy(), pk1[0])
    assert np.array_equal(wl.scales[0, cap - 1].cpu().numpy(), s1[0])


@pytest.mark.parametrize("H", [64, 16, 20, 128])
def test_attention_decode_shapes(fk, H):
    B, cap, k = 3, 8192, 2048
    rng = np.random.default_rng(H)
    idx = np.stack([np.sort(rng.choice(cap, k, replace=False)) for _ in range(B)])
    _attn_case(fk, 21, B, cap, H, [cap] * B, idx, sm_scale=1.0)


def test_attention_edge_cases(fk):
    B, cap, k = 5, 600, 300
    rng = np.random.default_rng(5)
    idx = np.stack([rng.choice(cap, k, replace=False) for _ in range(B)]).astype(np.int64)
    idx[0, :50] = -1                   # holes
    idx[1, :20] = idx[1, 20]           # duplicates count
    idx[2, :] = -1                     # nothing valid: out = 0, lse = -inf
    idx[3, 10:] = 10 ** 6              # beyond the cache
    lens = [600, 600, 600, 600, 250]   # sequence 4: entries >= 250 invisible
    out, lse = _attn_case(fk, 31, B, cap, 64, lens, idx, sm_scale=0.75)
    assert np.all(out[2] == 0) and np.all(np.isneginf(lse[2]))


def test_attention_single_entry_returns_the_row(fk):
    B, cap, k = 2, 100, 1
    idx = np.array([[7], [99]])
    out, _ = _attn_case(fk, 41, B, cap, 16, [100, 100], idx)
    rows = P.kv_rows_host(41, 0, 0, [7], 512)
    pk, sc = O.kv_quant_fp4(rows)
    vh = O.kv_dequant_fp4(pk, sc)[0]
    assert np.allclose(out[0], np.broadcast_to(vh, out[0].shape), rtol=1e-6, atol=1e-6)


def test_workspace_is_left_clean_and_status_zero(fk):
    B, cap, k = 2, 5000, 128
    q, w, keys = _indexer_inputs(13, B, cap, 32, True)
    lens = torch.tensor([5000, 4000], dtype=torch.int32, device=DEV)
    ws = fk.alloc_workspace(fk.workspace_bytes(fk.OP_INDEXER_TOPK, B, cap, 32, k), DEV)
    a = fk.indexer_topk(q, w, keys, lens, k, ws=ws).clone()
    b = fk.indexer_topk(q, w, keys, lens, k, ws=ws)
    assert torch.equal(a, b)
    assert fk.workspace_status(ws) == 0


def test_bounded_wait_reports_a_timeout_and_the_context_stays_usable(fk):
    """Failure detection without a device fault: a kernel waits on a barrier that nothing
    signals, gives up after 20 ms, sets the workspace's wait-timeout bit and returns; the
    host reads the bit, and the same context then quantizes bit-exactly."""
    ws = fk.alloc_workspace(256, DEV)
    fk.selftest_wait_timeout(20000, ws)
    assert fk.workspace_status(ws) == 1
    assert fk.workspace_status(ws) == 0  # reading clears the word
    x = P.kv_rows_dev(17, 0, 1, 64, 512, torch.device(DEV))[0]
    packed = torch.empty((64, 256), dtype=torch.uint8, device=DEV)
    scales = torch.empty((64, 32), dtype=torch.uint8, device=DEV)
    fk.kv_quant_fp4(x, packed, scales)
    pk, sc = O.kv_quant_fp4(P.to_f64(x.cpu()))
    assert np.array_equal(packed.cpu().numpy(), pk)
    assert np.array_equal(scales.cpu().numpy(), sc)


def test_selftest_hook_rejects_bad_arguments(fk):
    ws = fk.alloc_workspace(256, DEV)
    for bad in (0, -5, 1000001):
        with pytest.raises(fk.Fp4kvError):
            fk.selftest_wait_timeout(bad, ws)
    assert fk.workspace_status(ws) == 0


# ----------------------------------------------------------------------------------------
# FP4 (E2M1 + per-16 E4M3 scale) indexer query and keys
# ----------------------------------------------------------------------------------------

def _fp4_indexer_inputs(fk, seed, B, cap, H_I, layer=0):
    """bf16 indexer query / keys from the generator, stored as FP4 by the library."""
    qb, w = synth.indexer_query(seed, layer, B, H_I, fp8=False, device=DEV)
    kb = P.keys_dev(seed, B, cap, False, DEV)
    q4 = fk.E2M1Planes(B, H_I, DEV).quantize_from(qb)
    k4 = fk.E2M1Planes(B, cap, DEV).quantize_from(kb)
    return qb, w, kb, q4, k4


def _fp4_oracle_scores(qb_b, w_b, kb_b, L, ks=None):
    """The oracle's own FP4 storage of the bf16 inputs, then its scores (fp32)."""
    return O.indexer_scores(O.indexer_fp4_values(P.to_f64(qb_b)), w_b.detach().cpu().double().numpy(),
                            O.indexer_fp4_values(P.to_f64(kb_b[:L])),
                            None if ks is None else ks[:L].detach().cpu().double().numpy())


def test_fp4_indexer_planes_are_the_quantizer_output(fk):
    qb, _, kb, q4, k4 = _fp4_indexer_inputs(fk, 21, 2, 600, 32)
    for x, planes in ((qb, q4), (kb, k4)):
        pk, sc = O.kv_quant_fp4(P.to_f64(x.reshape(-1, 128)))
        assert np.array_equal(planes.codes.reshape(-1, 64).cpu().numpy(), pk)
        assert np.array_equal(planes.scales.reshape(-1, 8).cpu().numpy(), sc)


@pytest.mark.parametrize("H_I", [8, 32, 48, 64])
def test_fp4_indexer_scores_match_oracle(fk, H_I):
    B, cap = 2, 1000
    qb, w, kb, q4, k4 = _fp4_indexer_inputs(fk, 22, B, cap, H_I)
    lens = torch.tensor([1000, 613], dtype=torch.int32, device=DEV)
    ks = torch.rand((B, cap), generator=torch.Generator().manual_seed(2)).to(DEV) + 0.5
    for key_scale in (None, ks):
        got = fk.indexer_scores(q4, w, k4, lens, key_scale=key_scale).cpu().numpy()
        for b in range(B):
            L = int(lens[b])
            ref = _fp4_oracle_scores(qb[b], w[b], kb[b], L, None if key_scale is None else ks[b])
            err = np.abs(got[b, :L].astype(np.float64) - ref) / np.maximum(np.abs(ref), 1e-3)
            assert err.max() <= 2e-6, err.max()
            assert np.all(np.isneginf(got[b, L:]))


@pytest.mark.parametrize("case", [
    dict(seed=23, B=3, cap=5000, lens=[5000, 4093, 77], H_I=32, k=300),
    dict(seed=24, B=2, cap=70000, lens=[70000, 65537], H_I=32, k=2048),
    dict(seed=25, B=2, cap=3000, lens=[3000, 2999], H_I=8, k=1),
    dict(seed=26, B=1, cap=9000, lens=[9000], H_I=64, k=4096),
])
def test_fp4_indexer_topk_matches_oracle(fk, case):
    qb, w, kb, q4, k4 = _fp4_indexer_inputs(fk, case["seed"], case["B"], case["cap"], case["H_I"])
    lens = torch.tensor(case["lens"], dtype=torch.int32, device=DEV)
    k = case["k"]
    idx = fk.indexer_topk(q4, w, k4, lens, k).cpu().numpy()
    for b in range(case["B"]):
        L = case["lens"][b]
        P.check_topk(idx[b], _fp4_oracle_scores(qb[b], w[b], kb[b], L), np.arange(L), k, f"b={b}")


def test_fp4_hier_pool_select_and_reindex_match_oracle(fk):
    B, cap, k, npb = 2, 20000, 256, 64
    qb, w, kb, q4, k4 = _fp4_indexer_inputs(fk, 27, B, cap, 32)
    q2b, w2 = synth.indexer_query(27, 1, B, 32, fp8=False, device=DEV)
    q24 = fk.E2M1Planes(B, 32, DEV).quantize_from(q2b)
    lens = torch.tensor([20000, 12346], dtype=torch.int32, device=DEV)
    idx, pool = fk.hier_pool_select(q4, w, k4, lens, k, npb)
    idx, pool_np = idx.cpu().numpy(), pool.cpu().numpy()
    idx2 = fk.indexer_topk(q24, w2, k4, lens, k, pool=pool).cpu().numpy()
    for b in range(B):
        L = int(lens[b])
        ref = _fp4_oracle_scores(qb[b], w[b], kb[b], L)
        P.check_topk(idx[b], ref, np.arange(L), k, f"idx b={b}")
        P.check_topk(pool_np[b], O.block_max(ref, L, 8), np.arange((L + 7) // 8), npb, f"pool b={b}")
        pos = O.pool_positions(pool_np[b], L, 8)
        ref2 = _fp4_oracle_scores(q2b[b], w2[b], kb[b], L)[pos]
        P.check_topk(idx2[b], ref2, pos, k, f"reindex b={b}")


def test_fp4_indexer_rejects_odd_sizes(fk):
    _, w, _, q4, _ = _fp4_indexer_inputs(fk, 28, 1, 64, 32)
    k_odd = fk.E2M1Planes(1, 63, DEV)
    k_odd.buf.zero_()
    lens = torch.tensor([63], dtype=torch.int32, device=DEV)
    with pytest.raises(fk.Fp4kvError):
        fk.indexer_topk(q4, w, k_odd, lens, 8)
    q_odd = fk.E2M1Planes(1, 31, DEV)
    q_odd.buf.zero_()
    k_even = fk.E2M1Planes(1, 64, DEV)
    k_even.buf.zero_()
    with pytest.raises(fk.Fp4kvError):
        fk.indexer_topk(q_odd, w[:, :31].contiguous(), k_even, lens, 8)


# ----------------------------------------------------------------------------------------
# Sliding-window branch: FP8 window rows in the same softmax as the selected FP4 rows
# ----------------------------------------------------------------------------------------

SWA_LAYER = 700  # generator stream of the window rows (a different projection than the main KV)


def test_swa_quant_fp8_bit_exact_over_all_finite_bf16(fk):
    bits = np.arange(0, 0x7F80, dtype=np.uint16)
    v = O.bf16_bits_to_f64(bits)
    x = np.concatenate([v, -v])
    x = np.concatenate([x, np.zeros((-x.size) % 512)]).reshape(-1, 512)
    xd = _bf16_from_f64(x).to(DEV)
    out = torch.empty(x.shape, dtype=torch.uint8, device=DEV)
    fk.swa_quant_fp8(xd, out)
    assert np.array_equal(out.cpu().numpy(), O.swa_quant_fp8(x))
    # scattered rows (dst_row), rows outside the buffer skipped
    dst = torch.tensor([3, -1, 0, 10 ** 9], dtype=torch.int64, device=DEV)
    out2 = torch.zeros((4, 512), dtype=torch.uint8, device=DEV)
    fk.swa_quant_fp8(xd[:4].contiguous(), out2, dst_row=dst)
    want = np.zeros((4, 512), dtype=np.uint8)
    want[3], want[0] = O.swa_quant_fp8(x[0]), O.swa_quant_fp8(x[2])
    assert np.array_equal(out2.cpu().numpy(), want)


def _swa_case(fk, seed, B, cap, H, lens, idx_np, n_win, sm_scale=1.0):
    """Selected FP4 rows + the window of the last min(n_win, len) positions (E4M3, ring slot
    = position % n_win), one softmax; checked against the oracle per sequence."""
    d = 512
    x = P.kv_rows_dev(seed, 0, B, cap, d, DEV)
    packed = torch.empty((B, cap, d // 2), dtype=torch.uint8, device=DEV)
    scales = torch.empty((B, cap, d // 16), dtype=torch.uint8, device=DEV)
    fk.kv_quant_fp4(x.view(B * cap, d), packed.view(B * cap, d // 2), scales.view(B * cap, d // 16))
    del x
    swa = torch.zeros((B, n_win, d), dtype=torch.uint8, device=DEV)
    win_pos = []
    for b in range(B):
        L = lens[b]
        pos = np.arange(max(0, L - n_win), L, dtype=np.int64)
        win_pos.append(pos)
        if pos.size:
            rows = synth.kv_rows(seed, SWA_LAYER, b, torch.as_tensor(pos, device=DEV), d)
            dst = torch.as_tensor(b * n_win + pos % n_win, device=DEV)
            fk.swa_quant_fp8(rows, swa.view(B * n_win, d), dst_row=dst)
    q = synth.attn_query(seed, 0, B, H, d, device=DEV)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    idx = torch.tensor(idx_np, dtype=torch.int32, device=DEV)
    out, lse = fk.sparse_attn_decode(q, packed, scales, lens_t, idx, sm_scale, swa=swa)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    qh = P.to_f64(q.cpu())
    for b in range(B):
        sel = np.asarray(idx_np[b])
        sel = sel[(sel >= 0) & (sel < lens[b])]
        v_sel = np.zeros((0, d))
        if sel.size:
            pk, sc = O.kv_quant_fp4(P.kv_rows_host(seed, 0, b, sel, d))
            v_sel = O.kv_dequant_fp4(pk, sc)
        v_win = O.e4m3_decode(O.swa_quant_fp8(P.kv_rows_host(seed, SWA_LAYER, b, win_pos[b], d)))
        if sel.size + win_pos[b].size:
            ro, rl = O.sparse_swa_attn_decode_rows(qh[b], v_sel, v_win.reshape(-1, d), sm_scale)
        else:
            ro, rl = np.zeros((H, d)), np.full(H, -np.inf)
        P.check_attn(out[b], lse[b], ro, rl, f"b={b}")
    return out, lse


def _rand_idx(rng, B, top_k, lens, pad_frac=0.1):
    idx = np.full((B, top_k), -1, dtype=np.int64)
    for b in range(B):
        m = min(top_k, lens[b])
        idx[b, :m] = np.sort(rng.choice(lens[b], size=m, replace=False))
        holes = rng.random(top_k) < pad_frac
        idx[b, holes] = -1
    return idx


@pytest.mark.parametrize("case", [
    dict(seed=31, B=3, cap=5000, H=64, top_k=300, lens=[5000, 100, 60], n_win=128),
    dict(seed=32, B=2, cap=9000, H=16, top_k=2048, lens=[9000, 8999], n_win=128),
    dict(seed=33, B=2, cap=3000, H=64, top_k=512, lens=[3000, 40], n_win=64),
    dict(seed=34, B=160, cap=300, H=16, top_k=128, lens=[300] * 160, n_win=128),  # one chunk per sequence
])
def test_sparse_swa_attention_matches_oracle(fk, case):
    rng = np.random.default_rng(case["seed"])
    idx = _rand_idx(rng, case["B"], case["top_k"], case["lens"])
    _swa_case(fk, case["seed"], case["B"], case["cap"], case["H"], case["lens"], idx, case["n_win"])


def test_sparse_swa_attention_window_only_and_nothing(fk):
    B, cap, H = 2, 1000, 64
    idx = np.full((B, 256), -1, dtype=np.int64)  # no selected entry: the window alone
    _swa_case(fk, 35, B, cap, H, [1000, 77], idx, 128)
    out, lse = _swa_case(fk, 36, 1, cap, H, [0], np.full((1, 128), -1, dtype=np.int64), 128)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ----------------------------------------------------------------------------------------
# Context-sharded decode: exact merge of per-range top-K lists, LSE combine of partials
# ----------------------------------------------------------------------------------------

def test_topk_merge_matches_oracle_with_ties_and_holes(fk):
    rng = np.random.default_rng(51)
    R, B, kp, K = 3, 4, 300, 256
    bases = [0, 5000, 9000]
    idx = np.full((R, B, kp), -1, dtype=np.int32)
    sc = np.full((R, B, kp), -np.inf, dtype=np.float32)
    for r in range(R):
        for b in range(B):
            m = [300, 120, 0, 37][b]
            idx[r, b, :m] = rng.choice(4000, size=m, replace=False)
            sc[r, b, :m] = rng.integers(0, 40, size=m).astype(np.float32) / 8  # many equal scores
    lo, hi = 5000, 9000
    out_score = torch.empty((B, K), dtype=torch.float32, device=DEV)
    got, local = fk.topk_merge(torch.from_numpy(sc).to(DEV), torch.from_numpy(idx).to(DEV), bases, K,
                               local_range=(lo, hi), out_score=out_score)
    got, local, out_score = got.cpu().numpy(), local.cpu().numpy(), out_score.cpu().numpy()
    for b in range(B):
        s_all, p_all = [], []
        for r in range(R):
            ok = idx[r, b] >= 0
            s_all.append(sc[r, b][ok])
            p_all.append(idx[r, b][ok].astype(np.int64) + bases[r])
        s_all, p_all = np.concatenate(s_all), np.concatenate(p_all)
        want = O.topk_positions(s_all, p_all, K)
        assert np.array_equal(got[b], want), b
        assert np.array_equal(local[b], np.where((want >= lo) & (want < hi), want - lo, -1)), b
        s_of = dict(zip(p_all.tolist(), s_all.tolist()))
        m = int((want >= 0).sum())
        assert np.array_equal(out_score[b, :m], np.array([s_of[p] for p in want[:m]], dtype=np.float32))
        assert np.all(np.isneginf(out_score[b, m:]))


def test_lse_combine_matches_oracle(fk):
    rng = np.random.default_rng(52)
    R, B, H, d = 4, 3, 64, 512
    outs = rng.normal(0, 1, (R, B, H, d)).astype(np.float32)
    lses = rng.normal(5, 3, (R, B, H)).astype(np.float32)
    lses[1, 0] = -np.inf          # a part without rows
    lses[:, 2, :5] = -np.inf      # heads with no row anywhere
    outs[:, 2, :5] = 0
    out, lse = fk.lse_combine(torch.from_numpy(outs).to(DEV), torch.from_numpy(lses).to(DEV))
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        ro, rl = O.attn_lse_merge(outs[:, b].astype(np.float64), lses[:, b].astype(np.float64))
        fin = np.isfinite(rl)
        assert np.allclose(out[b], ro, rtol=1e-5, atol=1e-6)
        assert np.allclose(lse[b][fin], rl[fin], rtol=1e-6, atol=1e-5) and np.all(np.isneginf(lse[b][~fin]))


@pytest.mark.parametrize("world", [2, 3])
def test_context_sharded_step_emulated_on_one_gpu(fk, world):
    """The sharded protocol with the library's kernels, its ranks run one after another on
    one GPU (no rank waits on another: the exchanges are stacks of the ranks' outputs)."""
    from fp4_sparse_attention_kv_b200 import shard
    B, cap, H, K, d = 3, 20000, 64, 512, 512
    lens = [20000, 13001, 3000]
    q_idx, w, keys = _indexer_inputs(53, B, cap, 32, True)
    x = P.kv_rows_dev(53, 0, B, cap, d, DEV)
    packed = torch.empty((B, cap, d // 2), dtype=torch.uint8, device=DEV)
    scales = torch.empty((B, cap, d // 16), dtype=torch.uint8, device=DEV)
    fk.kv_quant_fp4(x.view(B * cap, d), packed.view(B * cap, d // 2), scales.view(B * cap, d // 16))
    del x
    q = synth.attn_query(53, 0, B, H, d, device=DEV)
    ops = shard.LibraryOps(fk)
    ranges = [shard.shard_range(cap, r, world) for r in range(world)]
    p1 = [shard.local_topk_phase(ops, world, r, cap, lens, q_idx, w, keys[:, lo:hi].contiguous(), K)
          for r, (lo, hi) in enumerate(ranges)]
    all_idx = torch.stack([p[1] for p in p1])
    all_score = torch.stack([p[2] for p in p1])
    idxs, outs, lses = [], [], []
    for r, (lo, hi) in enumerate(ranges):
        i, o, l = shard.merge_attend_phase(ops, world, r, cap, all_score, all_idx, K, q,
                                           packed[:, lo:hi].contiguous(), scales[:, lo:hi].contiguous(), p1[r][0], 1.0)
        idxs.append(i.cpu().numpy())
        outs.append(o)
        lses.append(l)
    out, lse = ops.combine(torch.stack(outs), torch.stack(lses))
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for r in range(1, world):
        assert np.array_equal(idxs[r], idxs[0])
    qh = P.to_f64(q.cpu())
    for b in range(B):
        L = lens[b]
        sc = P.oracle_scores_seq(q_idx[b], w[b], keys[b], L)
        P.check_topk(idxs[0][b], sc, np.arange(L), K, f"sharded top-K b={b}")
        sel = idxs[0][b][idxs[0][b] >= 0]
        pk, s8 = O.kv_quant_fp4(P.kv_rows_host(53, 0, b, sel, d))
        ro, rl = O.sparse_attn_decode_rows(qh[b], O.kv_dequant_fp4(pk, s8), 1.0)
        P.check_attn(out[b], lse[b], ro, rl, f"sharded attention b={b}")
