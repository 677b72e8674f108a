"""Parity at the full workload sizes, in the launch configuration the bench times.

bench.py's own workload classes build the data (the whole cache, quantized by the library)
and run one step exactly as the bench does; sampled sequences are then checked against the
oracle. The oracle regenerates every input it needs from the seeded generator (the FP4 rows
it attends over are quantized by the oracle itself, never read back from the GPU cache), so
nothing it consumes comes from the CUDA path except the selections whose consumers are
being checked (the attention is checked over the GPU's indices; the Reindex layer over the
GPU's pool), each of which is itself checked against the oracle first.
"""
import os
import sys

import numpy as np
import pytest
import torch

from oracle import fp4kv_oracle as O
from tests import parity as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu
D = 512


@pytest.fixture(scope="module")
def fk(cuda_lib):
    import fp4_sparse_attention_kv_b200 as fk
    return fk


def _attn_check(seed, layer, b, q_b, idx_b, seq_len, new_row, out_b, lse_b, what):
    """Oracle attention of one sequence over the given selection; rows regenerated on the
    host and quantized by the oracle; row seq_len - 1 is the row the step wrote."""
    sel = np.asarray(idx_b, dtype=np.int64)
    sel = sel[(sel >= 0) & (sel < seq_len)]
    rows = P.kv_rows_host(seed, layer, b, sel, D)
    last = sel == seq_len - 1
    if last.any():
        rows[last] = new_row
    pk, sc = O.kv_quant_fp4(rows)
    ro, rl = O.sparse_attn_decode_rows(P.to_f64(q_b.cpu()), O.kv_dequant_fp4(pk, sc), 1.0)
    P.check_attn(out_b, lse_b, ro, rl, what)


def _new_row_check(wl, b, layer_packed, layer_scales, x_new, what):
    pk, sc = O.kv_quant_fp4(P.to_f64(x_new[b:b + 1].cpu()))
    assert np.array_equal(layer_packed[b, wl.cap - 1].cpu().numpy(), pk[0]), what
    assert np.array_equal(layer_scales[b, wl.cap - 1].cpu().numpy(), sc[0]), what


@pytest.mark.timeout(900)
@pytest.mark.parametrize("name,seqs", [("decode32", (0, 17, 31)), ("long", (0, 3))])
def test_decode_step_at_full_size(fk, name, seqs):
    cfg = bench.CONFIGS[name]
    wl = bench.DecodeWorkload(cfg, fk, torch.device("cuda"))
    wl.step()
    torch.cuda.synchronize()
    idx = wl.idx.cpu().numpy()
    out, lse = wl.out.cpu().numpy(), wl.lse.cpu().numpy()
    seed = cfg["seed"]
    for b in seqs:
        sc = P.oracle_scores_seq(wl.qi[b], wl.w[b], wl.keys[b], wl.cap)
        P.check_topk(idx[b], sc, np.arange(wl.cap), wl.K, f"{name} top-K b={b}")
        new_row = P.to_f64(wl.x_new[b].cpu())
        _attn_check(seed, 0, b, wl.q[b], idx[b], wl.cap, new_row, out[b], lse[b], f"{name} attention b={b}")
        _new_row_check(wl, b, wl.packed, wl.scales, wl.x_new, f"{name} new row b={b}")


@pytest.mark.timeout(1200)
def test_hierarchical_step_at_full_size(fk):
    cfg = bench.CONFIGS["hier"]
    wl = bench.HierWorkload(cfg, fk, torch.device("cuda"))
    wl.step()
    torch.cuda.synchronize()
    seed, b, cap, K, npb = cfg["seed"], 0, wl.cap, wl.K, wl.npb
    # layer 1 (Full): flat top-K and the pool of the best blocks
    sc = P.oracle_scores_seq(wl.qi[0][b], wl.w[0][b], wl.keys[b], cap)
    P.check_topk(wl.idx[0][b].cpu().numpy(), sc, np.arange(cap), K, "Full top-K")
    bm = O.block_max(sc, cap, 8)
    pool = wl.pool[b].cpu().numpy()
    P.check_topk(pool, bm, np.arange(bm.size), npb, "pool")
    # layer 2 (Reindex): this layer's query scored inside the pool
    pos = O.pool_positions(pool, cap, 8)
    sc2 = P.oracle_scores_seq(wl.qi[1][b], wl.w[1][b], wl.keys[b], cap)[pos]
    idx1 = wl.idx[1][b].cpu().numpy()
    P.check_topk(idx1, sc2, pos, K, "Reindex top-K")
    # attention of layers 1, 2 (over their own indices) and 3 (Reuse: layer 2's indices)
    # (the step wrote every layer's new row with one call: x_new is [layers * B, d], layer-major)
    for layer, sel in ((0, wl.idx[0][b]), (1, wl.idx[1][b]), (2, wl.idx[1][b]), (19, wl.idx[19][b])):
        x_layer = wl.x_new[layer * wl.B:(layer + 1) * wl.B]
        new_row = P.to_f64(x_layer[b].cpu())
        _attn_check(seed, layer, b, wl.q[layer][b], sel.cpu().numpy(), cap, new_row,
                    wl.out[layer][b].cpu().numpy(), wl.lse[layer][b].cpu().numpy(),
                    f"hier layer {layer + 1} attention")
        _new_row_check(wl, b, wl.packed[layer], wl.scales[layer], x_layer, f"hier layer {layer + 1} new row")


@pytest.mark.timeout(900)
def test_quant_sweep_at_full_size_sampled_rows(fk):
    cfg = bench.CONFIGS["quant"]
    wl = bench.QuantWorkload(cfg, fk, torch.device("cuda"))
    wl.step()
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(wl.n, size=4096, replace=False))
    rows_t = torch.as_tensor(rows, device="cuda")
    pk, sc = O.kv_quant_fp4(P.to_f64(wl.x[rows_t].cpu()))
    assert np.array_equal(wl.packed[rows_t].cpu().numpy(), pk)
    assert np.array_equal(wl.scales[rows_t].cpu().numpy(), sc)


@pytest.mark.timeout(1200)
def test_csa2_decoder_step_at_full_size(fk):
    cfg = bench.CONFIGS["csa2_decoder"]
    wl = bench.Csa2DecoderWorkload(cfg, fk, torch.device("cuda"))
    wl.step()
    torch.cuda.synchronize()
    seed, b, cap, K, npb, G = cfg["seed"], 0, wl.cap, wl.K, wl.npb, wl.G
    # layer 1 (Full): flat top-K 512 and the pool of 2048 blocks
    sc = P.oracle_scores_seq(wl.qi[0][b], wl.w[0][b], wl.keys[b], cap)
    P.check_topk(wl.idx[0][b].cpu().numpy(), sc, np.arange(cap), K, "Full top-K")
    pool = wl.pool[b].cpu().numpy()
    P.check_topk(pool, O.block_max(sc, cap, 8), np.arange((cap + 7) // 8), npb, "pool")
    # the Reindex layers of the second and the last group, inside the pool
    pos = O.pool_positions(pool, cap, 8)
    for g in (1, len(wl.qi) - 1):
        sc2 = P.oracle_scores_seq(wl.qi[g][b], wl.w[g][b], wl.keys[b], cap)[pos]
        P.check_topk(wl.idx[g][b].cpu().numpy(), sc2, pos, K, f"Reindex group {g + 1}")
    # attention over the shared KV: Full, a Reuse of it, a Reindex layer, the last Reuse
    new_row = P.to_f64(wl.x_new[b].cpu())
    for l in (0, G - 1, G, wl.L - 1):
        _attn_check(seed, 0, b, wl.q[l][b], wl.idx[l // G][b].cpu().numpy(), cap, new_row,
                    wl.out[l][b].cpu().numpy(), wl.lse[l][b].cpu().numpy(), f"CSA2 layer {l + 1} attention")
    _new_row_check(wl, b, wl.packed, wl.scales, wl.x_new, "CSA2 new row")


@pytest.mark.timeout(900)
def test_decode_step_with_sliding_window_at_full_size(fk):
    cfg = bench.CONFIGS["decode32_swa"]
    wl = bench.DecodeWorkload(cfg, fk, torch.device("cuda"))
    wl.step()
    torch.cuda.synchronize()
    idx = wl.idx.cpu().numpy()
    out, lse = wl.out.cpu().numpy(), wl.lse.cpu().numpy()
    seed, cap, nw = cfg["seed"], wl.cap, wl.n_win
    for b in (0, 31):
        sc = P.oracle_scores_seq(wl.qi[b], wl.w[b], wl.keys[b], cap)
        P.check_topk(idx[b], sc, np.arange(cap), wl.K, f"top-K b={b}")
        sel = idx[b][(idx[b] >= 0) & (idx[b] < cap)]
        rows = P.kv_rows_host(seed, 0, b, sel, D)
        rows[sel == cap - 1] = P.to_f64(wl.x_new[b].cpu())
        v_sel = O.kv_dequant_fp4(*O.kv_quant_fp4(rows))
        # the window: positions cap - nw .. cap - 1, the last one the row this step wrote
        wrows = P.kv_rows_host(seed, bench.SWA_LAYER, b, np.arange(cap - nw, cap), D)
        wrows[-1] = P.to_f64(wl.x_swa_new[b].cpu())
        v_win = O.e4m3_decode(O.swa_quant_fp8(wrows))
        ro, rl = O.sparse_swa_attn_decode_rows(P.to_f64(wl.q[b].cpu()), v_sel, v_win, 1.0)
        P.check_attn(out[b], lse[b], ro, rl, f"attention + window b={b}")
        slot = (cap - 1) % nw
        assert np.array_equal(wl.swa[b, slot].cpu().numpy(), O.swa_quant_fp8(wrows[-1])), "window write"


@pytest.mark.timeout(1200)
def test_csa2_encoder_step_at_full_size(fk):
    """The pages' encoder schedule: window-only layers 1-2, then 3 groups of 6 (Full + 5
    Reuse) over each group's own 524,288-entry FP4 KV and FP8 keys, top-K 512."""
    cfg = bench.CONFIGS["csa2_encoder"]
    wl = bench.Csa2EncoderWorkload(cfg, fk, torch.device("cuda"))
    wl.step()
    torch.cuda.synchronize()
    seed, cap, K, nw = cfg["seed"], wl.cap, wl.K, wl.n_win
    for b in (0, wl.B - 1):
        # the window-only layers: one softmax over the window's E4M3 rows (this step's row
        # in slot (cap - 1) % nw)
        for l in range(wl.NS):
            wrows = P.kv_rows_host(seed, bench.SWA_LAYER + l, b, np.arange(cap - nw, cap), D)
            wrows[-1] = P.to_f64(wl.x_swa_new[l][b].cpu())
            v_win = O.e4m3_decode(O.swa_quant_fp8(wrows))
            ro, rl = O.sparse_attn_decode_rows(P.to_f64(wl.q[l][b].cpu()), v_win, 1.0)
            P.check_attn(wl.out[l][b].cpu().numpy(), wl.lse[l][b].cpu().numpy(), ro, rl,
                         f"encoder window-only layer {l + 1} b={b}")
        for g in (0, wl.NG - 1):
            src = wl.src[g]
            sc = P.oracle_scores_seq(wl.qi[g][b], wl.w[g][b], wl.keys[g][b], cap)
            idx = wl.idx[g][b].cpu().numpy()
            P.check_topk(idx, sc, np.arange(cap), K, f"encoder group {g + 1} top-K b={b}")
            new_row = P.to_f64(wl.x_new[g][b].cpu())
            for l in (src, src + wl.G - 1):  # the group's Full layer and its last Reuse layer
                _attn_check(seed, src, b, wl.q[l][b], idx, cap, new_row, wl.out[l][b].cpu().numpy(),
                            wl.lse[l][b].cpu().numpy(), f"encoder layer {l + 1} attention b={b}")
            _new_row_check(wl, b, wl.packed[g], wl.scales[g], wl.x_new[g], f"encoder group {g + 1} new row")
