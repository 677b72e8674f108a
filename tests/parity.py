"""Shared helpers for the GPU parity tests: comparisons against the oracle under the stated
tolerances, and builders for seeded inputs (through ``synth``) on the device and the host.

Tolerances (the contract the GPU path is held to):
* packed FP4 bytes and E4M3 scale bytes: bit-exact;
* top-K indices and pool blocks: exact, except entries whose oracle score lies within
  1e-5 relative of the K-th oracle score (those may be swapped with each other);
* attention output: relative L2 <= 1e-3 and max-abs <= 5e-3 per sequence; lse within
  1e-4 absolute (-inf where the oracle gives -inf).
"""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import fp4kv_oracle as O

TOPK_REL = 1e-5
ATTN_REL_L2 = 1e-3
ATTN_MAX_ABS = 5e-3
LSE_ABS = 1e-4


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 values of a bf16 tensor, or of FP8 E4M3 codes held as uint8."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return O.bf16_bits_to_f64(t.view(torch.int16).numpy().astype(np.uint16))
    if t.dtype == torch.uint8:
        return O.fp8_e4m3_to_f64(t.numpy())
    return t.numpy().astype(np.float64)


def check_topk(gpu_idx, scores, positions, k, what="top-k"):
    """gpu_idx: np int [k]; scores (fp32) at `positions`. Exact up to the tie band."""
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    positions = np.asarray(positions, dtype=np.int64)
    scores = np.asarray(scores, dtype=np.float32)
    n = positions.size
    m = min(k, n)
    want = O.topk_positions(scores, positions, k)
    # structure: ascending, unique, valid positions, padding
    sel = gpu_idx[:m]
    assert np.all(gpu_idx[m:] == -1), f"{what}: padding"
    assert np.all(np.diff(sel) > 0), f"{what}: not strictly ascending"
    assert np.isin(sel, positions).all(), f"{what}: position outside the scored set"
    if np.array_equal(gpu_idx, want):
        return 0
    s_of = dict(zip(positions.tolist(), scores.astype(np.float64).tolist()))
    sk = np.sort(scores.astype(np.float64))[::-1][m - 1]
    tol = TOPK_REL * max(abs(sk), 1e-30)
    extra = set(sel.tolist()) - set(want[:m].tolist())
    missing = set(want[:m].tolist()) - set(sel.tolist())
    for p in extra | missing:
        assert abs(s_of[p] - sk) <= tol, (
            f"{what}: position {p} (score {s_of[p]!r}) differs from the oracle outside the "
            f"tie band around the K-th score {sk!r}")
    return len(extra)


def check_attn(out, lse, ref_out, ref_lse, what="attn"):
    out = np.asarray(out, dtype=np.float64)
    ref_out = np.asarray(ref_out, dtype=np.float64)
    diff = out - ref_out
    nrm = np.linalg.norm(ref_out)
    rel = np.linalg.norm(diff) / nrm if nrm > 0 else np.linalg.norm(diff)
    mx = np.abs(diff).max() if diff.size else 0.0
    assert rel <= ATTN_REL_L2, f"{what}: relative L2 {rel:.3e}"
    assert mx <= ATTN_MAX_ABS, f"{what}: max abs {mx:.3e}"
    if lse is not None:
        lse = np.asarray(lse, dtype=np.float64)
        ref_lse = np.asarray(ref_lse, dtype=np.float64)
        inf = np.isneginf(ref_lse)
        assert np.array_equal(np.isneginf(lse), inf), f"{what}: lse -inf pattern"
        if (~inf).any():
            assert np.abs(lse[~inf] - ref_lse[~inf]).max() <= LSE_ABS, f"{what}: lse"
    return rel, mx


# ----------------------------------------------------------------------------------------
# Input builders (the generator runs identically on the device and on the host)
# ----------------------------------------------------------------------------------------

def kv_rows_dev(seed, layer, B, cap, d, device, heavy=0.0):
    """bf16 [B, cap, d] KV rows on the device."""
    x = torch.empty((B, cap, d), dtype=torch.bfloat16, device=device)
    rows = torch.arange(cap, dtype=torch.int64, device=device)
    for b in range(B):
        x[b] = synth.kv_rows(seed, layer, b, rows, d, heavy_frac=heavy)
    return x


def kv_rows_host(seed, layer, b, positions, d, heavy=0.0):
    rows = torch.as_tensor(np.asarray(positions, dtype=np.int64))
    return to_f64(synth.kv_rows(seed, layer, b, rows, d, heavy_frac=heavy))


def keys_dev(seed, B, cap, fp8, device, dk=128):
    dt = torch.uint8 if fp8 else torch.bfloat16
    k = torch.empty((B, cap, dk), dtype=dt, device=device)
    rows = torch.arange(cap, dtype=torch.int64, device=device)
    for b in range(B):
        k[b] = synth.indexer_keys(seed, b, rows, dk, fp8)
    return k


def oracle_scores_seq(q, w, keys_b, seq_len, ks=None):
    """Oracle scores of one sequence from device/host tensors (fp32 numpy)."""
    return O.indexer_scores(to_f64(q), w.detach().cpu().double().numpy(),
                            to_f64(keys_b[:seq_len]),
                            None if ks is None else ks[:seq_len].detach().cpu().double().numpy())
