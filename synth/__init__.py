"""Seeded synthetic inputs shared by the tests, the bench and the CPU oracle runs.

This module holds no step of the method: it only draws numbers. Every value is a pure
function of (seed, stream, row, column) through a counter-based 32-bit integer hash, so
the same call gives bit-identical tensors on the CPU and on a GPU, and any single row of
a huge cache can be regenerated on the host without storing the cache.

Integer arithmetic is done on int64 tensors holding values in [0, 2^32); every multiplier
is below 2^31, so no product overflows int64. A normal deviate is a lookup into a 65,536-
entry bf16 table of N(0,1) quantiles built once on the host (``torch.special.ndtri`` in
fp64, then rounded to bf16); its tails reach about +-4.17.

Workload shapes (the value distributions are the same for every configuration):

* KV rows: bf16 N(0,1), d channels; 1 % of the channels (round(0.01 d), chosen by the hash
  per layer) are multiplied by 20; optionally a fraction of rows (chosen by the hash) is
  multiplied by 100 to exercise saturation.
* Attention query: bf16 N(0,1) / sqrt(d).
* Indexer keys: bf16 N(0,1), optionally cast to FP8 E4M3 (round-to-nearest-even).
* Indexer query: N(0,1) / sqrt(dk), either kept in bf16 or quantized per head to FP8 E4M3
  with scale amax / 448; the scale is folded into the head weight.
* Head weights: U(0.5, 1.5) / H_I.
"""
from __future__ import annotations

import math

import torch

MASK32 = 0xFFFFFFFF
_M1 = 0x7FEB352D
_M2 = 0x2C1B3C6D
_M3 = 0x6B43A9B5 & 0x7FFFFFFF
_GOLD = 0x61C88647

# Stream ids: one per kind of tensor.
S_KV, S_Q, S_KEYS, S_QI, S_W, S_OUTLIER, S_HEAVY, S_MISC = range(1, 9)


def _mix32(x: torch.Tensor) -> torch.Tensor:
    """Avalanche mix of 32-bit values held in int64 (xorshift-multiply rounds)."""
    x = x ^ (x >> 16)
    x = (x * _M1) & MASK32
    x = x ^ (x >> 15)
    x = (x * _M2) & MASK32
    x = x ^ (x >> 16)
    return x


def _key(seed: int, stream: int, *ids: int) -> int:
    """Scalar stream key from the seed, a stream id and further small ids."""
    k = torch.tensor([(seed * 0x9E3779B1 + 0x85EBCA6B) & MASK32], dtype=torch.int64)
    k = _mix32(k ^ (stream & MASK32))
    for i in ids:
        k = _mix32((k + ((int(i) * _M3) & MASK32)) & MASK32)
    return int(k.item())


def hash_rows_cols(key: int, rows: torch.Tensor, ncols: int) -> torch.Tensor:
    """h[r, c] = mix(mix(key ^ mix(row_r)) ^ (c * golden)), int64 in [0, 2^32)."""
    rows = rows.to(torch.int64)
    rk = _mix32((_mix32(rows & MASK32) ^ key) & MASK32)
    ck = (torch.arange(ncols, dtype=torch.int64, device=rows.device) * _GOLD) & MASK32
    return _mix32(rk[:, None] ^ ck[None, :])


_NORMAL_TABLES = {}


def normal_table(device) -> torch.Tensor:
    """65,536 bf16 N(0,1) quantiles: ndtri((i + 0.5) / 65536), fp64 then bf16."""
    key = str(torch.device(device))
    if key not in _NORMAL_TABLES:
        if "cpu" not in _NORMAL_TABLES:
            p = (torch.arange(65536, dtype=torch.float64) + 0.5) / 65536.0
            _NORMAL_TABLES["cpu"] = torch.special.ndtri(p).to(torch.bfloat16)
        _NORMAL_TABLES[key] = _NORMAL_TABLES["cpu"].to(device)
    return _NORMAL_TABLES[key]


def normal_bf16(h: torch.Tensor) -> torch.Tensor:
    """Hash values -> bf16 N(0,1) through the quantile table (top 16 bits)."""
    return normal_table(h.device)[(h >> 16)]


def uniform01(h: torch.Tensor) -> torch.Tensor:
    """Hash values -> fp64 in [0, 1)."""
    return h.to(torch.float64) / 4294967296.0


def outlier_channels(seed: int, layer: int, d: int, frac: float = 0.01) -> torch.Tensor:
    """round(frac * d) distinct channels chosen by the hash for this (seed, layer)."""
    n = int(round(frac * d))
    if n == 0:
        return torch.zeros(0, dtype=torch.int64)
    k = _key(seed, S_OUTLIER, layer)
    h = _mix32((torch.arange(d, dtype=torch.int64) * _GOLD ^ k) & MASK32)
    return torch.argsort(h, stable=True)[:n].sort().values


def kv_rows(seed: int, layer: int, seq: int, rows: torch.Tensor, d: int,
            outlier_mult: float = 20.0, heavy_frac: float = 0.0,
            heavy_mult: float = 100.0) -> torch.Tensor:
    """bf16 KV rows [len(rows), d] for (seed, layer, sequence); rows are row numbers."""
    dev = rows.device
    h = hash_rows_cols(_key(seed, S_KV, layer, seq), rows, d)
    x = normal_bf16(h).to(torch.float32)
    mult = torch.ones(d, dtype=torch.float32, device=dev)
    oc = outlier_channels(seed, layer, d)
    if oc.numel():
        mult[oc.to(dev)] = outlier_mult
    x = x * mult[None, :]
    if heavy_frac > 0:
        hr = _mix32((_mix32(rows.to(torch.int64) & MASK32) ^ _key(seed, S_HEAVY, layer, seq))
                    & MASK32)
        heavy = uniform01(hr) < heavy_frac
        x = torch.where(heavy[:, None], x * heavy_mult, x)
    return x.to(torch.bfloat16)


def attn_query(seed: int, layer: int, B: int, H: int, d: int, device="cpu") -> torch.Tensor:
    """bf16 [B, H, d] attention queries, N(0,1) / sqrt(d). Drawn on the host (small) and
    copied, so every device gets the same bits."""
    rows = torch.arange(B * H, dtype=torch.int64)
    h = hash_rows_cols(_key(seed, S_Q, layer), rows, d)
    x = normal_bf16(h).to(torch.float32) * (1.0 / math.sqrt(d))
    return x.to(torch.bfloat16).reshape(B, H, d).to(device)


def indexer_keys(seed: int, seq: int, rows: torch.Tensor, dk: int = 128,
                 fp8: bool = True, source: int = 0) -> torch.Tensor:
    """Indexer keys [len(rows), dk]: bf16 N(0,1), cast to FP8 E4M3 when fp8 (returned as
    uint8 codes), else bf16. `source` selects the key set of one KV source layer (0: the
    stream every single-source workload uses)."""
    key = _key(seed, S_KEYS, seq) if source == 0 else _key(seed, S_KEYS, seq, source)
    h = hash_rows_cols(key, rows, dk)
    k = normal_bf16(h)
    if fp8:
        return k.to(torch.float8_e4m3fn).view(torch.uint8)
    return k


def indexer_query(seed: int, layer: int, B: int, H_I: int, dk: int = 128, fp8: bool = True,
                  device="cpu"):
    """Indexer query and head weights for a batch.

    Returns (q [B, H_I, dk] as uint8 E4M3 codes when fp8 else bf16, w [B, H_I] fp32).
    With fp8 the query is quantized per (b, h) with scale amax / 448 and the scale is
    multiplied into w (exact: a positive scale commutes with max(0, .)). Drawn on the host
    (small) and copied, so every device gets the same bits."""
    rows = torch.arange(B * H_I, dtype=torch.int64)
    h = hash_rows_cols(_key(seed, S_QI, layer), rows, dk)
    q = (normal_bf16(h).to(torch.float32) * (1.0 / math.sqrt(dk))).reshape(B, H_I, dk)
    hw = hash_rows_cols(_key(seed, S_W, layer), torch.arange(B, dtype=torch.int64), H_I)
    w = ((0.5 + uniform01(hw)) / H_I).to(torch.float32)
    if not fp8:
        return q.to(torch.bfloat16).to(device), w.to(device)
    amax = q.abs().amax(dim=2).clamp_min(1e-30)
    scale = amax / 448.0
    q8 = (q / scale[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return q8.to(device), (w * scale).to(torch.float32).to(device)
