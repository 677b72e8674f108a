"""Python binding of libfp4kv: ctypes marshalling only.

Every function here checks tensor dtypes / devices / shapes, passes raw pointers and the
current CUDA stream to the C ABI declared in ``include/fp4kv.h``, and raises
``Fp4kvError`` on a non-zero status. No arithmetic of the method is done here, and there
is no fallback: if the shared library is missing or cannot be loaded, every call raises.
PyTorch is used only for device memory and streams.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp4kv.so")

KEY_BF16, KEY_E4M3, KEY_E2M1 = 0, 1, 2
OP_KV_QUANT, OP_INDEXER_TOPK, OP_REINDEX_TOPK, OP_HIER_POOL_SELECT, OP_SPARSE_ATTN, \
    OP_INDEXER_SCORES = range(6)

STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA",
                4: "WORKSPACE_TOO_SMALL", 5: "DEVICE_FLAG"}

# (name, restype, argtypes) of every exported symbol
_P, _I32, _I64, _SZ, _F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, \
    ctypes.c_float
SIGNATURES = [
    ("fp4kv_last_error", ctypes.c_char_p, []),
    ("fp4kv_version", ctypes.c_char_p, []),
    ("fp4kv_workspace_bytes", _SZ, [_I32, _I32, _I64, _I32, _I32, _I32]),
    ("fp4kv_workspace_init", ctypes.c_int, [_P, _SZ, _P]),
    ("fp4kv_workspace_status", ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32), _P]),
    ("fp4kv_kv_quant_fp4", ctypes.c_int, [_P, _I64, _I32, _I64, _P, _P, _P, _I64, _P]),
    ("fp4kv_indexer_scores", ctypes.c_int,
     [_P, _P, _I32, _P, _I32, _P, _I64, _P, _I32, _P, _P, _SZ, _P]),
    ("fp4kv_indexer_topk", ctypes.c_int,
     [_P, _P, _I32, _P, _I32, _P, _I64, _P, _I32, _P, _I32, _I32, _I32, _P, _P, _P, _SZ, _P]),
    ("fp4kv_hier_pool_select", ctypes.c_int,
     [_P, _P, _I32, _P, _I32, _P, _I64, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _SZ, _P]),
    ("fp4kv_sparse_attn_decode", ctypes.c_int,
     [_P, _I32, _I32, _I32, _P, _P, _I64, _P, _P, _I32, _F32, _P, _P, _P, _SZ, _P]),
    ("fp4kv_indexer_topk_noalloc", ctypes.c_int,
     [_P, _P, _I32, _P, _I32, _P, _I64, _P, _I32, _P, _I32, _I32, _I32, _P, _P, _P]),
    ("fp4kv_profile_enable", ctypes.c_int, [_I32]),
    ("fp4kv_profile_read", ctypes.c_int, [ctypes.POINTER(_I32), ctypes.POINTER(_F32)]),
    ("fp4kv_selftest_wait_timeout", ctypes.c_int, [_I32, _P, _SZ, _P]),
    ("fp4kv_sparse_swa_attn_decode", ctypes.c_int,
     [_P, _I32, _I32, _I32, _P, _P, _I64, _P, _P, _I32, _P, _I32, _F32, _P, _P, _P, _SZ, _P]),
    ("fp4kv_swa_quant_fp8", ctypes.c_int, [_P, _I64, _I32, _I64, _P, _P, _I64, _P]),
    ("fp4kv_topk_merge", ctypes.c_int, [_P, _P, _I32, _I32, _I32, ctypes.POINTER(_I32), _I32, _I32, _I32, _P,
                                        _P, _P, _P]),
    ("fp4kv_lse_combine", ctypes.c_int, [_P, _P, _I32, _I32, _I32, _I32, _P, _P, _P]),
    ("fp4kv_noalloc_status", ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _P]),
    ("fp4kv_selftest_wait_timeout_noalloc", ctypes.c_int, [_I32, _P]),
]

KERNEL_KINDS = ("kv_quant_fp4", "index_score", "topk_select", "sparse_attn")


class Fp4kvError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libfp4kv {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfp4kv.so (building it first if the sources are newer). Raises if missing."""
    global _lib
    if _lib is None:
        from . import build as _build
        if not _build.up_to_date():
            try:
                _build.build()
            except Exception as e:  # no toolchain on this host: only a prebuilt lib will do
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"libfp4kv.so is missing and could not be built: {e}")
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libfp4kv.so not found at {LIB_PATH}")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise Fp4kvError(status, lib().fp4kv_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, E2M1Planes):
        t = t.buf
    return ctypes.c_void_p(t.data_ptr())


class E2M1Planes:
    """An FP4 indexer operand of shape [B, rows, 128]: E2M1 codes [B][rows][64] followed,
    in the same buffer, by the E4M3 scales [B][rows][8] (the layout of key_dtype E2M1)."""

    DK = 128

    def __init__(self, B: int, rows: int, device):
        self.B, self.rows = int(B), int(rows)
        n = self.B * self.rows
        self.buf = torch.empty(n * (self.DK // 2 + self.DK // 16), dtype=torch.uint8, device=device)
        self.codes = self.buf[:n * (self.DK // 2)].view(self.B, self.rows, self.DK // 2)
        self.scales = self.buf[n * (self.DK // 2):].view(self.B, self.rows, self.DK // 16)

    @property
    def device(self):
        return self.buf.device

    @property
    def shape(self):
        return (self.B, self.rows, self.DK)

    def quantize_from(self, x: torch.Tensor):
        """Fill from bf16 x [B, rows, 128] with the library's FP4 quantizer."""
        if tuple(x.shape) != self.shape:
            raise ValueError(f"x: expected shape {self.shape}, got {tuple(x.shape)}")
        kv_quant_fp4(x.reshape(-1, self.DK), self.codes.view(-1, self.DK // 2),
                     self.scales.view(-1, self.DK // 16))
        return self


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, dtype, name, device=None, contiguous=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def version() -> str:
    return lib().fp4kv_version().decode()


def workspace_bytes(op: int, B: int, cap: int, heads: int = 0, top_k: int = 0,
                    n_pool_blocks: int = 0) -> int:
    return int(lib().fp4kv_workspace_bytes(op, B, cap, heads, top_k, n_pool_blocks))


def workspace_init(ws: torch.Tensor):
    _need(ws, torch.uint8, "ws")
    _check(lib().fp4kv_workspace_init(_ptr(ws), ws.numel(), _stream(ws.device)))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """Allocate (with torch) and zero a workspace of at least nbytes (256-byte aligned)."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    workspace_init(ws)
    return ws


def workspace_status(ws: torch.Tensor) -> int:
    """Read and clear the workspace's device status word (synchronises the stream)."""
    out = ctypes.c_uint32(0)
    st = lib().fp4kv_workspace_status(_ptr(ws), ctypes.byref(out), _stream(ws.device))
    if st not in (0, 5):
        _check(st)
    return int(out.value)


def selftest_wait_timeout(limit_us: int, ws: torch.Tensor):
    """Test hook: a kernel waits on a barrier nothing signals, bounded by limit_us; the
    timeout lands in ws's status word (read it with workspace_status)."""
    _check(lib().fp4kv_selftest_wait_timeout(int(limit_us), _ptr(ws), ws.numel(), _stream(ws.device)))


def kv_quant_fp4(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                 dst_row: torch.Tensor | None = None):
    """Quantize bf16 rows x [n, d] (row stride may exceed d) into packed [cap, d/2] and
    scales [cap, d/16] (uint8), at rows dst_row (int64 [n]) or 0..n-1."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise TypeError("x: expected a CUDA bf16 [n, d] tensor with unit column stride")
    _need(packed, torch.uint8, "packed", x.device)
    _need(scales, torch.uint8, "scales", x.device)
    n, d = x.shape
    cap = packed.numel() // (d // 2)
    if packed.numel() != cap * (d // 2) or scales.numel() < cap * (d // 16):
        raise ValueError("packed / scales do not match d")
    if dst_row is not None:
        _need(dst_row, torch.int64, "dst_row", x.device)
    _check(lib().fp4kv_kv_quant_fp4(_ptr(x), n, d, x.stride(0), _ptr(dst_row), _ptr(packed),
                                    _ptr(scales), cap, _stream(x.device)))


def _key_dtype(keys):
    if isinstance(keys, E2M1Planes):
        return KEY_E2M1
    if keys.dtype == torch.uint8:
        return KEY_E4M3
    if keys.dtype == torch.bfloat16:
        return KEY_BF16
    raise TypeError("keys: expected uint8 (E4M3 codes), bf16 or E2M1Planes")


def _check_indexer(q, w, keys, seq_lens, key_scale):
    kd = _key_dtype(keys)
    if kd == KEY_E2M1:
        if not isinstance(q, E2M1Planes) or q.device != keys.device:
            raise TypeError("q: expected E2M1Planes on the keys' device (keys are E2M1Planes)")
    else:
        _need(q, keys.dtype, "q", keys.device)
        _need(keys, keys.dtype, "keys")
    _need(w, torch.float32, "w", keys.device)
    _need(seq_lens, torch.int32, "seq_lens", keys.device)
    if key_scale is not None:
        _need(key_scale, torch.float32, "key_scale", keys.device)
    B, cap, dk = keys.shape
    if dk != 128 or q.shape[0] != B or q.shape[2] != 128 or w.shape != q.shape[:2]:
        raise ValueError("shapes: keys [B, cap, 128], q [B, H_I, 128], w [B, H_I]")
    return kd, B, cap, q.shape[1]


def indexer_scores(q, w, keys, seq_lens, key_scale=None, ws=None):
    """fp32 scores [B, cap] of every visible entry (entries >= seq_len are left as -inf)."""
    kd, B, cap, H_I = _check_indexer(q, w, keys, seq_lens, key_scale)
    out = torch.full((B, cap), float("-inf"), dtype=torch.float32, device=keys.device)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(OP_INDEXER_SCORES, B, cap), keys.device)
    _check(lib().fp4kv_indexer_scores(_ptr(q), _ptr(w), H_I, _ptr(keys), kd, _ptr(key_scale),
                                      cap, _ptr(seq_lens), B, _ptr(out), _ptr(ws), ws.numel(),
                                      _stream(keys.device)))
    return out


def indexer_topk(q, w, keys, seq_lens, top_k, pool=None, block_size=8, key_scale=None,
                 ws=None, out_idx=None, out_score=None):
    """Full mode (pool None) or Reindex mode (pool [B, n_pool_blocks] int32). Returns
    out_idx int32 [B, top_k] (and fills out_score if given)."""
    kd, B, cap, H_I = _check_indexer(q, w, keys, seq_lens, key_scale)
    npb = 0
    if pool is not None:
        _need(pool, torch.int32, "pool", keys.device)
        npb = pool.shape[1]
    op = OP_REINDEX_TOPK if pool is not None else OP_INDEXER_TOPK
    if out_idx is None:
        out_idx = torch.empty((B, top_k), dtype=torch.int32, device=keys.device)
    _need(out_idx, torch.int32, "out_idx", keys.device)
    if out_score is not None:
        _need(out_score, torch.float32, "out_score", keys.device)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(op, B, cap, H_I, top_k, npb), keys.device)
    _check(lib().fp4kv_indexer_topk(_ptr(q), _ptr(w), H_I, _ptr(keys), kd, _ptr(key_scale), cap,
                                    _ptr(seq_lens), B, _ptr(pool), npb, block_size, top_k,
                                    _ptr(out_idx), _ptr(out_score), _ptr(ws), ws.numel(),
                                    _stream(keys.device)))
    return out_idx


def hier_pool_select(q, w, keys, seq_lens, top_k, n_pool_blocks, block_size=8,
                     key_scale=None, ws=None, out_idx=None, out_pool=None, out_score=None):
    """First Full decoder layer: returns (out_idx [B, top_k], out_pool [B, n_pool_blocks])."""
    kd, B, cap, H_I = _check_indexer(q, w, keys, seq_lens, key_scale)
    dev = keys.device
    if out_idx is None:
        out_idx = torch.empty((B, top_k), dtype=torch.int32, device=dev)
    if out_pool is None:
        out_pool = torch.empty((B, n_pool_blocks), dtype=torch.int32, device=dev)
    _need(out_idx, torch.int32, "out_idx", dev)
    _need(out_pool, torch.int32, "out_pool", dev)
    if out_score is not None:
        _need(out_score, torch.float32, "out_score", dev)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(OP_HIER_POOL_SELECT, B, cap, H_I, top_k,
                                             n_pool_blocks), dev)
    _check(lib().fp4kv_hier_pool_select(_ptr(q), _ptr(w), H_I, _ptr(keys), kd, _ptr(key_scale),
                                        cap, _ptr(seq_lens), B, top_k, block_size, n_pool_blocks,
                                        _ptr(out_idx), _ptr(out_pool), _ptr(out_score), _ptr(ws),
                                        ws.numel(), _stream(dev)))
    return out_idx, out_pool


def sparse_attn_decode(q, packed, scales, seq_lens, idx, sm_scale=1.0, ws=None, out=None,
                       lse=None, want_lse=True, swa=None):
    """q bf16 [B, H, d]; packed uint8 [B, cap, d/2]; scales uint8 [B, cap, d/16];
    idx int32 [B, top_k]; swa (optional) uint8 [B, n_win, d] E4M3 sliding-window rows, attended
    in the same softmax. Returns (out fp32 [B, H, d], lse fp32 [B, H] or None)."""
    _need(q, torch.bfloat16, "q")
    dev = q.device
    _need(packed, torch.uint8, "packed", dev)
    _need(scales, torch.uint8, "scales", dev)
    _need(seq_lens, torch.int32, "seq_lens", dev)
    _need(idx, torch.int32, "idx", dev)
    B, H, d = q.shape
    cap = packed.shape[1]
    if packed.shape != (B, cap, d // 2) or scales.shape != (B, cap, d // 16):
        raise ValueError("packed [B, cap, d/2] and scales [B, cap, d/16] expected")
    top_k = idx.shape[1]
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    if ws is None:
        ws = alloc_workspace(workspace_bytes(OP_SPARSE_ATTN, B, cap, H, top_k), dev)
    if swa is None:
        _check(lib().fp4kv_sparse_attn_decode(_ptr(q), B, H, d, _ptr(packed), _ptr(scales), cap,
                                              _ptr(seq_lens), _ptr(idx), top_k, float(sm_scale),
                                              _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                              _stream(dev)))
    else:
        _need(swa, torch.uint8, "swa", dev)
        if swa.dim() != 3 or swa.shape[0] != B or swa.shape[2] != d:
            raise ValueError("swa: expected uint8 [B, n_win, d]")
        _check(lib().fp4kv_sparse_swa_attn_decode(_ptr(q), B, H, d, _ptr(packed), _ptr(scales), cap,
                                                  _ptr(seq_lens), _ptr(idx), top_k, _ptr(swa),
                                                  swa.shape[1], float(sm_scale), _ptr(out), _ptr(lse),
                                                  _ptr(ws), ws.numel(), _stream(dev)))
    return out, lse


def swa_quant_fp8(x: torch.Tensor, out: torch.Tensor, dst_row: torch.Tensor | None = None):
    """E4M3 codes of bf16 rows x [n, d] into out [cap, d] (uint8), at rows dst_row (int64
    [n]) or 0..n-1: the sliding-window KV's write."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise TypeError("x: expected a CUDA bf16 [n, d] tensor with unit column stride")
    _need(out, torch.uint8, "out", x.device)
    n, d = x.shape
    cap = out.numel() // d
    if out.numel() != cap * d:
        raise ValueError("out does not match d")
    if dst_row is not None:
        _need(dst_row, torch.int64, "dst_row", x.device)
    _check(lib().fp4kv_swa_quant_fp8(_ptr(x), n, d, x.stride(0), _ptr(dst_row), _ptr(out), cap,
                                     _stream(x.device)))


def profile_enable(on: bool = True):
    """Bracket every library kernel launch with CUDA events (benchmarks only)."""
    _check(lib().fp4kv_profile_enable(1 if on else 0))


def profile_read() -> dict:
    """{kernel kind: (launches, total device ms)} since the last read; clears the records."""
    n = (ctypes.c_int32 * 4)()
    ms = (ctypes.c_float * 4)()
    _check(lib().fp4kv_profile_read(n, ms))
    return {KERNEL_KINDS[i]: (int(n[i]), float(ms[i])) for i in range(4)}


def indexer_topk_noalloc(q, w, keys, seq_lens, top_k, pool=None, block_size=8, key_scale=None,
                         out_idx=None, out_score=None):
    """Same as ``indexer_topk`` but without a workspace: the library uses its own fixed 8 MiB
    device scratch (for callers that cannot allocate device memory). Calls on one device
    must not overlap on the GPU. Output tensors, when not given, are allocated here by torch
    for convenience; pass them to keep the call itself allocation-free."""
    kd, B, cap, H_I = _check_indexer(q, w, keys, seq_lens, key_scale)
    npb = 0
    if pool is not None:
        _need(pool, torch.int32, "pool", keys.device)
        npb = pool.shape[1]
    if out_idx is None:
        out_idx = torch.empty((B, top_k), dtype=torch.int32, device=keys.device)
    _need(out_idx, torch.int32, "out_idx", keys.device)
    if out_score is not None:
        _need(out_score, torch.float32, "out_score", keys.device)
    _check(lib().fp4kv_indexer_topk_noalloc(_ptr(q), _ptr(w), H_I, _ptr(keys), kd, _ptr(key_scale),
                                            cap, _ptr(seq_lens), B, _ptr(pool), npb, block_size,
                                            top_k, _ptr(out_idx), _ptr(out_score),
                                            _stream(keys.device)))
    return out_idx


def noalloc_status(device=None) -> int:
    """Read and clear the status word of the allocation-free entry point's scratch on the
    current device (synchronises the device's current stream)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    out = ctypes.c_uint32(0)
    st = lib().fp4kv_noalloc_status(ctypes.byref(out), _stream(dev))
    if st not in (0, 5):
        _check(st)
    return int(out.value)


def selftest_wait_timeout_noalloc(limit_us: int, device=None):
    """Test hook: selftest_wait_timeout on the allocation-free entry point's scratch (read
    the result with noalloc_status)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check(lib().fp4kv_selftest_wait_timeout_noalloc(int(limit_us), _stream(dev)))


def topk_merge(cand_score: torch.Tensor, cand_idx: torch.Tensor, part_base, top_k: int,
               local_range=None, out_idx=None, out_local=None, out_score=None):
    """Exact top-K of the union of per-part candidate lists. cand_score fp32 / cand_idx int32
    [n_parts, B, k_part] (range-local positions, -1 absent); part_base: the first global
    position of each part's range (host ints). Returns (out_idx [B, top_k] global positions
    ascending, out_local [B, top_k] positions local to local_range=(lo, hi) or None)."""
    _need(cand_score, torch.float32, "cand_score")
    _need(cand_idx, torch.int32, "cand_idx", cand_score.device)
    R, B, k_part = cand_idx.shape
    if tuple(cand_score.shape) != (R, B, k_part) or len(part_base) != R:
        raise ValueError("cand_score / cand_idx must be [n_parts, B, k_part] with one base per part")
    dev = cand_idx.device
    if out_idx is None:
        out_idx = torch.empty((B, top_k), dtype=torch.int32, device=dev)
    _need(out_idx, torch.int32, "out_idx", dev)
    lo, hi = (0, 0) if local_range is None else (int(local_range[0]), int(local_range[1]))
    if local_range is not None and out_local is None:
        out_local = torch.empty((B, top_k), dtype=torch.int32, device=dev)
    if out_local is not None:
        _need(out_local, torch.int32, "out_local", dev)
    if out_score is not None:
        _need(out_score, torch.float32, "out_score", dev)
    bases = (_I32 * R)(*[int(x) for x in part_base])
    _check(lib().fp4kv_topk_merge(_ptr(cand_score), _ptr(cand_idx), R, k_part, B, bases, top_k, lo, hi,
                                  _ptr(out_idx), _ptr(out_local), _ptr(out_score), _stream(dev)))
    return out_idx, out_local


def lse_combine(part_out: torch.Tensor, part_lse: torch.Tensor, out=None, lse=None):
    """Attention over the union of disjoint row sets from the parts: part_out fp32
    [R, B, H, d], part_lse fp32 [R, B, H]. Returns (out [B, H, d], lse [B, H])."""
    _need(part_out, torch.float32, "part_out")
    _need(part_lse, torch.float32, "part_lse", part_out.device)
    R, B, H, d = part_out.shape
    if tuple(part_lse.shape) != (R, B, H):
        raise ValueError("part_lse must be [R, B, H]")
    dev = part_out.device
    if out is None:
        out = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    _check(lib().fp4kv_lse_combine(_ptr(part_out), _ptr(part_lse), R, B, H, d, _ptr(out), _ptr(lse), _stream(dev)))
    return out, lse
