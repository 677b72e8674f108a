"""CPU-only checks of the C-ABI boundary: the shared library builds and loads, exports every
symbol ``include/fp4kv.h`` declares, and rejects bad arguments on the host before any
kernel is launched (no GPU needed: validation happens before the first CUDA call)."""
import ctypes
import os
import re

import pytest

from fp4_sparse_attention_kv_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "fp4kv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp4kv_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    syms = _declared_symbols()
    for name in ("fp4kv_kv_quant_fp4", "fp4kv_indexer_topk", "fp4kv_hier_pool_select",
                 "fp4kv_sparse_attn_decode", "fp4kv_workspace_bytes", "fp4kv_last_error"):
        assert name in syms


def test_library_loads_and_exports_every_declared_symbol():
    L = binding.lib()
    for name in _declared_symbols():
        assert hasattr(L, name), name
    assert set(n for n, _, _ in binding.SIGNATURES) == set(_declared_symbols())
    assert "sm_100a" in binding.version()


def _call(name, *args):
    L = binding.lib()
    st = getattr(L, name)(*args)
    return st, L.fp4kv_last_error().decode()


def test_host_validation_rejects_bad_arguments_without_a_gpu():
    P = ctypes.c_void_p
    fake = P(0x10000)  # never dereferenced: validation fails first
    # null pointers
    st, msg = _call("fp4kv_kv_quant_fp4", None, 4, 512, 512, None, None, None, 4, None)
    assert st == 1 and "null" in msg
    # unsupported d
    st, msg = _call("fp4kv_kv_quant_fp4", fake, 4, 48, 48, None, fake, fake, 4, None)
    assert st == 2 and "d=48" in msg
    # zero rows is a no-op success
    st, msg = _call("fp4kv_kv_quant_fp4", None, 0, 512, 512, None, None, None, 0, None)
    assert st == 0 and msg == ""
    # indexer: H_I out of range, top_k out of range, misaligned keys, bad block size
    st, msg = _call("fp4kv_indexer_topk", fake, fake, 65, fake, 1, None, 100, fake, 1, None, 0,
                    8, 16, fake, None, fake, 1 << 20, None)
    assert st == 2 and "H_I" in msg
    st, msg = _call("fp4kv_indexer_topk", fake, fake, 32, fake, 1, None, 100, fake, 1, None, 0,
                    8, 5000, fake, None, fake, 1 << 20, None)
    assert st == 2 and "top_k" in msg
    st, msg = _call("fp4kv_indexer_topk", fake, fake, 32, P(0x10001), 1, None, 100, fake, 1,
                    None, 0, 8, 16, fake, None, fake, 1 << 20, None)
    assert st == 1 and "aligned" in msg
    st, msg = _call("fp4kv_hier_pool_select", fake, fake, 32, fake, 1, None, 100, fake, 1, 16, 4,
                    8, fake, fake, None, fake, 1 << 20, None)
    assert st == 2 and "block_size" in msg
    # workspace too small
    need = binding.workspace_bytes(binding.OP_INDEXER_TOPK, 1, 100, 32, 16)
    st, msg = _call("fp4kv_indexer_topk", fake, fake, 32, fake, 1, None, 100, fake, 1, None, 0,
                    8, 16, fake, None, fake, need - 1, None)
    assert st == 4 and "ws_bytes" in msg
    # attention: d must be 512, H <= 128
    st, msg = _call("fp4kv_sparse_attn_decode", fake, 1, 16, 256, fake, fake, 10, fake, fake, 4,
                    ctypes.c_float(1.0), fake, None, fake, 1 << 20, None)
    assert st == 2 and "d=256" in msg
    st, msg = _call("fp4kv_sparse_attn_decode", fake, 1, 129, 512, fake, fake, 10, fake, fake, 4,
                    ctypes.c_float(1.0), fake, None, fake, 1 << 20, None)
    assert st == 2 and "H=129" in msg


def test_workspace_sizes_cover_the_configurations():
    wb = binding.workspace_bytes
    # scores + candidate list dominate: at least 12 bytes per scored entry
    assert wb(binding.OP_INDEXER_TOPK, 4, 1 << 20, 32, 2048) >= 4 * (1 << 20) * 12
    assert wb(binding.OP_HIER_POOL_SELECT, 8, 1 << 20, 32, 2048, 1024) > wb(
        binding.OP_INDEXER_TOPK, 8, 1 << 20, 32, 2048)
    assert wb(binding.OP_REINDEX_TOPK, 8, 1 << 20, 32, 2048, 1024) < (2 << 20)
    assert wb(binding.OP_SPARSE_ATTN, 32, 65536, 64, 2048) > 0
    assert wb(binding.OP_KV_QUANT, 1, 1) == 0


def test_binding_raises_typed_errors():
    with pytest.raises(binding.Fp4kvError) as ei:
        binding._check(2)
    assert ei.value.status == 2


def test_host_validation_of_the_window_shard_and_selftest_calls():
    P = ctypes.c_void_p
    fake = P(0x10000)
    f1 = ctypes.c_float(1.0)
    # sliding-window write: d must be a multiple of 16, pointers 16-byte aligned
    st, msg = _call("fp4kv_swa_quant_fp8", fake, 4, 40, 40, None, fake, 4, None)
    assert st == 2 and "d=40" in msg
    st, msg = _call("fp4kv_swa_quant_fp8", fake, 4, 512, 512, None, P(0x10008), 4, None)
    assert st == 1 and "aligned" in msg
    # attention with a window: n_win in [1, 128], swa required
    st, msg = _call("fp4kv_sparse_swa_attn_decode", fake, 1, 16, 512, fake, fake, 10, fake, fake, 4, fake, 129, f1,
                    fake, None, fake, 1 << 20, None)
    assert st == 2 and "n_win" in msg
    st, msg = _call("fp4kv_sparse_swa_attn_decode", fake, 1, 16, 512, fake, fake, 10, fake, fake, 4, None, 64, f1,
                    fake, None, fake, 1 << 20, None)
    assert st == 1 and "swa" in msg
    # exact merge of per-range lists: at most 64 parts and 16384 candidates, bases >= 0
    bases = (ctypes.c_int32 * 65)(*([0] * 65))
    st, msg = _call("fp4kv_topk_merge", fake, fake, 65, 8, 1, bases, 8, 0, 0, fake, None, None, None)
    assert st == 2 and "n_parts" in msg
    st, msg = _call("fp4kv_topk_merge", fake, fake, 8, 4096, 1, bases, 8, 0, 0, fake, None, None, None)
    assert st == 2 and "k_part" in msg
    # each part must keep top_k candidates, or the merge could miss a global winner
    st, msg = _call("fp4kv_topk_merge", fake, fake, 2, 8, 1, bases, 16, 0, 0, fake, None, None, None)
    assert st == 2 and "k_part=8 < top_k=16" in msg
    neg = (ctypes.c_int32 * 2)(0, -5)
    st, msg = _call("fp4kv_topk_merge", fake, fake, 2, 8, 1, neg, 8, 0, 0, fake, None, None, None)
    assert st == 1 and "part_base" in msg
    st, msg = _call("fp4kv_lse_combine", fake, fake, 0, 1, 16, 512, fake, None, None)
    assert st == 2 and "n_parts" in msg
    st, msg = _call("fp4kv_lse_combine", fake, fake, 2, 1, 129, 512, fake, None, None)
    assert st == 2 and "H=129" in msg
    # FP4 indexer operands need an even H_I and cap
    st, msg = _call("fp4kv_indexer_topk", fake, fake, 31, fake, 2, None, 100, fake, 1, None, 0, 8, 16, fake, None,
                    fake, 1 << 20, None)
    assert st == 2 and "even" in msg
    # the bounded-wait test hook checks its limit and workspace before launching anything
    st, msg = _call("fp4kv_selftest_wait_timeout", 0, fake, 256, None)
    assert st == 1 and "limit_us" in msg
    st, msg = _call("fp4kv_selftest_wait_timeout", 1000, None, 256, None)
    assert st == 1 and "workspace" in msg
    st, msg = _call("fp4kv_selftest_wait_timeout_noalloc", 0, None)
    assert st == 1 and "limit_us" in msg
    st, msg = _call("fp4kv_noalloc_status", None, None)
    assert st == 1 and "host_status" in msg


def test_shard_ranges_cover_the_context_once():
    from fp4_sparse_attention_kv_b200 import shard
    for cap in (1, 7, 8, 1000, 65536, 1 << 20):
        for world in (1, 2, 3, 4, 8):
            rs = [shard.shard_range(cap, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == cap
            for (lo, hi), (lo2, _) in zip(rs, rs[1:]):
                assert hi == lo2 and lo <= hi
            assert all(lo % 8 == 0 or lo == cap for lo, _ in rs)
