"""The allocation-free indexer entry point (fp4kv_indexer_topk_noalloc).

It exists for callers that cannot allocate device memory: code running inside a host
runtime that owns all device memory (a serving engine with a fixed, pre-reserved pool, or
a plugin interface that provides no allocator), and latency-critical decode loops that
cannot afford cudaMalloc's implicit device-wide synchronisation. Instead of a caller
workspace it uses the library's own fixed 8 MiB device scratch.

These tests call it through the C ABI and compare it with the regular workspace-based
entry point on the same inputs: top-K indices must be identical (the same kernels run on
the same inputs) and scores equal. Two calls in a row with different inputs check that
whatever the shared scratch keeps from the previous call does not leak into the next.
This file is named so that pytest collects it last; it also passes when run on its own.
"""
import numpy as np
import pytest
import torch

import synth
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fk(cuda_lib):
    import fp4_sparse_attention_kv_b200 as fk
    return fk


def _inputs(seed, B, cap, lens):
    q, w = synth.indexer_query(seed, 0, B, 32, fp8=True, device=DEV)
    keys = P.keys_dev(seed, B, cap, True, DEV)
    return q, w, keys, torch.tensor(lens, dtype=torch.int32, device=DEV)


def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row(fk):
    k = 512
    for seed, B, cap, lens in [(51, 3, 20000, [20000, 17001, 300]), (52, 2, 9000, [9000, 8999])]:
        q, w, keys, lens_t = _inputs(seed, B, cap, lens)
        ref_score = torch.empty((B, k), dtype=torch.float32, device=DEV)
        ref = fk.indexer_topk(q, w, keys, lens_t, k, out_score=ref_score)
        got_score = torch.empty((B, k), dtype=torch.float32, device=DEV)
        got = fk.indexer_topk_noalloc(q, w, keys, lens_t, k, out_score=got_score)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        assert torch.equal(got_score, ref_score)
        # and both agree with the oracle within the top-K tie band
        for b in range(B):
            sc = P.oracle_scores_seq(q[b], w[b], keys[b], lens[b])
            P.check_topk(got[b].cpu().numpy(), sc, np.arange(lens[b]), k, f"noalloc b={b}")


def test_noalloc_reindex_mode_matches(fk):
    B, cap, k, npb = 2, 12000, 256, 64
    q, w, keys, lens_t = _inputs(53, B, cap, [12000, 11000])
    pool = torch.stack([torch.arange(0, 2 * npb, 2, dtype=torch.int32),
                        torch.arange(5, 5 + npb, dtype=torch.int32)]).to(DEV)
    ref = fk.indexer_topk(q, w, keys, lens_t, k, pool=pool)
    got = fk.indexer_topk_noalloc(q, w, keys, lens_t, k, pool=pool)
    assert torch.equal(got, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch(fk):
    q, w, keys, lens_t = _inputs(54, 1, 1000, [1000])
    big_keys = torch.empty((1, 1 << 20, 128), dtype=torch.uint8, device=DEV)
    with pytest.raises(fk.Fp4kvError) as ei:
        fk.indexer_topk_noalloc(q, w, big_keys, lens_t, 64)
    assert ei.value.status == 2 and "maximum" in str(ei.value)


def test_noalloc_status_reports_a_bounded_wait_that_gave_up(fk):
    """A bounded wait that gives up in a kernel running on the allocation-free scratch sets
    the scratch's status bit; an indexer call afterwards keeps it (it clears only the
    histograms and counters), fp4kv_noalloc_status reports it once and clears it, and the
    next call's results are again exact."""
    torch.cuda.synchronize()
    assert fk.noalloc_status() == 0
    fk.selftest_wait_timeout_noalloc(20000)  # 20 ms, then the bit is set
    q, w, keys, lens_t = _inputs(55, 2, 6000, [6000, 5000])
    ref = fk.indexer_topk(q, w, keys, lens_t, 128)
    got = fk.indexer_topk_noalloc(q, w, keys, lens_t, 128)
    assert fk.noalloc_status() == 1
    assert fk.noalloc_status() == 0  # reading clears the word
    assert torch.equal(got, ref)
    got2 = fk.indexer_topk_noalloc(q, w, keys, lens_t, 128)
    assert torch.equal(got2, ref) and fk.noalloc_status() == 0
