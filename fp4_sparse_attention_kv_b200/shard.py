"""Context-sharded decode step: ranks (one GPU each) split every sequence's context positions
into contiguous ranges, and each rank holds the indexer keys and the FP4 rows of its range
only. One step, per rank:

1. indexer top-K over its own range (range-local positions and their scores);
2. all-gather of the (score, position) lists: 8 * top_k bytes per sequence and rank;
3. ``topk_merge``: the exact top-K of the union, which is the top-K of the whole context
   (every rank computes the same result), plus the part of it that lies in this rank's range;
4. sparse attention over those rows of its range: a partial output and lse;
5. all-gather of the partials (B * H * (d + 1) floats per rank) and ``lse_combine``: the
   attention over the whole selection.

The only exchanges are the two all-gathers (NCCL over NVLink between GPUs); every step of
the computation is a library call. ``ops`` and ``allgather`` are parameters so that the same
protocol runs with the library on GPUs (``LibraryOps``, ``torch_allgather``) and, in the
tests, with other implementations of the four steps.
"""
from __future__ import annotations

import torch


def shard_range(cap: int, rank: int, world: int, align: int = 8) -> tuple[int, int]:
    """Positions [lo, hi) of `rank` when `world` ranks split a cache of `cap` positions into
    contiguous ranges of a multiple of `align` positions (the last one may be shorter)."""
    per = -(-cap // world)
    per = -(-per // align) * align
    lo = min(cap, rank * per)
    return lo, min(cap, lo + per)


class LibraryOps:
    """The four per-rank steps as libfp4kv calls."""

    def __init__(self, fk):
        self.fk = fk

    def local_seq_lens(self, seq_lens_host, lo, hi, device):
        """Visible positions of each sequence inside [lo, hi), from host lengths."""
        lens = [max(0, min(int(n), hi) - lo) for n in seq_lens_host]
        return torch.tensor(lens, dtype=torch.int32, device=device)

    def local_topk(self, q, w, keys_local, lens_local, top_k):
        B = lens_local.shape[0]
        if keys_local.shape[1] == 0:  # an empty range (a context shorter than the ranks' split)
            return (torch.full((B, top_k), -1, dtype=torch.int32, device=lens_local.device),
                    torch.full((B, top_k), float("-inf"), dtype=torch.float32, device=lens_local.device))
        score = torch.empty((B, top_k), dtype=torch.float32, device=lens_local.device)
        idx = self.fk.indexer_topk(q, w, keys_local, lens_local, top_k, out_score=score)
        return idx, score

    def merge(self, all_score, all_idx, bases, top_k, lo, hi):
        return self.fk.topk_merge(all_score, all_idx, bases, top_k, local_range=(lo, hi))

    def local_attention(self, q, packed_local, scales_local, lens_local, sel_local, sm_scale):
        if packed_local.shape[1] == 0:  # an empty range holds no row: weight 0 in the combine
            B, H, d = q.shape
            return (torch.zeros((B, H, d), dtype=torch.float32, device=q.device),
                    torch.full((B, H), float("-inf"), dtype=torch.float32, device=q.device))
        return self.fk.sparse_attn_decode(q, packed_local, scales_local, lens_local, sel_local, sm_scale)

    def combine(self, all_out, all_lse):
        return self.fk.lse_combine(all_out, all_lse)


def torch_allgather(group=None):
    """all-gather of one tensor per rank, stacked into [world, *shape] (torch.distributed)."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        t = t.contiguous()
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t, group=group)
        return torch.stack(parts)

    return gather


def local_topk_phase(ops, world: int, rank: int, cap: int, seq_lens_host, q_idx, w, keys_local, top_k: int):
    """Step 1: this rank's range-local top-K. Returns (lens_local, idx_local, score_local)."""
    lo, hi = shard_range(cap, rank, world)
    lens_local = ops.local_seq_lens(seq_lens_host, lo, hi, w.device)
    idx_l, score_l = ops.local_topk(q_idx, w, keys_local, lens_local, top_k)
    return lens_local, idx_l, score_l


def merge_attend_phase(ops, world: int, rank: int, cap: int, all_score, all_idx, top_k: int, q, packed_local,
                       scales_local, lens_local, sm_scale: float):
    """Steps 3-4: the exact global top-K from every rank's lists ([world, B, top_k] each), then
    this rank's partial attention over the selected rows it holds. Returns (idx, out_l, lse_l)."""
    lo, hi = shard_range(cap, rank, world)
    bases = [shard_range(cap, r, world)[0] for r in range(world)]
    idx, sel_local = ops.merge(all_score, all_idx, bases, top_k, lo, hi)
    out_l, lse_l = ops.local_attention(q, packed_local, scales_local, lens_local, sel_local, sm_scale)
    return idx, out_l, lse_l


def decode_step(ops, allgather, world: int, rank: int, cap: int, seq_lens_host, q_idx, w, keys_local,
                top_k: int, q, packed_local, scales_local, sm_scale: float = 1.0):
    """One context-sharded decode step on this rank. keys_local / packed_local / scales_local
    hold positions shard_range(cap, rank, world) of every sequence. Returns (idx [B, top_k]
    global positions, out [B, H, d], lse [B, H]), the same on every rank."""
    lens_local, idx_l, score_l = local_topk_phase(ops, world, rank, cap, seq_lens_host, q_idx, w, keys_local, top_k)
    idx, out_l, lse_l = merge_attend_phase(ops, world, rank, cap, allgather(score_l), allgather(idx_l), top_k, q,
                                           packed_local, scales_local, lens_local, sm_scale)
    out, lse = ops.combine(allgather(out_l), allgather(lse_l))
    return idx, out, lse
