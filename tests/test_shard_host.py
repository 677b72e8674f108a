"""The context-sharded decode protocol on two gloo ranks (CPU, no GPU): every rank holds one
range of the context, runs the four steps with the oracle standing in for the library's
kernels, and exchanges its lists and partials through torch.distributed. The result must be
the oracle's top-K and attention over the whole, unsharded context."""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

B, CAP, H_I, H, D, K = 3, 1500, 8, 4, 512, 64
LENS = [1500, 1100, 300]  # the last sequence lies entirely in rank 0's range
SEED = 41


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    import synth
    from oracle import fp4kv_oracle as O
    rows = torch.arange(CAP, dtype=torch.int64)
    keys = torch.stack([synth.indexer_keys(SEED, b, rows, 128, True) for b in range(B)])
    q_idx, w = synth.indexer_query(SEED, 0, B, H_I)
    x = torch.stack([synth.kv_rows(SEED, 0, b, rows, D) for b in range(B)])
    xf = O.bf16_bits_to_f64(x.view(torch.int16).numpy().astype(np.uint16))
    packed, scales = O.kv_quant_fp4(xf.reshape(-1, D))
    packed = torch.from_numpy(packed.reshape(B, CAP, D // 2))
    scales = torch.from_numpy(scales.reshape(B, CAP, D // 16))
    q = synth.attn_query(SEED, 0, B, H, D)
    return keys, q_idx, w, packed, scales, q


class OracleOps:
    """The four per-rank steps computed by the oracle on CPU tensors."""

    def __init__(self):
        from oracle import fp4kv_oracle as O
        self.O = O

    @staticmethod
    def _f64_fp8(t):
        from oracle import fp4kv_oracle as O
        return O.fp8_e4m3_to_f64(t.numpy())

    def local_seq_lens(self, seq_lens_host, lo, hi, device):
        return torch.tensor([max(0, min(int(n), hi) - lo) for n in seq_lens_host], dtype=torch.int32)

    def local_topk(self, q, w, keys_local, lens_local, top_k):
        idx = torch.full((B, top_k), -1, dtype=torch.int32)
        score = torch.full((B, top_k), float("-inf"), dtype=torch.float32)
        for b in range(B):
            L = int(lens_local[b])
            sc = self.O.indexer_scores(self._f64_fp8(q[b]), w[b].double().numpy(), self._f64_fp8(keys_local[b, :L]))
            t = self.O.topk_positions(sc, np.arange(L), top_k)
            m = int((t >= 0).sum())
            idx[b] = torch.from_numpy(t.astype(np.int32))
            score[b, :m] = torch.from_numpy(sc[t[:m]].astype(np.float32))
        return idx, score

    def merge(self, all_score, all_idx, bases, top_k, lo, hi):
        idx = torch.full((B, top_k), -1, dtype=torch.int32)
        for b in range(B):
            sc, pos = [], []
            for r, base in enumerate(bases):
                v = all_idx[r, b].numpy()
                ok = v >= 0
                sc.append(all_score[r, b].numpy()[ok])
                pos.append(v[ok].astype(np.int64) + base)
            idx[b] = torch.from_numpy(self.O.topk_positions(np.concatenate(sc), np.concatenate(pos), top_k).astype(np.int32))
        local = torch.where((idx >= lo) & (idx < hi), idx - lo, torch.full_like(idx, -1))
        return idx, local

    def local_attention(self, q, packed_local, scales_local, lens_local, sel_local, sm_scale):
        out = torch.zeros((B, H, D), dtype=torch.float64)
        lse = torch.full((B, H), float("-inf"), dtype=torch.float64)
        for b in range(B):
            sel = sel_local[b].numpy()
            sel = sel[(sel >= 0) & (sel < int(lens_local[b]))]
            if sel.size:
                v = self.O.kv_dequant_fp4(packed_local[b, sel].numpy(), scales_local[b, sel].numpy())
                qf = self.O.bf16_bits_to_f64(q[b].view(torch.int16).numpy().astype(np.uint16))
                o, l = self.O.sparse_attn_decode_rows(qf, v, sm_scale)
                out[b], lse[b] = torch.from_numpy(o), torch.from_numpy(l)
        return out, lse

    def combine(self, all_out, all_lse):
        out = torch.zeros((B, H, D), dtype=torch.float64)
        lse = torch.zeros((B, H), dtype=torch.float64)
        for b in range(B):
            o, l = self.O.attn_lse_merge(all_out[:, b].numpy(), all_lse[:, b].numpy())
            out[b], lse[b] = torch.from_numpy(o), torch.from_numpy(l)
        return out, lse


def _rank_main(rank, world, port, result):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from fp4_sparse_attention_kv_b200 import shard
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    keys, q_idx, w, packed, scales, q = _inputs()
    lo, hi = shard.shard_range(CAP, rank, world)
    idx, out, lse = shard.decode_step(OracleOps(), shard.torch_allgather(), world, rank, CAP, LENS, q_idx, w,
                                      keys[:, lo:hi].contiguous(), K, q, packed[:, lo:hi].contiguous(),
                                      scales[:, lo:hi].contiguous())
    result[rank] = (idx.numpy(), out.numpy(), lse.numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_context_sharded_step_on_two_gloo_ranks_equals_the_whole_context():
    sys.path.insert(0, ROOT)
    from oracle import fp4kv_oracle as O
    world = 2
    with mp.get_context("spawn").Manager() as m:
        result = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), result), nprocs=world, join=True)
        result = dict(result)
    keys, q_idx, w, packed, scales, q = _inputs()
    for b in range(B):
        L = LENS[b]
        sc = O.indexer_scores(O.fp8_e4m3_to_f64(q_idx[b].numpy()), w[b].double().numpy(),
                              O.fp8_e4m3_to_f64(keys[b, :L].numpy()))
        want = O.topk_positions(sc, np.arange(L), K)
        sel = want[want >= 0]
        v = O.kv_dequant_fp4(packed[b, sel].numpy(), scales[b, sel].numpy())
        qf = O.bf16_bits_to_f64(q[b].view(torch.int16).numpy().astype(np.uint16))
        ro, rl = O.sparse_attn_decode_rows(qf, v, 1.0)
        for r in range(world):
            idx, out, lse = result[r]
            assert np.array_equal(idx[b], want), (r, b)
            assert np.allclose(out[b], ro, rtol=1e-9, atol=1e-9) and np.allclose(lse[b], rl, rtol=1e-9, atol=1e-9)
