#!/usr/bin/env python
"""Benchmark of decode-time sparse attention over an FP4 KV cache (libfp4kv, B200).

One step = one decode pass of the hot path for a batch of sequences, on inputs already
resident in HBM: quantize-on-write of the new token's KV row, the indexer scan with exact
top-K, and sparse attention over the selected rows. The hierarchical configuration runs a
20-layer step (one Full layer that also selects the candidate pool, Reindex layers inside
the pool, Reuse layers on the previous indices); the CSA2 decoder configuration runs the
pages' own 20-layer schedule (groups of 4 over one shared KV, top-K 512, pool of 2048
blocks). Prints ONE JSON line (rank 0).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--config long|hier|csa2_decoder|csa2_encoder|decode32|decode32_fp4idx|decode32_swa|tiny|quant]
The default is `long` (batch 4 x 1,048,576 entries): the largest single-GPU decode step and
one of the two 1M-entry workloads on which the HBM target is stated.
Under torchrun (N > 1) each rank runs the same per-GPU workload on its own GPU (weak
scaling; the path has no exchange step, so there is no collective in the data path); the
step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import faulthandler
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "sparse FP4 decode-attention tokens/s; achieved HBM GB/s (% of B200 peak)"
D = 512
DK = 128
ROW_BYTES = D // 2 + D // 16  # 288
SWA_LAYER = 700  # generator stream of the sliding-window rows
L2_BYTES = 126 * 2 ** 20

CONFIGS = {
    "decode32": dict(B=32, cap=65536, H=64, H_I=32, K=2048, fp8=True, seed=1,
                     workload="decode batch 32 x 65,536 FP4 entries, 64 heads, FP8 indexer "
                              "keys, top-K 2048"),
    # the same decode step with the indexer query and keys stored in FP4 (E2M1 + one E4M3
    # scale per 16 dims), the format the pages give the indexer
    "decode32_fp4idx": dict(B=32, cap=65536, H=64, H_I=32, K=2048, fp8=False, idx="fp4", seed=1,
                            workload="decode batch 32 x 65,536 FP4 entries, 64 heads, FP4 indexer "
                                     "query and keys (E2M1 + E4M3 per 16 dims), top-K 2048"),
    # the same decode step with the sliding-window branch: the last 128 positions' KV in FP8,
    # attended in the same softmax as the selected rows
    "decode32_swa": dict(B=32, cap=65536, H=64, H_I=32, K=2048, fp8=True, swa=128, seed=1,
                         workload="decode batch 32 x 65,536 FP4 entries + a 128-token FP8 sliding "
                                  "window, 64 heads, FP8 indexer keys, top-K 2048"),
    # the default: the largest single-GPU decode step, one of the 1M-entry configurations
    # the HBM target (indexer top-K + sparse attention at >= 70 % of HBM) is stated on
    "long": dict(B=4, cap=1 << 20, H=64, H_I=32, K=2048, fp8=True, seed=2,
                 workload="long context batch 4 x 1,048,576 FP4 entries, 64 heads, FP8 "
                          "indexer keys, top-K 2048"),
    "hier": dict(B=8, cap=1 << 20, H=64, H_I=32, K=2048, fp8=True, seed=3, layers=20, npb=1024,
                 workload="hierarchical batch 8 x 1,048,576 entries, 20 layers: Full + pool of "
                          "1024 blocks x 8, then Reindex / Reuse alternating, own FP4 KV per "
                          "layer, top-K 2048"),
    # the decoder schedule of the pages' CSA2 section: 20 layers in 5 groups of 4; the first
    # group is Full + 3 Reuse, the others Reindex + 3 Reuse; every layer reads the one main
    # KV and the one set of indexer keys the Full layer owns
    "csa2_decoder": dict(B=8, cap=1 << 20, H=64, H_I=32, K=512, fp8=True, seed=5, layers=20,
                         npb=2048, group=4,
                         workload="CSA2 decoder schedule batch 8 x 1,048,576 entries, 20 layers "
                                  "in groups of 4 (Full or Reindex, then 3 Reuse) over one shared "
                                  "FP4 KV and indexer key set, pool of 2048 blocks x 8, top-K 512"),
    # the encoder schedule of the same section: layers 1-2 attend over their sliding window
    # only; the other 18 run CSA2 at compression m = 2 in 3 groups of 6 (one Full layer that
    # owns the group's KV and indexer keys, then 5 Reuse layers); a 1M-token context is
    # 524,288 compressed entries
    "csa2_encoder": dict(B=8, cap=1 << 19, H=64, H_I=32, K=512, fp8=True, seed=6, swa=128,
                         swa_layers=2, groups=3, group=6,
                         workload="CSA2 encoder schedule batch 8 x 524,288 entries (1M tokens at "
                                  "m = 2), 2 sliding-window-only layers (128-token FP8 window) "
                                  "then 3 groups of 6 (Full + 5 Reuse), own FP4 KV and FP8 "
                                  "indexer keys per group, top-K 512"),
    "tiny": dict(B=1, cap=4096, H=16, H_I=32, K=256, fp8=False, seed=0,
                 workload="tiny batch 1 x 4096 entries, 16 heads, bf16 indexer keys, top-K 256"),
    "quant": dict(tokens=131072, layers=20, seed=4,
                  workload="quantize-on-write sweep 131,072 tokens x 20 layers, d=512"),
}


# sizes a command line may override (the JSON line then lists them under config.overrides)
OVERRIDES = (("B", int), ("cap", int), ("H", int), ("H_I", int), ("K", int), ("npb", int), ("seed", int))


def apply_overrides(cfg: dict, args) -> dict:
    cfg = dict(cfg)
    over = {k: getattr(args, k) for k, _ in OVERRIDES if getattr(args, k, None) is not None}
    for k, v in over.items():
        if k not in cfg:
            raise SystemExit(f"--{k.replace('_', '-')} does not apply to this configuration")
        cfg[k] = v
    if over:
        cfg["overrides"] = over
    return cfg


# ----------------------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------------------
# clocks during the timed region (NVML polling thread; read-only)
# ----------------------------------------------------------------------------------------

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self._h = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nv = nv
            bus = None
            try:  # torch reports the PCI location as integers
                pr = torch.cuda.get_device_properties(device_index)
                dom, b, dv = int(pr.pci_domain_id), int(pr.pci_bus_id), int(pr.pci_device_id)
                bus = f"{dom:08X}:{b:02X}:{dv:02X}.0".encode()
            except Exception:
                bus = None
            if isinstance(bus, bytes):
                self._h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            else:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = int(vis.split(",")[device_index]) if vis and vis.split(",")[0].isdigit() else device_index
                self._h = nv.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM))
            self._get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception as e:  # NVML unavailable: report no clock data
            self._err = str(e)
            self._h = None
        self.period = period_s

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)))
                self.reasons |= int(self._get_reasons(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._h is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self):
        if self._thr is not None:
            self._stop.set()
            self._thr.join()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for bit, n in REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense 16-bit tensor-core peak in TFLOP/s: the measured bf16 GEMM burst figure (fp16,
    which the attention's MMAs use, has the same nominal rate)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured (bf16 burst)"
    return 1590.0, "fallback"


def attn_flops_per_row(H: int) -> int:
    """Algorithmic flops of the attention per selected row and sequence: q.k and p*v over
    d channels for each of the H heads (2 flops per multiply-add, twice)."""
    return 4 * H * D


def traffic_record(kernel: str, workload: str):
    """dram bytes per launch from the committed ncu summary, if the kernel source has not
    changed since it was captured (the summary stores the source digest)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    src = {"index_score": "indexer.cu", "sparse_attn": "attn.cu", "kv_quant_fp4": "kv_quant.cu"}[kernel]
    digest = hashlib.sha256(open(os.path.join(ROOT, "fp4_sparse_attention_kv_b200", "csrc", src),
                                 "rb").read()).hexdigest()[:16]
    for line in open(path):
        m = dict(re.findall(r"(\w+)=(\S+)", line))
        if m.get("kernel") == kernel and m.get("workload") == workload and m.get("src") == digest:
            return float(m["dram_bytes_per_launch"])
    return None


class TwoSets:
    """Per-step inputs and outputs in two buffer sets, so that the end-to-end run can copy one
    step's data while another step computes. `in_attrs` / `out_attrs` name the attributes
    (tensors or lists of tensors) that hold them; `use_set(k)` rebinds them to set k."""

    in_attrs: tuple = ()
    out_attrs: tuple = ()

    def _flat(self, names, k):
        out = []
        for a in names:
            v = self._sets[k][a]
            out.extend(v if isinstance(v, list) else [v])
        return out

    def make_second_set(self):
        if getattr(self, "_sets", None) is not None:
            return
        first = {a: getattr(self, a) for a in self.in_attrs + self.out_attrs}
        second = {a: ([t.clone() for t in v] if isinstance(v, list) else v.clone()) for a, v in first.items()}
        self._sets = [first, second]

    def use_set(self, k):
        for a, v in self._sets[k].items():
            setattr(self, a, v)

    def inputs_of(self, k):
        return self._flat(self.in_attrs, k)

    graphs = None

    def capture_graphs(self):
        """Capture one step per buffer set in a CUDA graph (the library enqueues on the
        current stream and allocates nothing, so a step is capturable); on any failure the
        steps stay eager."""
        self.make_second_set()
        try:
            gs = []
            for k in range(2):
                self.use_set(k)
                cs = torch.cuda.Stream()
                cs.wait_stream(torch.cuda.current_stream())
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cs, capture_error_mode="relaxed"):
                    self.step()
                torch.cuda.current_stream().wait_stream(cs)
                gs.append(g)
            torch.cuda.synchronize()
            self.graphs = gs
        except Exception as e:  # noqa: BLE001 - any capture failure falls back to eager steps
            phase(f"graph capture failed, eager steps: {e}")
            self.graphs = None
        self.use_set(0)

    def run_step(self, k=0):
        """One step on buffer set k: a graph replay when captured, else eager launches."""
        if getattr(self, "_sets", None) is not None:
            self.use_set(k)
        if self.graphs is not None:
            self.graphs[k].replay()
        else:
            self.step()

    def outputs_of(self, k):
        return self._flat(self.out_attrs, k)


class DecodeWorkload(TwoSets):
    """Tiny / decode32 / long: one decoder layer per step (write the new row, Full-mode
    indexer top-K over the whole cache, attention over the selected rows)."""

    def __init__(self, cfg, fk, device, rank=0):
        self.cfg, self.fk, self.dev = cfg, fk, device
        B, cap, H, H_I, K = cfg["B"], cfg["cap"], cfg["H"], cfg["H_I"], cfg["K"]
        seed = cfg["seed"] + 1000 * rank
        self.B, self.cap, self.H, self.H_I, self.K = B, cap, H, H_I, K
        fp8 = cfg["fp8"]
        self.fp4_idx = cfg.get("idx") == "fp4"
        self.key_bytes = DK // 2 + DK // 16 if self.fp4_idx else DK * (1 if fp8 else 2)
        # resident cache: FP4 rows + indexer keys, filled through the library's quantizer
        self.packed = torch.empty((B, cap, D // 2), dtype=torch.uint8, device=device)
        self.scales = torch.empty((B, cap, D // 16), dtype=torch.uint8, device=device)
        if self.fp4_idx:
            self.keys = fk.E2M1Planes(B, cap, device)
        else:
            self.keys = torch.empty((B, cap, DK), dtype=torch.uint8 if fp8 else torch.bfloat16, device=device)
        chunk = 1 << 18
        for b in range(B):
            for r0 in range(0, cap, chunk):
                rows = torch.arange(r0, min(cap, r0 + chunk), dtype=torch.int64, device=device)
                x = synth.kv_rows(seed, 0, b, rows, D)
                fk.kv_quant_fp4(x, self.packed[b, r0:r0 + rows.numel()], self.scales[b, r0:r0 + rows.numel()])
                kr = synth.indexer_keys(seed, b, rows, DK, fp8)
                if self.fp4_idx:  # stored with the library's quantizer (d = 128)
                    fk.kv_quant_fp4(kr, self.keys.codes[b, r0:r0 + rows.numel()],
                                    self.keys.scales[b, r0:r0 + rows.numel()])
                else:
                    self.keys[b, r0:r0 + rows.numel()] = kr
        # per-step inputs (device copies, and pinned host copies for the end-to-end run)
        self.q = synth.attn_query(seed, 0, B, H, D, device=device)
        self.qi, self.w = synth.indexer_query(seed, 0, B, H_I, fp8=fp8, device=device)
        # FP4 indexer: the bf16 query is stored as FP4 inside each step
        self.qi4 = fk.E2M1Planes(B, H_I, device) if self.fp4_idx else None
        # sliding window: ring of the last n_win positions' rows (E4M3), slot = position % n_win
        self.n_win = cfg.get("swa", 0)
        self.swa = None
        if self.n_win:
            nw = self.n_win
            self.swa = torch.empty((B, nw, D), dtype=torch.uint8, device=device)
            pos = torch.arange(cap - nw, cap, dtype=torch.int64, device=device)
            for b in range(B):
                fk.swa_quant_fp8(synth.kv_rows(seed, SWA_LAYER, b, pos, D), self.swa[b],
                                 dst_row=pos % nw)
            self.x_swa_new = synth.kv_rows(seed, SWA_LAYER, 10 ** 6, torch.arange(B, dtype=torch.int64, device=device), D)
            self.swa_dst = torch.arange(B, dtype=torch.int64, device=device) * nw + (cap - 1) % nw
        self.x_new = synth.kv_rows(seed, 0, 10 ** 6, torch.arange(B, dtype=torch.int64, device=device), D)
        self.dst = (torch.arange(B, dtype=torch.int64, device=device) * cap + (cap - 1))
        self.lens = torch.full((B,), cap, dtype=torch.int32, device=device)
        self.idx = torch.empty((B, K), dtype=torch.int32, device=device)
        self.out = torch.empty((B, H, D), dtype=torch.float32, device=device)
        self.lse = torch.empty((B, H), dtype=torch.float32, device=device)
        self.ws_i = fk.alloc_workspace(fk.workspace_bytes(fk.OP_INDEXER_TOPK, B, cap, H_I, K), device)
        self.ws_a = fk.alloc_workspace(fk.workspace_bytes(fk.OP_SPARSE_ATTN, B, cap, H, K), device)
        self.inputs = [self.q, self.qi, self.w, self.x_new]
        self.in_attrs, self.out_attrs = ("q", "qi", "w", "x_new"), ("out", "lse")
        if self.n_win:
            self.inputs.append(self.x_swa_new)
            self.in_attrs = self.in_attrs + ("x_swa_new",)
        self.outputs = [self.out, self.lse]
        # quantize, scan, select, attention (its chunk CTAs combine in-kernel) (+ the query's
        # FP4 quantize with an FP4 indexer, + the window row's FP8 write)
        self.launches_per_step = 4 + (1 if self.fp4_idx else 0) + (1 if self.n_win else 0)
        self.attn_rows_per_step = B * (K + self.n_win)
        self.tokens_per_step = B

    def step(self):
        fk = self.fk
        fk.kv_quant_fp4(self.x_new, self.packed.view(-1, D // 2), self.scales.view(-1, D // 16),
                        dst_row=self.dst)
        if self.n_win:
            fk.swa_quant_fp8(self.x_swa_new, self.swa.view(-1, D), dst_row=self.swa_dst)
        if self.fp4_idx:
            self.qi4.quantize_from(self.qi)
            fk.indexer_topk(self.qi4, self.w, self.keys, self.lens, self.K, ws=self.ws_i, out_idx=self.idx)
        else:
            fk.indexer_topk(self.qi, self.w, self.keys, self.lens, self.K, ws=self.ws_i, out_idx=self.idx)
        fk.sparse_attn_decode(self.q, self.packed, self.scales, self.lens, self.idx, 1.0,
                              ws=self.ws_a, out=self.out, lse=self.lse, swa=self.swa)

    def algorithmic_bytes(self):
        return {"index_score": self.B * self.cap * self.key_bytes,
                "sparse_attn": self.B * (self.K * ROW_BYTES + self.n_win * D),
                "kv_quant_fp4": self.B * (2 * D + ROW_BYTES) + (self.B * (2 * D + D) if self.n_win else 0)}


class HierWorkload(TwoSets):
    """Hierarchical: 20 layers per step. Layer 1 (Full): hier_pool_select over all entries
    -> top-K + pool; layers 2, 4, .., 20 (Reindex): own indexer query scored inside the pool
    over layer 1's keys; layers 3, 5, .., 19 (Reuse): the previous layer's indices. Every
    layer has its own FP4 KV and attends over it. The new rows of all 20 layers are written
    by one quantize call at the start of the step: in the pages' causal encoder-decoder every
    decoder layer's global KV is a projection of the encoder's last hidden state, so all of
    them exist before the first decoder layer runs (the queries do not: each layer computes
    its own from its own hidden state, so the layers' scans and attentions stay in order)."""

    def __init__(self, cfg, fk, device, rank=0):
        self.cfg, self.fk, self.dev = cfg, fk, device
        B, cap, H, H_I, K, L, npb = (cfg["B"], cfg["cap"], cfg["H"], cfg["H_I"], cfg["K"],
                                      cfg["layers"], cfg["npb"])
        seed = cfg["seed"] + 1000 * rank
        self.B, self.cap, self.H, self.H_I, self.K, self.L, self.npb = B, cap, H, H_I, K, L, npb
        # the 20 layers' caches in one allocation (layer-major), so one call writes every
        # layer's new row
        self.packed_all = torch.empty((L, B, cap, D // 2), dtype=torch.uint8, device=device)
        self.scales_all = torch.empty((L, B, cap, D // 16), dtype=torch.uint8, device=device)
        self.packed = [self.packed_all[l] for l in range(L)]
        self.scales = [self.scales_all[l] for l in range(L)]
        self.keys = torch.empty((B, cap, DK), dtype=torch.uint8, device=device)
        chunk = 1 << 18
        for b in range(B):
            for r0 in range(0, cap, chunk):
                rows = torch.arange(r0, min(cap, r0 + chunk), dtype=torch.int64, device=device)
                self.keys[b, r0:r0 + rows.numel()] = synth.indexer_keys(seed, b, rows, DK, True)
                for l in range(L):
                    x = synth.kv_rows(seed, l, b, rows, D)
                    fk.kv_quant_fp4(x, self.packed[l][b, r0:r0 + rows.numel()],
                                    self.scales[l][b, r0:r0 + rows.numel()])
        self.q = [synth.attn_query(seed, l, B, H, D, device=device) for l in range(L)]
        qw = [synth.indexer_query(seed, l, B, H_I, fp8=True, device=device) for l in range(L)]
        self.qi = [a for a, _ in qw]
        self.w = [b_ for _, b_ in qw]
        # new rows [L * B, d] (layer-major) and their rows in the layer-major caches
        self.x_new = torch.cat([synth.kv_rows(seed, l, 10 ** 6, torch.arange(B, dtype=torch.int64, device=device), D)
                                for l in range(L)])
        self.dst = torch.arange(L * B, dtype=torch.int64, device=device) * cap + (cap - 1)
        self.lens = torch.full((B,), cap, dtype=torch.int32, device=device)
        self.idx = [torch.empty((B, K), dtype=torch.int32, device=device) for _ in range(L)]
        self.pool = torch.empty((B, npb), dtype=torch.int32, device=device)
        self.out = [torch.empty((B, H, D), dtype=torch.float32, device=device) for _ in range(L)]
        self.lse = [torch.empty((B, H), dtype=torch.float32, device=device) for _ in range(L)]
        self.ws_h = fk.alloc_workspace(fk.workspace_bytes(fk.OP_HIER_POOL_SELECT, B, cap, H_I, K, npb), device)
        self.ws_r = fk.alloc_workspace(fk.workspace_bytes(fk.OP_REINDEX_TOPK, B, cap, H_I, K, npb), device)
        self.ws_a = fk.alloc_workspace(fk.workspace_bytes(fk.OP_SPARSE_ATTN, B, cap, H, K), device)
        self.inputs = self.q + self.qi + self.w + [self.x_new]
        self.outputs = self.out + self.lse
        self.in_attrs, self.out_attrs = ("q", "qi", "w", "x_new"), ("out", "lse")
        # one quantize; the Full layer and each Reindex layer a scan and a select (the Full
        # layer's pool and position selects share one launch); per layer an attention
        self.launches_per_step = 1 + 2 + (L // 2) * 2 + L
        self.tokens_per_step = B

    def step(self):
        fk, L = self.fk, self.L
        fk.kv_quant_fp4(self.x_new, self.packed_all.view(-1, D // 2), self.scales_all.view(-1, D // 16),
                        dst_row=self.dst)
        for l in range(L):
            if l == 0:
                fk.hier_pool_select(self.qi[0], self.w[0], self.keys, self.lens, self.K, self.npb,
                                    ws=self.ws_h, out_idx=self.idx[0], out_pool=self.pool)
                idx = self.idx[0]
            elif l % 2 == 1:  # layers 2, 4, .. (1-based): Reindex inside the pool
                fk.indexer_topk(self.qi[l], self.w[l], self.keys, self.lens, self.K, pool=self.pool,
                                ws=self.ws_r, out_idx=self.idx[l])
                idx = self.idx[l]
            else:  # Reuse: the previous layer's indices
                idx = self.idx[l - 1]
            fk.sparse_attn_decode(self.q[l], self.packed[l], self.scales[l], self.lens, idx, 1.0,
                                  ws=self.ws_a, out=self.out[l], lse=self.lse[l])

    def algorithmic_bytes(self):
        B, L = self.B, self.L
        n_reindex = (L - 1 + 1) // 2
        return {"index_score": B * self.cap * DK + n_reindex * B * self.npb * 8 * DK,
                "sparse_attn": L * B * self.K * ROW_BYTES,
                "kv_quant_fp4": L * B * (2 * D + ROW_BYTES)}


class Csa2DecoderWorkload(TwoSets):
    """The decoder schedule of the pages' CSA2 section: 20 layers in groups of 4. Layer 1
    (Full) scores every entry -> top-K + candidate pool and is the only layer that writes a
    KV row; the first layer of every later group (Reindex) re-scores inside the pool with
    its own indexer query; the other layers (Reuse) take their group's indices. Every layer
    attends with its own query over the one shared FP4 KV."""

    def __init__(self, cfg, fk, device, rank=0):
        self.cfg, self.fk, self.dev = cfg, fk, device
        B, cap, H, H_I, K, L, npb, G = (cfg["B"], cfg["cap"], cfg["H"], cfg["H_I"], cfg["K"],
                                         cfg["layers"], cfg["npb"], cfg["group"])
        seed = cfg["seed"] + 1000 * rank
        self.B, self.cap, self.H, self.H_I, self.K, self.L, self.npb, self.G = B, cap, H, H_I, K, L, npb, G
        n_src = (L + G - 1) // G
        self.packed = torch.empty((B, cap, D // 2), dtype=torch.uint8, device=device)
        self.scales = torch.empty((B, cap, D // 16), dtype=torch.uint8, device=device)
        self.keys = torch.empty((B, cap, DK), dtype=torch.uint8, device=device)
        chunk = 1 << 18
        for b in range(B):
            for r0 in range(0, cap, chunk):
                rows = torch.arange(r0, min(cap, r0 + chunk), dtype=torch.int64, device=device)
                self.keys[b, r0:r0 + rows.numel()] = synth.indexer_keys(seed, b, rows, DK, True)
                fk.kv_quant_fp4(synth.kv_rows(seed, 0, b, rows, D), self.packed[b, r0:r0 + rows.numel()],
                                self.scales[b, r0:r0 + rows.numel()])
        self.q = [synth.attn_query(seed, l, B, H, D, device=device) for l in range(L)]
        # one indexer query per group (the group's Full or Reindex layer)
        qw = [synth.indexer_query(seed, g * G, B, H_I, fp8=True, device=device) for g in range(n_src)]
        self.qi = [a for a, _ in qw]
        self.w = [b_ for _, b_ in qw]
        self.x_new = synth.kv_rows(seed, 0, 10 ** 6, torch.arange(B, dtype=torch.int64, device=device), D)
        self.dst = torch.arange(B, dtype=torch.int64, device=device) * cap + (cap - 1)
        self.lens = torch.full((B,), cap, dtype=torch.int32, device=device)
        self.idx = [torch.empty((B, K), dtype=torch.int32, device=device) for _ in range(n_src)]
        self.pool = torch.empty((B, npb), dtype=torch.int32, device=device)
        self.out = [torch.empty((B, H, D), dtype=torch.float32, device=device) for _ in range(L)]
        self.lse = [torch.empty((B, H), dtype=torch.float32, device=device) for _ in range(L)]
        self.ws_h = fk.alloc_workspace(fk.workspace_bytes(fk.OP_HIER_POOL_SELECT, B, cap, H_I, K, npb), device)
        self.ws_r = fk.alloc_workspace(fk.workspace_bytes(fk.OP_REINDEX_TOPK, B, cap, H_I, K, npb), device)
        self.ws_a = fk.alloc_workspace(fk.workspace_bytes(fk.OP_SPARSE_ATTN, B, cap, H, K), device)
        self.inputs = self.q + self.qi + self.w + [self.x_new]
        self.outputs = self.out + self.lse
        self.in_attrs, self.out_attrs = ("q", "qi", "w", "x_new"), ("out", "lse")
        # one quantize; a scan and a select per group; an attention per layer
        self.launches_per_step = 1 + 2 * n_src + L
        self.tokens_per_step = B

    def step(self):
        fk, G = self.fk, self.G
        fk.kv_quant_fp4(self.x_new, self.packed.view(-1, D // 2), self.scales.view(-1, D // 16),
                        dst_row=self.dst)
        for l in range(self.L):
            g = l // G
            if l == 0:
                fk.hier_pool_select(self.qi[0], self.w[0], self.keys, self.lens, self.K, self.npb,
                                    ws=self.ws_h, out_idx=self.idx[0], out_pool=self.pool)
            elif l % G == 0:
                fk.indexer_topk(self.qi[g], self.w[g], self.keys, self.lens, self.K, pool=self.pool,
                                ws=self.ws_r, out_idx=self.idx[g])
            fk.sparse_attn_decode(self.q[l], self.packed, self.scales, self.lens, self.idx[g], 1.0,
                                  ws=self.ws_a, out=self.out[l], lse=self.lse[l])

    def algorithmic_bytes(self):
        B, L, G = self.B, self.L, self.G
        n_reindex = (L + G - 1) // G - 1
        return {"index_score": B * self.cap * DK + n_reindex * B * self.npb * 8 * DK,
                "sparse_attn": L * B * self.K * ROW_BYTES,
                "kv_quant_fp4": B * (2 * D + ROW_BYTES)}


class Csa2EncoderWorkload(TwoSets):
    """The encoder schedule of the pages' CSA2 section: layers 1-2 attend over their own
    sliding window only (its KV kept in FP8); the other 18 layers run CSA2 at compression
    m = 2 in 3 groups of 6. The first layer of a group (Full) writes the group's new KV row,
    scores every entry with its indexer query over the group's own keys and keeps the top-K;
    the 5 Reuse layers attend with their own queries over the same KV and indices. Encoder
    layers run in order: each group's KV and query come from its own layer's hidden state."""

    def __init__(self, cfg, fk, device, rank=0):
        self.cfg, self.fk, self.dev = cfg, fk, device
        B, cap, H, H_I, K = cfg["B"], cfg["cap"], cfg["H"], cfg["H_I"], cfg["K"]
        G, NG, NS, nw = cfg["group"], cfg["groups"], cfg["swa_layers"], cfg["swa"]
        seed = cfg["seed"] + 1000 * rank
        self.B, self.cap, self.H, self.H_I, self.K, self.G, self.NG, self.NS, self.n_win = B, cap, H, H_I, K, G, NG, NS, nw
        self.L = NS + NG * G
        self.src = [NS + g * G for g in range(NG)]  # the groups' Full (KV source) layers
        self.packed = [torch.empty((B, cap, D // 2), dtype=torch.uint8, device=device) for _ in range(NG)]
        self.scales = [torch.empty((B, cap, D // 16), dtype=torch.uint8, device=device) for _ in range(NG)]
        self.keys = [torch.empty((B, cap, DK), dtype=torch.uint8, device=device) for _ in range(NG)]
        chunk = 1 << 18
        for g in range(NG):
            for b in range(B):
                for r0 in range(0, cap, chunk):
                    rows = torch.arange(r0, min(cap, r0 + chunk), dtype=torch.int64, device=device)
                    fk.kv_quant_fp4(synth.kv_rows(seed, self.src[g], b, rows, D),
                                    self.packed[g][b, r0:r0 + rows.numel()], self.scales[g][b, r0:r0 + rows.numel()])
                    self.keys[g][b, r0:r0 + rows.numel()] = synth.indexer_keys(seed, b, rows, DK, True,
                                                                               source=self.src[g])
        # the sliding-window-only layers: a ring of the last nw positions' rows (E4M3)
        pos = torch.arange(cap - nw, cap, dtype=torch.int64, device=device)
        self.swa = [torch.empty((B, nw, D), dtype=torch.uint8, device=device) for _ in range(NS)]
        for l in range(NS):
            for b in range(B):
                fk.swa_quant_fp8(synth.kv_rows(seed, SWA_LAYER + l, b, pos, D), self.swa[l][b], dst_row=pos % nw)
        ar = torch.arange(B, dtype=torch.int64, device=device)
        self.x_swa_new = [synth.kv_rows(seed, SWA_LAYER + l, 10 ** 6, ar, D) for l in range(NS)]
        self.swa_dst = ar * nw + (cap - 1) % nw
        self.x_new = [synth.kv_rows(seed, self.src[g], 10 ** 6, ar, D) for g in range(NG)]
        self.dst = ar * cap + (cap - 1)
        self.q = [synth.attn_query(seed, l, B, H, D, device=device) for l in range(self.L)]
        qw = [synth.indexer_query(seed, self.src[g], B, H_I, fp8=True, device=device) for g in range(NG)]
        self.qi = [a for a, _ in qw]
        self.w = [b_ for _, b_ in qw]
        self.lens = torch.full((B,), cap, dtype=torch.int32, device=device)
        self.idx = [torch.empty((B, K), dtype=torch.int32, device=device) for _ in range(NG)]
        self.no_idx = torch.full((B, 1), -1, dtype=torch.int32, device=device)  # window-only layers
        self.out = [torch.empty((B, H, D), dtype=torch.float32, device=device) for _ in range(self.L)]
        self.lse = [torch.empty((B, H), dtype=torch.float32, device=device) for _ in range(self.L)]
        self.ws_i = fk.alloc_workspace(fk.workspace_bytes(fk.OP_INDEXER_TOPK, B, cap, H_I, K), device)
        self.ws_a = fk.alloc_workspace(fk.workspace_bytes(fk.OP_SPARSE_ATTN, B, cap, H, K), device)
        self.inputs = self.q + self.qi + self.w + self.x_new + self.x_swa_new
        self.outputs = self.out + self.lse
        self.in_attrs, self.out_attrs = ("q", "qi", "w", "x_new", "x_swa_new"), ("out", "lse")
        # per window-only layer a window write and an attention; per group a quantize, a
        # scan, a select and G attentions
        self.launches_per_step = 2 * NS + NG * (3 + G)
        self.attn_rows_per_step = NG * G * B * K + NS * B * nw
        self.tokens_per_step = B

    def step(self):
        fk = self.fk
        for l in range(self.NS):
            fk.swa_quant_fp8(self.x_swa_new[l], self.swa[l].view(-1, D), dst_row=self.swa_dst)
            fk.sparse_attn_decode(self.q[l], self.packed[0], self.scales[0], self.lens, self.no_idx, 1.0,
                                  ws=self.ws_a, out=self.out[l], lse=self.lse[l], swa=self.swa[l])
        for g in range(self.NG):
            fk.kv_quant_fp4(self.x_new[g], self.packed[g].view(-1, D // 2), self.scales[g].view(-1, D // 16),
                            dst_row=self.dst)
            fk.indexer_topk(self.qi[g], self.w[g], self.keys[g], self.lens, self.K, ws=self.ws_i,
                            out_idx=self.idx[g])
            for j in range(self.G):
                l = self.src[g] + j
                fk.sparse_attn_decode(self.q[l], self.packed[g], self.scales[g], self.lens, self.idx[g], 1.0,
                                      ws=self.ws_a, out=self.out[l], lse=self.lse[l])

    def algorithmic_bytes(self):
        B, NG, G, NS = self.B, self.NG, self.G, self.NS
        return {"index_score": NG * B * self.cap * DK,
                "sparse_attn": NG * G * B * self.K * ROW_BYTES + NS * B * self.n_win * D,
                "kv_quant_fp4": NG * B * (2 * D + ROW_BYTES) + NS * B * (2 * D + D)}


class QuantWorkload(TwoSets):
    """Quantize-on-write sweep: 131,072 tokens x 20 layers of bf16 rows -> FP4 + scales."""

    def __init__(self, cfg, fk, device, rank=0):
        self.fk = fk
        n = cfg["tokens"] * cfg["layers"]
        seed = cfg["seed"] + 1000 * rank
        self.x = torch.empty((n, D), dtype=torch.bfloat16, device=device)
        chunk = 1 << 18
        for r0 in range(0, n, chunk):
            rows = torch.arange(r0, min(n, r0 + chunk), dtype=torch.int64, device=device)
            self.x[r0:r0 + rows.numel()] = synth.kv_rows(seed, r0 // cfg["tokens"], 0, rows, D,
                                                         heavy_frac=0.001)
        self.packed = torch.empty((n, D // 2), dtype=torch.uint8, device=device)
        self.scales = torch.empty((n, D // 16), dtype=torch.uint8, device=device)
        self.n = n
        self.inputs = [self.x]
        self.outputs = [self.packed, self.scales]
        self.in_attrs, self.out_attrs = ("x",), ("packed", "scales")
        self.launches_per_step = 1
        self.tokens_per_step = cfg["tokens"]

    def step(self):
        self.fk.kv_quant_fp4(self.x, self.packed, self.scales)

    def algorithmic_bytes(self):
        return {"kv_quant_fp4": self.n * (2 * D + ROW_BYTES)}


# ----------------------------------------------------------------------------------------
# timing
# ----------------------------------------------------------------------------------------

def timed_steps(wl, steps, warmup, flush, sampler, fk):
    """Device time of `steps` steps. When `flush` is given, L2 is flushed (a write larger
    than L2) before each step, outside the timed windows; otherwise every step streams more
    than twice the L2 capacity, so no step starts with the previous step's data cached.

    The steps are timed bare (CUDA events around each step only), then run once more with
    the library's per-launch events on for the per-kernel breakdown: events recorded
    between two launches would keep the second from starting early as a programmatic
    dependent of the first, so they stay out of the headline timing."""
    s = torch.cuda.current_stream()
    for _ in range(warmup):
        wl.run_step(0)
    torch.cuda.synchronize()

    def run(n, prof_pass=False):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for a, b in evs:
            if flush is not None:
                flush.zero_()
            a.record(s)
            if prof_pass:
                wl.step()  # eager: the library records its per-launch events as it launches
            else:
                wl.run_step(0)
            b.record(s)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    sampler.start()
    total_ms = run(steps)
    fk.profile_read()  # drop earlier records
    fk.profile_enable(True)
    run(steps, prof_pass=True)
    fk.profile_enable(False)
    sampler.stop()
    prof = fk.profile_read()
    return total_ms, prof


def e2e_steps(wl, steps, warmup):
    """Same step through the public API with host buffers: every step copies its inputs from
    pinned host memory and reads its outputs back inside the timed region. As in a serving
    loop, the copies run on an upload and a download stream against two buffer sets, so step
    i's inputs travel while step i - 1 computes and its outputs while step i + 1 computes;
    events order each set's upload, compute and read-back."""
    wl.make_second_set()
    dev = wl.inputs_of(0)[0].device
    h_in = [t.detach().cpu().pin_memory() for t in wl.inputs_of(0)]
    h_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in wl.outputs_of(0)] for _ in range(2)]
    torch.cuda.synchronize()
    # non-blocking streams of their own (no implicit ordering with the legacy default stream)
    comp, up, down = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            k = i & 1
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_free[k])  # set k's previous step has been read back
                for h, d in zip(h_in, wl.inputs_of(k)):
                    d.copy_(h, non_blocking=True)
                ev_up[k].record(up)
            with torch.cuda.stream(comp):
                comp.wait_event(ev_up[k])
                wl.run_step(k)  # the library enqueues on the current stream
                ev_comp[k].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(ev_comp[k])
                for h, d in zip(h_out[k], wl.outputs_of(k)):
                    h.copy_(d, non_blocking=True)
                ev_free[k].record(down)

    run(max(2, warmup))
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(up)
    run(steps)
    down.wait_stream(up)
    down.wait_stream(comp)
    b.record(down)
    torch.cuda.synchronize()
    wl.use_set(0)
    h2d = sum(t.numel() * t.element_size() for t in wl.inputs_of(0))
    d2h = sum(t.numel() * t.element_size() for t in wl.outputs_of(0))
    return a.elapsed_time(b), h2d, d2h


# ----------------------------------------------------------------------------------------
# CPU oracle baseline (the oracle as it stands, on a bounded sample)
# ----------------------------------------------------------------------------------------

def _bits(x):
    """bf16 tensor -> its uint16 bit patterns (numpy), the oracle's input form."""
    return x.view(torch.int16).numpy().astype(np.uint16)


def oracle_prepare_decode(cfg, seq: int):
    """Inputs of the whole decode step for ONE sequence, drawn from synth as the GPU workload
    draws them (untimed), and the oracle's run over them (timed)."""
    from oracle import fp4kv_oracle as O
    seed = cfg["seed"]
    cap, H, H_I, K, fp8 = cfg["cap"], cfg["H"], cfg["H_I"], cfg["K"], cfg["fp8"]
    rows = torch.arange(cap, dtype=torch.int64)
    keys = synth.indexer_keys(seed, seq, rows, DK, fp8)
    qi, w = synth.indexer_query(seed, 0, seq + 1, H_I, fp8=fp8)
    keys_in = keys.numpy() if fp8 else _bits(keys)
    qi_in = qi[seq].numpy() if fp8 else _bits(qi[seq])
    w_in = w[seq].double().numpy()
    x_new = _bits(synth.kv_rows(seed, 0, 10 ** 6, torch.tensor([seq]), D))
    q = _bits(synth.attn_query(seed, 0, seq + 1, H, D)[seq])
    nw = cfg.get("swa", 0)
    xw = _bits(synth.kv_rows(seed, SWA_LAYER, seq, torch.arange(cap - nw, cap, dtype=torch.int64), D)) if nw else None

    def rows_of(sel):  # the selected rows' bf16 values (the cache content), drawn on demand
        return _bits(synth.kv_rows(seed, 0, seq, torch.as_tensor(sel), D))

    def run():
        dec = O.fp8_e4m3_to_f64 if fp8 else O.bf16_bits_to_f64
        kf, qf = dec(keys_in), dec(qi_in)
        if cfg.get("idx") == "fp4":
            kf, qf = O.indexer_fp4_values(kf), O.indexer_fp4_values(qf)
        O.kv_quant_fp4(O.bf16_bits_to_f64(x_new))
        idx, _ = O.indexer_topk(qf, w_in, kf, cap, K)
        pk, sc = O.kv_quant_fp4(O.bf16_bits_to_f64(rows_of(idx[idx >= 0])))
        qf64 = O.bf16_bits_to_f64(q)
        if nw:
            vw = O.e4m3_decode(O.swa_quant_fp8(O.bf16_bits_to_f64(xw)))
            O.sparse_swa_attn_decode_rows(qf64, O.kv_dequant_fp4(pk, sc), vw, 1.0)
        else:
            O.sparse_attn_decode_rows(qf64, O.kv_dequant_fp4(pk, sc), 1.0)
    return run


def oracle_prepare_layers(cfg, seq: int):
    """The whole 20-layer step (hier or csa2_decoder) for ONE sequence: inputs drawn from
    synth (untimed) and the oracle's run (timed): the Full layer's scan with top-K and
    pool, the Reindex layers inside the pool, every layer's new-row write and attention."""
    from oracle import fp4kv_oracle as O
    seed, cap, H, H_I, K, L, npb = (cfg["seed"], cfg["cap"], cfg["H"], cfg["H_I"], cfg["K"],
                                     cfg["layers"], cfg["npb"])
    G = cfg.get("group")  # csa2_decoder: groups of G over one shared KV
    keys = synth.indexer_keys(seed, seq, torch.arange(cap, dtype=torch.int64), DK, True).numpy()
    writes = [l for l in range(L) if G is None or l == 0]  # csa2: only the Full layer writes
    x_new = {l: _bits(synth.kv_rows(seed, l, 10 ** 6, torch.tensor([seq]), D)) for l in writes}
    scans = [l for l in range(L) if l == 0 or (G is None and l % 2 == 1) or (G is not None and l % G == 0)]
    qw = {}
    for l in scans:
        src = l if G is None else (l // G) * G
        qi, w = synth.indexer_query(seed, src, seq + 1, H_I, fp8=True)
        qw[l] = (qi[seq].numpy(), w[seq].double().numpy())
    q = {l: _bits(synth.attn_query(seed, l, seq + 1, H, D)[seq]) for l in range(L)}

    def rows_of(l, sel):
        return _bits(synth.kv_rows(seed, l if G is None else 0, seq, torch.as_tensor(sel), D))

    def run():
        kf = O.fp8_e4m3_to_f64(keys)
        idx_of, pool = {}, None
        for l in range(L):
            if l in x_new:
                O.kv_quant_fp4(O.bf16_bits_to_f64(x_new[l]))
            if l in qw:
                qf = O.fp8_e4m3_to_f64(qw[l][0])
                if l == 0:
                    idx_of[l], pool, _ = O.hier_pool_select(qf, qw[l][1], kf, cap, K, 8, npb)
                else:
                    idx_of[l], _, _ = O.reindex_topk(qf, qw[l][1], kf, cap, pool, 8, K)
            else:
                idx_of[l] = idx_of[l - 1]
            pk, sc = O.kv_quant_fp4(O.bf16_bits_to_f64(rows_of(l, idx_of[l][idx_of[l] >= 0])))
            O.sparse_attn_decode_rows(O.bf16_bits_to_f64(q[l]), O.kv_dequant_fp4(pk, sc), 1.0)
    return run


def oracle_prepare_encoder(cfg, seq: int):
    """The whole csa2_encoder step for ONE sequence: inputs drawn from synth (untimed) and
    the oracle's run (timed): the window-only layers' writes and attentions, then per group
    the new row, the scan with top-K over the group's keys and the group's attentions."""
    from oracle import fp4kv_oracle as O
    seed, cap, H, H_I, K = cfg["seed"], cfg["cap"], cfg["H"], cfg["H_I"], cfg["K"]
    G, NG, NS, nw = cfg["group"], cfg["groups"], cfg["swa_layers"], cfg["swa"]
    src = [NS + g * G for g in range(NG)]
    rows = torch.arange(cap, dtype=torch.int64)
    keys = [synth.indexer_keys(seed, seq, rows, DK, True, source=src[g]).numpy() for g in range(NG)]
    qw = []
    for g in range(NG):
        qi, w = synth.indexer_query(seed, src[g], seq + 1, H_I, fp8=True)
        qw.append((qi[seq].numpy(), w[seq].double().numpy()))
    q = [_bits(synth.attn_query(seed, l, seq + 1, H, D)[seq]) for l in range(NS + NG * G)]
    x_new = [_bits(synth.kv_rows(seed, src[g], 10 ** 6, torch.tensor([seq]), D)) for g in range(NG)]
    win = []
    for l in range(NS):
        wr = _bits(synth.kv_rows(seed, SWA_LAYER + l, seq, torch.arange(cap - nw, cap, dtype=torch.int64), D))
        wr[-1] = _bits(synth.kv_rows(seed, SWA_LAYER + l, 10 ** 6, torch.tensor([seq]), D))[0]  # this step's row
        win.append(wr)

    def run():
        for l in range(NS):
            vw = O.e4m3_decode(O.swa_quant_fp8(O.bf16_bits_to_f64(win[l])))
            O.sparse_attn_decode_rows(O.bf16_bits_to_f64(q[l]), vw, 1.0)
        for g in range(NG):
            O.kv_quant_fp4(O.bf16_bits_to_f64(x_new[g]))
            kf = O.fp8_e4m3_to_f64(keys[g])
            idx, _ = O.indexer_topk(O.fp8_e4m3_to_f64(qw[g][0]), qw[g][1], kf, cap, K)
            sel = idx[idx >= 0]
            xr = _bits(synth.kv_rows(seed, src[g], seq, torch.as_tensor(sel), D))
            xr[sel == cap - 1] = x_new[g][0]
            vh = O.kv_dequant_fp4(*O.kv_quant_fp4(O.bf16_bits_to_f64(xr)))
            for j in range(G):
                O.sparse_attn_decode_rows(O.bf16_bits_to_f64(q[src[g] + j]), vh, 1.0)
    return run


def oracle_prepare_quant(cfg, rows=2048):
    from oracle import fp4kv_oracle as O
    x = _bits(synth.kv_rows(cfg["seed"], 0, 0, torch.arange(rows, dtype=torch.int64), D, heavy_frac=0.001))
    return lambda: O.kv_quant_fp4(O.bf16_bits_to_f64(x))


def oracle_sample(cfg_name, cfg, i: int):
    """One bounded sample of the workload for the oracle: (run, work). Building the inputs
    happens here, outside any timing; run() is the oracle's work on them. work is in the
    metric's unit: GB read + written for the quant sweep, else tokens (one sequence's whole
    step)."""
    if cfg_name == "quant":
        return oracle_prepare_quant(cfg), 2048 * (2 * D + ROW_BYTES) / 1e9
    if cfg_name == "csa2_encoder":
        return oracle_prepare_encoder(cfg, i % cfg["B"]), 1.0
    if "layers" in cfg:
        return oracle_prepare_layers(cfg, i % cfg["B"]), 1.0
    return oracle_prepare_decode(cfg, i % cfg["B"]), 1.0


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def _oracle_rate(cfg_name, cfg, budget_s, threads=None):
    """(work per second, samples, seconds, threads used) of the oracle on whole samples,
    taken until budget_s seconds of oracle time have passed (at least one sample); only
    run() is timed, the inputs are built outside."""
    from contextlib import nullcontext
    try:
        from threadpoolctl import threadpool_limits
        ctx = threadpool_limits(limits=threads, user_api="blas") if threads else nullcontext()
    except Exception:
        ctx = nullcontext()
    with ctx:
        used = oracle_threads()
        el, work, n = 0.0, 0.0, 0
        while n == 0 or el < budget_s:
            run, w = oracle_sample(cfg_name, cfg, n)
            t0 = time.perf_counter()
            run()
            el += time.perf_counter() - t0
            work += w
            n += 1
    return work / el, n, el, used


def cpu_baseline(cfg_name, cfg, budget_s=10.0):
    """Oracle throughput on a bounded sample of the workload, in the metric's unit: once
    single-threaded and once with the BLAS pool at its default size (the oracle's only
    parallelism is numpy's BLAS), with the host's core count."""
    unit = "GB/s" if cfg_name == "quant" else "tokens/s"
    what = ("rows of the quant sweep, 2048 per sample" if cfg_name == "quant" else
            "sequences, the whole step of one sequence per sample" +
            (f" ({cfg['layers']} layers)" if "layers" in cfg else "") +
            (" (20 layers)" if cfg_name == "csa2_encoder" else ""))
    v1, n1, el1, _ = _oracle_rate(cfg_name, cfg, budget_s, threads=1)
    vt, nt, elt, used = _oracle_rate(cfg_name, cfg, budget_s)
    return {"value": vt, "unit": unit, "cores": used, "nproc": os.cpu_count(), "kind": "oracle",
            "sample": f"{nt} {what} in {elt:.1f} s, BLAS on {used} threads",
            "single_thread": {"value": v1, "unit": unit, "cores": 1,
                              "sample": f"{n1} {what} in {el1:.1f} s"}}


# ----------------------------------------------------------------------------------------

def run_reference(args, cfg_name, cfg):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    unit = "GB/s" if cfg_name == "quant" else "tokens/s"
    # the oracle is plain CPU code: one untimed sample stands in for the warm-up steps
    oracle_sample(cfg_name, cfg, 0)[0]()
    el, work = 0.0, 0.0
    for i in range(args.steps):
        run, w = oracle_sample(cfg_name, cfg, i)  # inputs built outside the timing
        t0 = time.perf_counter()
        run()
        el += time.perf_counter() - t0
        work += w
    value = work / el
    cores = oracle_threads()
    sample = ("2048 rows of the sweep per step" if cfg_name == "quant" else
              "one sequence of the batch per step (its whole step" +
              (f", all {cfg['layers']} layers" if "layers" in cfg else "") + ")")
    line = {"metric": METRIC, "impl": "reference", "value": value, "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el * 1e3 / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg["workload"], "name": cfg_name, "sample": sample,
                       "timing": "oracle compute only, summed over the steps; inputs drawn "
                                 "from the generator outside the timing; one untimed warm-up "
                                 "sample"},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "nproc": os.cpu_count(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def phase(msg):
    print(f"[bench] {time.strftime('%H:%M:%S')} {msg}", file=sys.stderr, flush=True)


def main(argv=None):
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="long", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch each step eagerly instead of "
                    "replaying a captured CUDA graph")
    for key, kind in OVERRIDES:
        ap.add_argument("--" + key.replace("_", "-"), type=kind, default=None,
                        help=f"override the configuration's {key}")
    args = ap.parse_args(argv)
    cfg_name, cfg = args.config, apply_overrides(CONFIGS[args.config], args)
    if args.impl == "reference":
        return run_reference(args, cfg_name, cfg)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world, rank, local = dist_env()
    if world != args.gpus and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")

    import fp4_sparse_attention_kv_b200 as fk
    fk.lib()
    phase(f"building workload {cfg_name}")
    if cfg_name == "quant":
        wl = QuantWorkload(cfg, fk, device, rank)
    elif cfg_name == "hier":
        wl = HierWorkload(cfg, fk, device, rank)
    elif cfg_name == "csa2_decoder":
        wl = Csa2DecoderWorkload(cfg, fk, device, rank)
    elif cfg_name == "csa2_encoder":
        wl = Csa2EncoderWorkload(cfg, fk, device, rank)
    else:
        wl = DecodeWorkload(cfg, fk, device, rank)
    streamed = sum(wl.algorithmic_bytes().values())
    if streamed > 2 * L2_BYTES:
        flush = None
        l2_note = (f"inputs larger than L2: each step streams {streamed / 1e6:.0f} MB "
                   f"(> 2 x {L2_BYTES >> 20} MiB L2), no flush")
    else:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)
        l2_note = "flushed (256 MiB write) before every timed step"
    torch.cuda.synchronize()
    for _ in range(2):  # the library's first launches set kernel attributes
        wl.step()
    torch.cuda.synchronize()
    if not args.no_graph:
        phase("graph capture")
        wl.capture_graphs()

    phase("clock sampler")
    sampler = ClockSampler(local)
    barrier(world, device)
    phase("timed steps")
    total_ms, prof = timed_steps(wl, args.steps, args.warmup, flush, sampler, fk)
    barrier(world, device)
    step_ms = max_over_ranks(total_ms / args.steps, world, device)
    phase("end-to-end steps")
    e2e_ms, h2d, d2h = e2e_steps(wl, args.steps, args.warmup)
    e2e_step_ms = max_over_ranks(e2e_ms / args.steps, world, device)

    tokens = wl.tokens_per_step * world
    alg = wl.algorithmic_bytes()
    peak, peak_kind = measured_peaks()
    if cfg_name == "quant":
        value = alg["kv_quant_fp4"] * world / (step_ms * 1e-3) / 1e9
        unit = "GB/s"
        e2e_value = alg["kv_quant_fp4"] * world / (e2e_step_ms * 1e-3) / 1e9
        dom = "kv_quant_fp4"
    else:
        value = tokens / (step_ms * 1e-3)
        unit = "tokens/s"
        e2e_value = tokens / (e2e_step_ms * 1e-3)
        dom = max(("index_score", "sparse_attn"), key=lambda k: prof[k][1])
    n_l, ms_l = prof[dom]
    per_launch_ms = ms_l / max(1, n_l)
    bytes_per_launch = alg[dom] / max(1, n_l / args.steps)
    if dom == "sparse_attn":
        # 4*H*d flops per gathered row of 288 bytes (455 flop/B at H = 64) is above the
        # ridge point of the measured peaks: the attention is bound by the tensor cores
        rows = getattr(wl, "attn_rows_per_step", alg[dom] / ROW_BYTES)
        flops_per_launch = rows / max(1, n_l / args.steps) * attn_flops_per_row(wl.H)
        tpeak, tpeak_kind = measured_tensor_peak()
        achieved = flops_per_launch / (per_launch_ms * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": tpeak,
                "unit": "TFLOP/s", "frac": achieved / tpeak, "peak_kind": tpeak_kind,
                "algorithmic_flops_per_launch": flops_per_launch}
    else:
        achieved = bytes_per_launch / (per_launch_ms * 1e-3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind}
    roof.update({"traffic": traffic_record(dom, cfg_name),
                 "algorithmic_bytes_per_launch": bytes_per_launch, "ms_per_launch": per_launch_ms})
    step_bytes = sum(v for k, v in alg.items())
    # the HBM target's own quantity: the algorithmic bytes of indexer_topk + sparse_attn_decode
    # (indexer keys, FP4 rows and scales) per step over the device time of the whole step
    # (quantize-on-write included: the chained kernels are timed together)
    target = None
    if cfg_name != "quant":
        tb = alg["index_score"] + alg["sparse_attn"]
        tg = tb * world / (step_ms * 1e-3) / 1e9
        target = {"kernels": "indexer_topk + sparse_attn_decode", "bound": "hbm",
                  "algorithmic_bytes_per_step": tb, "ms_per_step": step_ms, "achieved": tg,
                  "peak": peak, "unit": "GB/s", "frac": tg / peak, "peak_kind": peak_kind,
                  "time": "device time of the whole step (CUDA events, max over ranks)"}
    kernels = {k: {"launches_per_step": n / args.steps, "ms_per_step": t / args.steps,
                   "algorithmic_bytes_per_step": alg.get(k), "gbs": (alg[k] / (t / args.steps * 1e-3) / 1e9) if k in alg and t > 0 else None}
               for k, (n, t) in prof.items() if n}

    # launches per step as the library recorded them in the profiled pass (the graph replays
    # the same sequence); the workload's own count is the cross-check
    recorded = sum(n for n, _ in prof.values()) / args.steps
    if recorded and abs(recorded - wl.launches_per_step) > 1e-9:
        print(f"bench: {recorded:g} library launches per step recorded, {wl.launches_per_step} expected",
              file=sys.stderr)
    launches = recorded if recorded else wl.launches_per_step
    result = None
    if rank == 0:
        clocks = sampler.summary()
        result = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp4-e2m1/e4m3 storage; fp16 MMA, fp32 accumulate", "data": "synthetic",
            "config": {"workload": cfg["workload"], "name": cfg_name, **({"overrides": cfg["overrides"]}
                                                                          if "overrides" in cfg else {}),
                       "l2": l2_note,
                       "parallelism": f"dp{world} (independent sequences per GPU)",
                       "launch": ("one CUDA graph replay per step" if wl.graphs is not None
                                  else "eager launches"),
                       "tokens_per_step": tokens},
            "hbm_gbs_step": step_bytes * world / (step_ms * 1e-3) / 1e9,
            "roofline": roof,
            "hbm_target": target,
            "kernels": kernels,
            "gpu_launches": int(round(launches * args.steps)),
            "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "clocks": clocks,
        }
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            phase("cpu baseline (oracle)")
            result["cpu_baseline"] = cpu_baseline(cfg_name, cfg)
        print(json.dumps(result), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
