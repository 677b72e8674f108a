"""Host-side logic of bench.py on the CPU: the multi-rank plumbing (gloo, two ranks) and the
reference arm's output contract. No GPU is used."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    ws, r, _ = bench.dist_env()
    dist = bench.init_dist(ws, "gloo")
    bench.barrier(ws)
    # each rank times a different duration: the job's time is the slowest rank's
    got = bench.max_over_ranks(1.0 + 2.5 * r, ws)
    bench.barrier(ws)
    out[r] = got
    dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        assert dict(out) == {0: 3.5, 1: 3.5}


def test_max_over_ranks_is_identity_on_one_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25, 1) == 4.25


@pytest.mark.timeout(300)
def test_reference_arm_prints_one_line_on_rank0_only():
    """The reference arm (the oracle on the host cores) prints one JSON line on rank 0 and
    exits 0 without work on the other ranks."""
    outs = []
    for rank in (0, 1):
        env = dict(os.environ, WORLD_SIZE="2", RANK=str(rank), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
        r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny",
                            "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                           capture_output=True, text=True, timeout=280)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append([ln for ln in r.stdout.splitlines() if ln.strip()])
    assert outs[1] == []
    assert len(outs[0]) == 1
    line = json.loads(outs[0][0])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"


def test_size_overrides_apply_and_are_reported():
    import argparse
    sys.path.insert(0, ROOT)
    import bench
    ns = argparse.Namespace(B=4, cap=None, H=None, H_I=None, K=512, npb=None, seed=None)
    cfg = bench.apply_overrides(bench.CONFIGS["decode32"], ns)
    assert (cfg["B"], cfg["K"], cfg["cap"]) == (4, 512, 65536) and cfg["overrides"] == {"B": 4, "K": 512}
    assert "overrides" not in bench.CONFIGS["decode32"]  # the table itself is unchanged
    with pytest.raises(SystemExit):
        bench.apply_overrides(bench.CONFIGS["quant"], ns)  # the sweep has no batch or top-K


@pytest.mark.timeout(300)
def test_cpu_baseline_reports_single_and_threaded_runs():
    """The oracle baseline is timed single-threaded and with the BLAS pool, and names the
    host's core count and the threads it used (inputs are built outside the timing)."""
    sys.path.insert(0, ROOT)
    import bench
    cb = bench.cpu_baseline("tiny", bench.CONFIGS["tiny"], budget_s=0.5)
    assert cb["kind"] == "oracle" and cb["unit"] == "tokens/s" and cb["value"] > 0
    assert cb["nproc"] == os.cpu_count() and cb["cores"] >= 1
    st = cb["single_thread"]
    assert st["cores"] == 1 and st["value"] > 0 and "sequences" in st["sample"]


def test_layered_oracle_sample_runs_every_layer_on_a_small_case():
    """The 20-layer oracle sample (hier schedule) runs on a reduced size: it calls the
    Full layer's pool select once, a Reindex per even layer and one attention per layer."""
    sys.path.insert(0, ROOT)
    import bench
    from oracle import fp4kv_oracle as O
    cfg = dict(bench.CONFIGS["hier"], cap=4096, K=64, npb=32, layers=6)
    calls = {"hier": 0, "reindex": 0, "attn": 0}
    orig = (O.hier_pool_select, O.reindex_topk, O.sparse_attn_decode_rows)

    def count(name, f):
        def g(*a, **k):
            calls[name] += 1
            return f(*a, **k)
        return g
    try:
        O.hier_pool_select = count("hier", orig[0])
        O.reindex_topk = count("reindex", orig[1])
        O.sparse_attn_decode_rows = count("attn", orig[2])
        run, work = bench.oracle_sample("hier", cfg, 1)
        run()
    finally:
        O.hier_pool_select, O.reindex_topk, O.sparse_attn_decode_rows = orig
    assert work == 1.0 and calls == {"hier": 1, "reindex": 3, "attn": 6}


def test_traffic_records_are_current_or_ignored_and_near_the_algorithmic_bytes():
    """profiles/traffic.txt: a record is used only while its kernel source digest matches; every
    record that matches carries DRAM bytes between 1.0x and 1.5x of the launch's algorithmic
    bytes (keys for the scan; gathered rows for the attention), so a record copied to the
    wrong workload or a capture of the wrong kernel fails here."""
    sys.path.insert(0, ROOT)
    import bench
    cfgs = bench.CONFIGS
    key_bytes = {"index_score": lambda c: c["B"] * c["cap"] * (128 if c.get("fp8") else 256),
                 "sparse_attn": lambda c: c["B"] * c["K"] * bench.ROW_BYTES}
    checked = 0
    for line in open(os.path.join(ROOT, "profiles", "traffic.txt")):
        if not line.startswith("kernel="):
            continue
        rec = dict(kv.split("=", 1) for kv in line.split())
        got = bench.traffic_record(rec["kernel"], rec["workload"])
        if got is None:  # the kernel has changed since the capture: the bench reports null
            continue
        assert got == float(rec["dram_bytes_per_launch"])
        alg = key_bytes[rec["kernel"]](cfgs[rec["workload"]])
        assert 1.0 <= got / alg <= 1.5, (rec, got / alg)
        checked += 1
    assert bench.traffic_record("sparse_attn", "no_such_workload") is None
    assert checked >= 1
