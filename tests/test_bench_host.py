"""bench.py's host-side plumbing on CPU: max/sum over ranks with gloo
(world size 2), clock parsing, roofline arithmetic and argument defaults."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import bench
from moe_inputs import config


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mx = bench.max_over_ranks(10.0 + rank, world)
        sm = bench.sum_over_ranks(128.0 * 3, world)
        dist.barrier()
        out[rank] = (mx, sm)
    finally:
        dist.destroy_process_group()


def test_rank_reductions_with_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (11.0, 768.0)


def test_single_rank_reductions_are_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(7.0, 1) == 7.0


def test_clock_summary_parsing():
    c = bench.ClockSampler(0)
    c.out = ("1935, 1965, Not Active, Not Active, Not Active, Active\n"
             "1950, 1965, Not Active, Not Active, Not Active, Not Active\n"
             "garbage\n")
    s = c.summary()
    assert s["sm_mhz"] == 1942.5 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 2


def test_roofline_figures_decode_shape():
    cfg = config(2)
    counts = np.zeros(cfg.E, dtype=np.int64)
    counts[:247] = 4
    flops, nbytes = bench.roofline_figures(cfg, [counts], {})
    per_expert = 3 * cfg.H * cfg.I * 2
    assert nbytes == 248 * per_expert + 2 * cfg.T * cfg.H * 2
    assert flops == (cfg.T * cfg.k + cfg.T) * 6 * cfg.H * cfg.I


def test_default_arguments():
    a = bench.parse_args([])
    assert (a.gpus, a.config, a.impl) == (1, 2, "ours") and a.warmup >= 3


def test_profiled_traffic_scaling_and_staleness(tmp_path, monkeypatch):
    """A full-size workload's traffic is its reduced case's measured bytes scaled
    by the ratio of algorithmic bytes; a changed kernel source voids it."""
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "split_weight_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "split_weight_b200" / "csrc" / "k.cuh").write_text("kernel v1")
    h = bench.kernel_source_hash(["k.cuh"])
    rec = {"small": {"kernel_files": ["k.cuh"], "kernel_source_hash": h,
                     "dram_bytes_per_call": 1100, "algorithmic_bytes_per_call": 1000},
           "full": {"scaled_from": "small"}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(path))
    assert bench.profiled_traffic("small", 1000.0) == 1100
    assert bench.profiled_traffic("full", 5000.0) == 5500
    assert bench.profiled_traffic("absent", 5000.0) is None
    # an edit of the comments keeps the capture; an edit of the code voids it
    (tmp_path / "split_weight_b200" / "csrc" / "k.cuh").write_text(
        "// a note\nkernel  /* block\n comment */ v1 // trailing\n")
    assert bench.profiled_traffic("full", 5000.0) == 5500
    (tmp_path / "split_weight_b200" / "csrc" / "k.cuh").write_text("kernel v2")
    assert bench.profiled_traffic("full", 5000.0) is None


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` runs the CPU oracle and prints exactly one JSON
    line with the contract's keys (run as a subprocess, as the driver does)."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "1"], cwd=root, capture_output=True,
                         text=True, timeout=600, check=True).stdout
    lines = [l for l in out.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
