"""bench.py's own arithmetic and output contract, on the CPU.

* the algorithmic bytes behind `roofline.achieved` (K + V of every filled
  slot once, plus every write), by hand for the throughput workload, a
  ragged batch and E4M3 storage;
* the kernel-source hash gate on the committed DRAM-traffic figure;
* the reference arm (`--impl reference`, the CPU oracle) prints one JSON line
  with the contract's keys, on the small workload.
"""
import importlib.util
import json
import os
import subprocess
import sys

import numpy as np
import pytest

from attention_lf_decode_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_bytes_throughput_by_hand():
    b = _bench()
    cfg = synth.CONFIGS["throughput"]
    by = b.algorithmic_bytes(cfg, cfg.budget)
    rows = 64 * 8
    assert by["kv_read"] == rows * 4096 * 128 * 2 * 2 == 1_073_741_824
    # out fp32 [64, 32, 128], new K and V rows, position and evicted index per row
    assert by["writes"] == 64 * 32 * 128 * 4 + rows * 128 * 2 * 2 + rows * 4 + rows * 4 == 1_314_816
    assert by["algorithmic"] == 1_075_056_640


def test_algorithmic_bytes_ragged_and_e4m3():
    b = _bench()
    cfg = synth.CONFIGS["ragged"]
    nb = synth.SynthDecode(cfg).seq_budgets()
    by = b.algorithmic_bytes(cfg, nb)
    assert by["kv_read"] == int(nb.astype(np.int64).sum()) * 8 * 128 * 2 * 2
    by8 = b.algorithmic_bytes(synth.CONFIGS["throughput"], 4096, kv_bytes=1)
    assert by8["kv_read"] == 1_073_741_824 // 2


def test_traffic_is_reported_only_for_the_profiled_source():
    b = _bench()
    t = b.ncu_traffic()
    with open(b.PROFILE_SUMMARY) as f:
        txt = f.read()
    if b.kernel_hash() in txt:
        assert t is not None and t > 1e9
    else:
        assert t is None


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, cwd=ROOT, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.parametrize("args", [["--kv", "fp8"], ["--score", "alpha_l1v"],
                                  ["--config", "ragged"]])
def test_reference_arm_options(args):
    env = dict(os.environ, OMP_NUM_THREADS="1")
    if "--config" not in args:
        args = ["--config", "tiny"] + args
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"] + args,
                       capture_output=True, text=True, cwd=ROOT, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert json.loads(r.stdout.splitlines()[-1])["value"] > 0
