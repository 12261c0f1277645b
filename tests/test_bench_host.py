"""Host-side pieces of bench.py on CPU: the reference arm's JSON line, the
L2-flush decision and the one-core oracle baseline (no GPU is used)."""
import json
import os
import subprocess
import sys

import numpy as np

import synth
from synth import TINY, NANO_DECODE, ULTRA_PREFILL

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line(built_oracle):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, env=env, stdout=subprocess.PIPE,
                       stderr=subprocess.PIPE, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_is_at_least_three(built_oracle):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env, stdout=subprocess.PIPE,
                       stderr=subprocess.PIPE, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert json.loads(r.stdout.strip().splitlines()[-1])["warmup"] == 3


def test_l2_flush_only_for_weights_that_fit_in_l2():
    import bench
    assert bench.weight_bytes_of(TINY) < bench.L2_BYTES
    assert "L2 flushed" in bench.l2_note(TINY)
    for w in (NANO_DECODE, ULTRA_PREFILL):
        assert bench.weight_bytes_of(w) > 2 * bench.L2_BYTES
        assert "no flush" in bench.l2_note(w)
    # ~22 GB of bf16 weights at the Ultra widths
    assert abs(bench.weight_bytes_of(ULTRA_PREFILL) / 1e9 - 21.886) < 0.01


def test_no_target_for_a_layer_whose_weights_fit_in_l2():
    """A latency-bound layer (its weights fit in L2) is reported with no target; the others are held to
    60% of the burst bf16 peak at prefill sizes and 70% of HBM at decode sizes."""
    sys.path.insert(0, ROOT)
    import bench
    summary = {"layer_frac_of_burst_bf16": 0.7, "layer_frac_of_hbm": 0.5}
    t = bench.target_of(TINY, summary, prefill=False)
    assert t["target"] is None and t["met"] is None and "latency" in t["note"]
    t = bench.target_of(ULTRA_PREFILL, summary, prefill=True)
    assert t == {"metric": "layer_frac_of_burst_bf16", "value": 0.7, "target": 0.6, "met": True}
    t = bench.target_of(NANO_DECODE, summary, prefill=False)
    assert t == {"metric": "layer_frac_of_hbm", "value": 0.5, "target": 0.7, "met": False}


def test_one_core_baseline_restores_the_thread_count(built_oracle):
    import ctypes
    import torch
    import bench
    host = synth.host_inputs(NANO_DECODE)
    dev = {"x": torch.from_numpy(host["x"].view(np.int16)).view(torch.bfloat16)}
    gomp = ctypes.CDLL("libgomp.so.1")
    gomp.omp_get_max_threads.restype = ctypes.c_int
    before = gomp.omp_get_max_threads()
    cb = bench.cpu_baseline_one_core(NANO_DECODE, host, dev, target_s=1.0)
    assert cb["cores"] == 1 and cb["kind"] == "oracle" and cb["value"] > 0
    assert gomp.omp_get_max_threads() == before
