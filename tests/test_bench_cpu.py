"""Host-side contract of bench.py that needs no GPU: the reference arm (the
CPU oracle timed on this host) prints one JSON line with the keys the
benchmark contract asks for, ranks other than 0 exit without output, and bad
arguments are refused before any work."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

from int8_dequant_gemm_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None, timeout=300):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          env=e, capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "0", "--ref-rows", "2")
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "data", "config"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["steps"] == 1
    assert d["config"]["workload"] == "blocks12_m4096"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "0",
               env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_on_a_non_block_workload_says_unavailable():
    r = _bench("--impl", "reference", "--workload", "m_sweep")
    assert r.returncode == 0
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and "unavailable" in d


def test_bad_arguments_are_refused():
    r = _bench("--impl", "reference", "--ref-rows", "1")
    assert r.returncode != 0 and "--ref-rows" in r.stderr
    r = _bench("--workload", "no_such_workload")
    assert r.returncode != 0


def test_row_sample_holds_both_ends():
    rows = wl.sample_rows(4096, 8, seed=3)
    assert len(rows) == 8 and rows[0] == 0 and rows[-1] == 4095
    assert np.all(np.diff(rows) > 0)
    assert np.array_equal(wl.sample_rows(5, 8, seed=3), np.arange(5))
    with pytest.raises(ValueError):
        wl.sample_rows(4096, 1, seed=3)


def test_roofline_bound_and_fraction_follow_from_their_inputs():
    import bench
    peaks = {"hbm_gbs": 6540.0, "bf16_tflops": 1683.8, "bf16_tflops_sustained": 1391.3,
             "source": "measured"}
    # w13 at M = 4096: 224 flop/B, so the HBM side binds (224 * 6.54 < 1683.8)
    flops = 2 * 4096 * 4096 * 512
    nbytes = 4096 * 256 + 4096 * 16 * 4 + 4 * 4096 * 512 + 4 * 4096 * 4096
    r = bench.roofline(flops, nbytes, 33.12e-6, peaks)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6540.0
    assert r["achieved"] == pytest.approx(nbytes / 33.12e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6540.0)
    assert r["attainable_tflops"] == pytest.approx(flops / nbytes * 6.540)
    assert r["tensor_peak"] == "burst"
    # a high-intensity call binds on the tensor side, against the burst peak
    r = bench.roofline(1e12, 1e8, 1e-3, peaks)
    assert r["bound"] == "tensor" and r["peak"] == 1683.8
    assert r["frac"] == pytest.approx(1000.0 / 1683.8)
    assert bench.roofline(1e12, 1e8, 1e-3, peaks, sustained=True)["peak"] == 1391.3
