"""The reference arm of bench.py (``--impl reference``: the oracle timed on
the host cores) keeps the bench line's contract: rank 0 prints exactly one
JSON line carrying the same metric, unit, direction and workload as the
library's own line, ``impl`` = "reference", a ``cpu_baseline`` object that
describes the run and an ``e2e`` object with no host copies; every other
rank exits 0 without work or output.  Also: the roofline's numerators (the
algorithmic FLOPs and bytes) are the hand-counted ones.  Runs on the CPU
(no GPU needed)."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env, *args):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    env.update(extra_env)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", *args], cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    p = _run({}, "--steps", "2", "--warmup", "1")
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["config"]["workload"] == bench.WORKLOAD
    assert (d["config"]["M"], d["config"]["K"], d["config"]["N"], d["config"]["r"]) == (
        bench.CASE.M, bench.CASE.K, bench.CASE.N, bench.CASE.r)
    assert d["n_gpus"] == 1 and d["data"] == "synthetic" and d["vs_baseline"] is None
    # the warm-up floor of the contract holds even when fewer are asked for
    assert d["warmup"] >= 3
    assert 1 <= d["steps"] <= d["steps_requested"] == 2
    assert d["value"] > 0 and d["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["unit"] == d["unit"]
    assert cb["value"] == d["value"]
    # value = the layer's FLOPs on the sampled rows / the time per step
    rows = int(cb["sample"].split()[0])
    assert cb["sample"].startswith(f"{rows} of {bench.CASE.M} rows")
    fl = bench.layer_flops(rows, bench.CASE.K, bench.CASE.N, bench.CASE.r)
    assert abs(d["value"] - fl / (d["ms_per_step"] * 1e-3) / 1e12) <= 1e-9 * d["value"]
    e2e = d["e2e"]
    assert e2e == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    p = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--steps", "1", "--warmup", "3")
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


def test_roofline_numerators_are_the_algorithmic_counts():
    # the headline layer M=4096, K=N=3072, r=32, counted by hand:
    # FP4 GEMM 2·M·N·K = 77 309 411 328 and low-rank 2·M·r·(K+N) = 1 610 612 736
    assert bench.layer_flops(4096, 3072, 3072, 32) == 78_920_024_064
    # quantize: read x 25 165 824 + s 12 288 + L1ᵀ 196 608; write codes
    # 6 291 456 + scales 786 432 + xl 524 288
    assert bench.quantize_bytes(4096, 3072, 32) == 32_976_896
    # no low-rank branch: no L1ᵀ and no xl
    assert bench.quantize_bytes(4096, 3072, 0) == 32_976_896 - 196_608 - 524_288
