"""The benchmark's JSON-line contract, checked on the CPU: the reference arm
(the CPU oracle on a bounded sample) prints one line with every required
key, and the algorithmic byte model matches the cache layout."""
import json
import os
import subprocess
import sys

import pytest

import bench
from channel_pruned_decode_b200.synth import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny", "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT, env={**os.environ, "RANK": "0"})
    assert out.returncode == 0, out.stderr
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["vs_baseline"] is None and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny", "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT, env={**os.environ, "RANK": "1"})
    assert out.returncode == 0, out.stderr
    assert not [x for x in out.stdout.splitlines() if x.startswith("{")]


def test_warmup_below_three_is_rejected():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--warmup", "2"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode != 0 and "--warmup" in out.stderr


@pytest.mark.parametrize("name,T,per_prune,per_decode", [("long", 26, 324, 324), ("llama1l", 64, 400, 400),
                                                          ("lsweep_0.3", 90, 452, 452)])
def test_byte_model(name, T, per_prune, per_decode):
    """Per token-head: prune reads the 256-byte key row and writes the
    16-byte mask and T bf16 values; decode reads the mask, the values and the
    256-byte V row (the layout of include/spark.h)."""
    wl = WORKLOADS[name]
    bm = bench._byte_model(wl, T, 1)
    assert bm["per_token_head_prune"] == per_prune == 256 + 16 + 2 * T
    assert bm["per_token_head_decode"] == per_decode == 16 + 2 * T + 256
    units = wl.BH * wl.S
    assert units * per_prune <= bm["prune"] <= units * per_prune * 1.01
    assert units * per_decode <= bm["decode"] <= units * per_decode * 1.01


def test_byte_model_eviction():
    wl = WORKLOADS["evict"]
    bm = bench._byte_model(wl, 64, 1)
    BH, S, keep = wl.BH, wl.S, wl.keep
    # keys read once for the scores, kept K and V rows read and written
    assert bm["snapkv"] >= BH * S * 256 + 4 * BH * keep * 256
    assert bm["prune"] >= BH * keep * (256 + 16 + 128)


def test_traffic_record_matches_source():
    """The committed ncu record is reported only for the kernel source it
    was taken on, with its DRAM bytes and issue/pipe counters."""
    rec = bench._traffic_record("prune_kernel", "long")
    if rec is None:
        pytest.skip("prune.cu changed since the committed capture")
    assert rec["bytes_per_launch"] > 0
    c = rec["ncu_counters"]
    assert 0 < c["issue_active_pct"] <= 100 and c["warp_inst_per_token_head"] > 0
    assert bench._traffic_record("no_such_kernel", "long") is None
