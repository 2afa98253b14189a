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


def _oracle_job(S=200, T=26, Hkv=2, G=4, seed=5):
    """A CPU stand-in for bench.Job whose cache and output hold the oracle's
    own results in the library's layouts (interleaved values)."""
    import types

    import numpy as np
    import torch

    import oracle
    from channel_pruned_decode_b200.binding import KCache
    from channel_pruned_decode_b200.synth import make_decode_step, make_prefill, scaled

    wl = scaled(WORKLOADS["llama1l"], S=S, Hkv=Hkv, G=G, seed=seed)
    pre = make_prefill(wl, "cpu")
    stp = make_decode_step(wl, 0, "cpu")
    BH, D = wl.BH, wl.D
    k = pre["k"].float().numpy().reshape(BH, S, D)
    v = pre["v"].float().numpy().reshape(BH, S, D)
    qn = oracle.qnorm(pre["q_obs"].float().numpy().reshape(BH * G, wl.W, D), G)
    m, vals, st = oracle.prune(k, qn, T)
    cap = 4
    kt = torch.zeros((wl.rows, Hkv, cap, D), dtype=pre["k"].dtype)
    vt = torch.zeros_like(kt)
    kt[:, :, 0] = stp["k_new"][:, :, 0] if stp["k_new"].dim() == 4 else stp["k_new"]
    vt[:, :, 0] = stp["v_new"][:, :, 0] if stp["v_new"].dim() == 4 else stp["v_new"]
    out = oracle.decode(stp["q"].float().numpy().reshape(BH * G, D), m, vals, qn, st, v,
                        kt.float().numpy().reshape(BH, cap, D), vt.float().numpy().reshape(BH, cap, D), 1, G)
    kc = KCache.empty(wl.rows, Hkv, S, D, T, pre["k"].dtype, device="cpu")
    kc.mask.copy_(torch.from_numpy(m.view(np.int32)).reshape(kc.mask.shape))
    S32 = (S + 31) // 32 * 32
    pad = np.zeros((BH, S32, T), np.float32)
    pad[:, :S] = vals
    inter = pad.reshape(BH, S32 // 32, 32, T).transpose(0, 1, 3, 2).reshape(kc.vals.shape)
    kc.vals.copy_(torch.from_numpy(np.ascontiguousarray(inter)).to(kc.vals.dtype))
    kc.stats.copy_(torch.from_numpy(st).reshape(kc.stats.shape))
    job = types.SimpleNamespace(wl=wl, T=T, kc=kc, out=torch.from_numpy(out).reshape(wl.rows, wl.Hq, D))
    data = dict(k=k, v=v, qn=qn, q=stp["q"].float().numpy().reshape(BH * G, D),
                kt=kt.float().numpy().reshape(BH, cap, D), vt=vt.float().numpy().reshape(BH, cap, D))
    return job, data


def test_sample_parity_accounting():
    """bench's parity report: zero for a cache and output equal to the
    oracle's, and it counts a planted mask difference, a planted value
    difference and an output error."""
    import oracle

    job, d = _oracle_job()
    wl, T, G = job.wl, job.T, job.wl.G
    S = wl.S
    sel = [0, 1]
    prs, outs = [], []
    for b in sel:
        qn = d["qn"][b:b + 1]
        pr = oracle.prune(d["k"][b:b + 1], qn, T)
        prs.append((qn, pr))
        m_o, v_o, s_o = pr
        outs.append(oracle.decode(d["q"][b * G:(b + 1) * G], m_o, v_o, qn, s_o, d["v"][b:b + 1],
                                  d["kt"][b:b + 1], d["vt"][b:b + 1], 1, G))
    rep = bench._sample_parity(job, sel, prs, outs, S)
    assert rep["mask_mismatch_tokens"] == 0 and rep["vals_mismatch_tokens"] == 0
    assert rep["stats_max_rel_err"] == 0.0 and rep["decode_max_abs_err"] == 0.0
    # plant: one token's mask word, another token's first value, one output
    job.kc.mask.view(-1, S, 4)[1, 7, 0] ^= 1
    job.kc.vals.view(-1)[0] += 1.0  # token 0 of head 0, value slot 0 (interleaved layout)
    job.out.view(-1)[3] += 0.5
    rep = bench._sample_parity(job, sel, prs, outs, S)
    assert rep["mask_mismatch_tokens"] == 1 and rep["vals_mismatch_tokens"] == 1
    assert abs(rep["decode_max_abs_err"] - 0.5) < 1e-3
