"""Failure detection on the GPU without a fault: a bounded device wait is made
to run out on purpose (an mbarrier that nothing arrives on), the status word
reports SPARK_ERR_TIMEOUT, the wait ends at its limit, and the context stays
usable for real work afterwards."""
import time

import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (spark_device_status, spark_selftest_wait_timeout, workspace,
                                        SparkError)
from channel_pruned_decode_b200.binding import SPARK_ERR_TIMEOUT
from channel_pruned_decode_b200.synth import WORKLOADS, make_prefill, scaled
from tests._parity import mask_np, run_prune, to_np

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    ws = workspace(256)
    assert spark_device_status(ws) == 0
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    spark_selftest_wait_timeout(ws, 20000)  # 20 ms
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert 0.015 <= dt <= 5.0, dt            # it waited about its limit, then returned
    assert spark_device_status(ws, clear=True) == SPARK_ERR_TIMEOUT
    assert spark_device_status(ws) == 0      # cleared


def test_context_usable_after_timeout():
    ws = workspace(256)
    spark_selftest_wait_timeout(ws, 1000)
    assert spark_device_status(ws) == SPARK_ERR_TIMEOUT
    wl = scaled(WORKLOADS["tiny"], S=300, Hkv=2, dtype="bf16", seed=4)
    pre = make_prefill(wl, "cuda")
    kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, 26)
    torch.cuda.synchronize()
    BH = wl.rows * wl.Hkv
    qn = oracle.qnorm(to_np(pre["q_obs"]).reshape(BH * wl.G, -1, 128), wl.G)
    m, _, _ = oracle.prune(to_np(pre["k"]).reshape(BH, 300, 128), qn, 26)
    assert np.array_equal(mask_np(kc), m)


def test_selftest_rejects_bad_limits():
    ws = workspace(256)
    with pytest.raises(SparkError):
        spark_selftest_wait_timeout(ws, 0)
    with pytest.raises(SparkError):
        spark_selftest_wait_timeout(ws, 2000000)
