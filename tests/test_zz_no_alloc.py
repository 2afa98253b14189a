"""The allocation-free pruning entry point, spark_prune_noalloc.

It exists for callers that cannot allocate device memory where they prune
(a serving engine whose pool owns the device after start-up, a plugin host
that passes only input/output buffers); it uses the library's fixed per-device
scratch array in place of a workspace.  Here it is called through the C ABI
and compared with spark_prune, the workspace entry point, on two calls in a
row: the second call reuses the scratch array the first one left behind.

Collected last on purpose (file name), so a failure here never hides the
result of another test; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from channel_pruned_decode_b200 import (KCache, SparkError, spark_lambda_to_T, spark_prune,
                                        spark_prune_noalloc, spark_workspace_bytes, workspace,
                                        SPARK_OP_PRUNE)
from channel_pruned_decode_b200.synth import WORKLOADS, make_prefill, scaled

pytestmark = pytest.mark.gpu

STATS_RTOL = 2e-6  # same tolerance the parity tests use for the statistics


def _prune_both(wl, T):
    pre = make_prefill(wl, "cuda")
    R, H, S, D, G, W = wl.rows, wl.Hkv, wl.S, wl.D, wl.G, wl.W
    ref = KCache.empty(R, H, S, D, T, wl.torch_dtype)
    ws = workspace(spark_workspace_bytes(SPARK_OP_PRUNE, R, H, G, S, D, T, 0))
    spark_prune(pre["k"], pre["q_obs"], G, W, ref, ws)
    got = KCache.empty(R, H, S, D, T, wl.torch_dtype)
    spark_prune_noalloc(pre["k"], pre["q_obs"], G, W, got)
    torch.cuda.synchronize()
    return ref, got


def _assert_same(ref: KCache, got: KCache):
    assert torch.equal(ref.mask, got.mask)
    assert torch.equal(ref.vals, got.vals)
    assert torch.equal(ref.qn, got.qn)
    np.testing.assert_allclose(got.stats.cpu().numpy(), ref.stats.cpu().numpy(), rtol=STATS_RTOL, atol=0)


def test_noalloc_matches_workspace_prune_two_calls():
    # first call: 8 heads x 9000 tokens; second call: a different, smaller
    # shape and dtype, so it runs over what the first call left in the scratch
    first = scaled(WORKLOADS["llama1l"], S=9000, seed=21)
    second = scaled(WORKLOADS["tiny"], S=700, Hkv=3, seed=22)
    for wl, lam in ((first, 0.8), (second, 0.5)):
        ref, got = _prune_both(wl, spark_lambda_to_T(lam))
        _assert_same(ref, got)


def test_noalloc_rejects_shapes_beyond_scratch():
    # 4 MiB of scratch holds 262128 (head, 256-token chunk) partials
    kc = KCache(1, 1024, 1 << 16, 128, 26, torch.bfloat16,
                torch.empty(16, dtype=torch.int32, device="cuda"),
                torch.empty(16, dtype=torch.bfloat16, device="cuda"),
                torch.empty(16, dtype=torch.float32, device="cuda"),
                torch.empty(16, dtype=torch.float64, device="cuda"))
    k = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(SparkError) as e:
        spark_prune_noalloc(k, k, 4, 32, kc)
    assert e.value.status == 5  # SPARK_ERR_WORKSPACE, nothing launched
