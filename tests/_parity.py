"""Test-side helpers: run the CUDA path through the C ABI binding and the CPU
oracle on the same seeded inputs, and convert the GPU cache layout to the
oracle's plain layout for comparison.  Nothing here computes the method."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from channel_pruned_decode_b200 import (KCache, spark_decode_attn, spark_prune, spark_tail_append,
                                        spark_workspace_bytes, workspace, SPARK_OP_DECODE,
                                        SPARK_OP_PRUNE, spark_lambda_to_T)

ATOL = 2e-3   # attention output tolerance: max-abs
RTOL = 1e-2   # and relative


def unpack_vals(kc: KCache) -> np.ndarray:
    """GPU interleaved value layout -> plain [B*Hkv, S, T] float32."""
    BH = kc.B * kc.Hkv
    S, T = kc.S, kc.T
    S32 = (S + 31) // 32 * 32
    v = kc.vals.float().reshape(BH, S32 // 32, T, 32).permute(0, 1, 3, 2).reshape(BH, S32, T)
    return v[:, :S].cpu().numpy()


def mask_np(kc: KCache) -> np.ndarray:
    return kc.mask.cpu().numpy().view(np.uint32).reshape(kc.B * kc.Hkv, kc.S, 4)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def run_prune(k, q_obs, G, W, T, stream=None) -> KCache:
    R, Hkv, S, D = k.shape
    kc = KCache.empty(R, Hkv, S, D, T, k.dtype, device=k.device)
    ws = workspace(spark_workspace_bytes(SPARK_OP_PRUNE, R, Hkv, G, S, D, T, 0), device=k.device)
    spark_prune(k, q_obs, G, W, kc, ws, stream)
    return kc


def compare_masks(gm: np.ndarray, om: np.ndarray, k_np, qn_np, T) -> dict:
    """Bit-exact mask comparison; any mismatching token must be a near-tie
    (T-th and (T+1)-th saliency within 1e-6 relative)."""
    diff = np.any(gm != om, axis=-1)
    n_bad = int(diff.sum())
    near = 0
    if n_bad:
        idx = np.argwhere(diff)
        for bh, t in idx:
            w = (qn_np[bh] * np.abs(k_np[bh, t])).astype(np.float32)
            srt = np.sort(w)[::-1]
            if 0 < T < len(w):
                a, b = float(srt[T - 1]), float(srt[T])
                if a == 0 or abs(a - b) <= 1e-6 * abs(a):
                    near += 1
    return {"tokens": int(diff.size), "mismatch": n_bad, "near_tie": near}


def assert_out_close(g: np.ndarray, o: np.ndarray, what=""):
    d = np.abs(g.astype(np.float64) - o.astype(np.float64))
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    assert d.max() <= ATOL, f"{what}: max-abs {d.max():.3e} > {ATOL}"
    np.testing.assert_allclose(g, o, rtol=RTOL, atol=ATOL, err_msg=what)
