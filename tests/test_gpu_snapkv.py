"""GPU parity of the SnapKV-style eviction pre-pass (a0) and of the stacked
path (eviction -> channel pruning -> decode), against the CPU oracle.

Scores are fp32 tensor-core sums on the GPU and fp64 in the oracle, so the
kept-token sets are compared exactly except for swaps between tokens whose
oracle pooled scores tie with the selection threshold to within 1e-4
relative; such swaps are counted and must stay under 0.01 % of the kept
prefix tokens.  Gathered K/V rows are compared bit for bit; the downstream
prune/decode parity runs both sides on the GPU's compacted cache."""
import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (KCache, spark_decode_attn, spark_device_status, spark_lambda_to_T,
                                        spark_snapkv_evict, spark_tail_append, spark_workspace_bytes,
                                        workspace, SPARK_OP_DECODE, SPARK_OP_SNAPKV)
from channel_pruned_decode_b200.synth import WORKLOADS, make_decode_step, make_prefill, scaled
from tests._parity import assert_out_close, compare_masks, mask_np, run_prune, to_np, unpack_vals

pytestmark = pytest.mark.gpu
D = 128
DEV = "cuda"


def _evict(wl, pre):
    R, H, S, G, W, keep = wl.rows, wl.Hkv, wl.S, wl.G, wl.W, wl.keep
    k_out = torch.empty((R, H, keep, D), dtype=pre["k"].dtype, device=DEV)
    v_out = torch.empty_like(k_out)
    idx = torch.empty((R, H, keep), dtype=torch.int32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_SNAPKV, R, H, G, S, D, 0, 0))
    spark_snapkv_evict(pre["k"], pre["v"], pre["q_obs"], G, W, keep, wl.pool, k_out, v_out, idx, ws)
    torch.cuda.synchronize()
    return k_out, v_out, idx, ws


def _gpu_scores(ws, BH, P):
    return ws[256:256 + BH * P * 4].view(torch.float32).reshape(BH, P).cpu().numpy()


def _check_selection(idx_g, idx_o, pooled_o, keep, W):
    """Exact set equality except near-tie swaps; returns the swap count."""
    kp = keep - W
    swaps = 0
    for b in range(idx_g.shape[0]):
        g, o = set(idx_g[b, :kp].tolist()), set(idx_o[b, :kp].tolist())
        diff = (g - o) | (o - g)
        if diff:
            thr = np.sort(pooled_o[b])[::-1][kp - 1]
            for t in diff:
                assert abs(pooled_o[b, t] - thr) <= 1e-4 * abs(thr), (b, t, pooled_o[b, t], thr)
            swaps += len(g - o)
        assert np.array_equal(idx_g[b, kp:], np.arange(idx_g.shape[1] - kp) + pooled_o.shape[1])
    return swaps


def _valid_idx(idx, S, keep, W):
    i = idx.reshape(-1, keep).cpu().numpy()
    assert np.all(np.diff(i, axis=1) > 0), "indices must be strictly ascending"
    assert i.min() >= 0 and i.max() < S
    assert np.array_equal(i[:, keep - W:], np.tile(np.arange(S - W, S), (i.shape[0], 1)))


@pytest.mark.parametrize("S,keep,G,W,pool", [(300, 128, 4, 32, 7), (1000, 400, 4, 16, 7), (513, 40, 2, 8, 3),
                                             (64, 64, 4, 32, 7), (777, 33, 8, 16, 1)])
def test_snapkv_small(S, keep, G, W, pool):
    wl = scaled(WORKLOADS["evict"], B=2, Hkv=3, S=S, keep=keep, G=G, W=W, pool=pool, seed=S + keep)
    pre = make_prefill(wl, DEV)
    k_out, v_out, idx, ws = _evict(wl, pre)
    BH, P = wl.BH, S - W
    _valid_idx(idx, S, keep, W)
    k_np = to_np(pre["k"]).reshape(BH, S, D)
    q_np = to_np(pre["q_obs"]).reshape(BH * G, W, D)
    sc_o = oracle.snapkv_scores(q_np, k_np, G)
    np.testing.assert_allclose(_gpu_scores(ws, BH, P), sc_o, rtol=2e-4, atol=1e-7)
    pooled = oracle.snapkv_pool(sc_o, pool)
    idx_o = oracle.snapkv_select(pooled, S, W, keep)
    swaps = _check_selection(idx.reshape(BH, keep).cpu().numpy(), idx_o, pooled, keep, W)
    assert swaps <= max(1, 1e-4 * BH * (keep - W))
    ig = idx.reshape(BH, keep).long()
    for src, dst in ((pre["k"], k_out), (pre["v"], v_out)):
        want = torch.gather(src.reshape(BH, S, D), 1, ig[..., None].expand(-1, -1, D))
        assert torch.equal(dst.reshape(BH, keep, D), want)


def test_evict_then_prune_then_decode_256_steps():
    """The `evict` workload: B=32, 8 kv heads, S=8192 -> keep 2048 (window 32,
    max-pool 7), then lambda=0.5 pruning and 256 decode steps; the oracle
    checks a sample of heads at several steps."""
    wl = WORKLOADS["evict"]
    pre = make_prefill(wl, DEV)
    k_out, v_out, idx, ws = _evict(wl, pre)
    BH, S, G, W, keep = wl.BH, wl.S, wl.G, wl.W, wl.keep
    _valid_idx(idx, S, keep, W)
    sel = np.array([0, 77, 150, 255])
    k_np = to_np(pre["k"].reshape(BH, S, D)[sel])
    q_np = to_np(pre["q_obs"].reshape(BH * G, W, D)[torch.as_tensor(
        np.concatenate([np.arange(b * G, (b + 1) * G) for b in sel]), device=DEV)])
    sc_o = oracle.snapkv_scores(q_np, k_np, G)
    np.testing.assert_allclose(_gpu_scores(ws, BH, S - W)[sel], sc_o, rtol=2e-4, atol=1e-7)
    pooled = oracle.snapkv_pool(sc_o, wl.pool)
    idx_o = oracle.snapkv_select(pooled, S, W, keep)
    idx_g = idx.reshape(BH, keep).cpu().numpy()
    swaps = _check_selection(idx_g[sel], idx_o, pooled, keep, W)
    assert swaps <= max(1, 1e-4 * len(sel) * (keep - W))
    # the gather on every one of the 256 heads: kept K and V rows are the
    # source rows at the kept indices, bit for bit
    ig = idx.reshape(BH, keep).long()
    for src, dst in ((pre["k"], k_out), (pre["v"], v_out)):
        want = torch.gather(src.reshape(BH, S, D), 1, ig[..., None].expand(-1, -1, D))
        assert torch.equal(dst.reshape(BH, keep, D), want)

    # stacked: prune the compacted keys with the same window queries.  The
    # oracle's side gathers the keys at the oracle's own kept indices, on the
    # sampled heads whose kept set agrees with the GPU's
    agree = np.array([np.array_equal(idx_g[b], idx_o[i]) for i, b in enumerate(sel)])
    assert agree.sum() >= len(sel) - 1
    sel, idx_o, k_np = sel[agree], idx_o[agree], k_np[agree]
    q_np = q_np.reshape(-1, G, W, D)[agree].reshape(-1, W, D)
    T = spark_lambda_to_T(wl.lam)
    kc = run_prune(k_out, pre["q_obs"], G, W, T)
    torch.cuda.synchronize()
    selt = torch.as_tensor(sel, device=DEV)
    kc_np = np.take_along_axis(k_np, idx_o[..., None].astype(np.int64), axis=1)
    qn_o = oracle.qnorm(q_np, G)
    m_o, v_o, st_o = oracle.prune(kc_np, qn_o, T)
    m_g = mask_np(kc)[sel]
    rep = compare_masks(m_g, m_o, kc_np, qn_o, T)
    assert rep["mismatch"] == rep["near_tie"] and rep["mismatch"] <= 1e-4 * rep["tokens"], rep
    cap = wl.tail_cap
    kt = torch.zeros((wl.rows, wl.Hkv, cap, D), dtype=wl.torch_dtype, device=DEV)
    vt = torch.zeros_like(kt)
    wsd = workspace(spark_workspace_bytes(SPARK_OP_DECODE, wl.rows, wl.Hkv, G, keep, D, T, cap))
    out = torch.empty((wl.rows, wl.Hq, D), dtype=torch.float32, device=DEV)
    qsel = torch.as_tensor(np.concatenate([np.arange(b * G, (b + 1) * G) for b in sel]), device=DEV)
    v_src = to_np(pre["v"].reshape(BH, S, D)[selt])
    vv_np = np.take_along_axis(v_src, idx_o[..., None].astype(np.int64), axis=1)
    for step in range(wl.steps):
        stp = make_decode_step(wl, step, DEV)
        spark_tail_append(stp["k_new"], stp["v_new"], kt, vt, wl.rows, wl.Hkv, D, cap, step)
        spark_decode_attn(stp["q"], kc, v_out, kt, vt, cap, step + 1, G, out, wsd)
        if step in (0, 100, 255):
            torch.cuda.synchronize()
            o_ref = oracle.decode(to_np(stp["q"].reshape(BH * G, D)[qsel]), m_o, v_o, qn_o, st_o, vv_np,
                                  to_np(kt.reshape(BH, cap, D)[selt]), to_np(vt.reshape(BH, cap, D)[selt]),
                                  step + 1, G)
            assert_out_close(out.reshape(BH * G, D)[qsel].cpu().numpy(), o_ref, f"evict step {step}")
    torch.cuda.synchronize()
    assert spark_device_status(wsd) == 0
