"""GPU parity of the stacked path with PyramidKV-style layer budgets: one
eviction call over all (layer, batch) rows with a budget per row
(spark_snapkv_evict_rows), then channel pruning and decode over caches whose
rows hold different numbers of tokens (spark_kcache.lens), against the CPU
oracle run row by row on each row's own tokens.

Budgets follow the library's reading of PyramidKV (R20, spark_pyramid_keep),
checked against the oracle's own copy of the rule.  Selections are compared
with the near-tie rule of the SnapKV tests; gathered rows bit for bit; masks
and kept values bit for bit (near-ties counted); statistics to fp32-partial
rounding; decode outputs within max-abs 2e-3 / rel 1e-2."""
import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (KCache, spark_decode_attn, spark_device_status, spark_lambda_to_T,
                                        spark_prune, spark_pyramid_keep, spark_snapkv_evict_rows,
                                        spark_tail_append, spark_workspace_bytes, workspace, SPARK_OP_DECODE,
                                        SPARK_OP_PRUNE, SPARK_OP_SNAPKV)
from channel_pruned_decode_b200.synth import WORKLOADS, make_decode_step, make_prefill, scaled
from tests._parity import assert_out_close, compare_masks, mask_np, to_np, unpack_vals
from tests.test_gpu_parity import STATS_RTOL
from tests.test_gpu_snapkv import _check_selection, _gpu_scores

pytestmark = pytest.mark.gpu
D = 128
DEV = "cuda"


def _row_budgets(wl, M, beta):
    keep_l = spark_pyramid_keep(wl.L, M, beta, wl.W, wl.S)
    assert keep_l == oracle.pyramid_keep(wl.L, M, beta, wl.W, wl.S)
    return [keep_l[r // wl.B] for r in range(wl.rows)]  # row = layer * B + batch


def _evict_rows(wl, pre, keep_rows):
    R, H, S, G, W = wl.rows, wl.Hkv, wl.S, wl.G, wl.W
    cap = max(keep_rows)
    k_out = torch.full((R, H, cap, D), 7.0, dtype=pre["k"].dtype, device=DEV)  # untouched past a row's budget
    v_out = torch.full_like(k_out, 7.0)
    idx = torch.full((R, H, cap), -5, dtype=torch.int32, device=DEV)
    kr = torch.tensor(keep_rows, dtype=torch.int32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_SNAPKV, R, H, G, S, D, 0, 0))
    spark_snapkv_evict_rows(pre["k"], pre["v"], pre["q_obs"], G, W, kr, cap, wl.pool, k_out, v_out, idx, ws)
    torch.cuda.synchronize()
    assert spark_device_status(ws) == 0
    return k_out, v_out, idx, kr, ws


def _check_rows(wl, pre, keep_rows, k_out, v_out, idx, ws, sample):
    """Selections of the sampled heads against the oracle (each with its row's
    budget), every head's gather bit for bit, and the untouched tail slots."""
    R, H, S, G, W = wl.rows, wl.Hkv, wl.S, wl.G, wl.W
    BH, P, cap = R * H, S - W, k_out.shape[2]
    idx_g = idx.reshape(BH, cap).cpu().numpy()
    sc_g = _gpu_scores(ws, BH, P)
    k_np = to_np(pre["k"]).reshape(BH, S, D)
    q_np = to_np(pre["q_obs"]).reshape(BH * G, W, D)
    swaps = 0
    for bh in sample:
        keep = keep_rows[bh // H]
        sc_o = oracle.snapkv_scores(q_np[bh * G:(bh + 1) * G], k_np[bh:bh + 1], G)
        np.testing.assert_allclose(sc_g[bh:bh + 1], sc_o, rtol=2e-4, atol=1e-7)
        pooled = oracle.snapkv_pool(sc_o, wl.pool)
        idx_o = oracle.snapkv_select(pooled, S, W, keep)
        swaps += _check_selection(idx_g[bh:bh + 1, :keep], idx_o, pooled, keep, W)
    assert swaps <= max(1, 1e-4 * sum(keep_rows[b // H] - W for b in sample))
    for bh in range(BH):
        keep = keep_rows[bh // H]
        row = idx_g[bh, :keep]
        assert np.all(np.diff(row) > 0) and row.min() >= 0 and row.max() < S
        assert np.array_equal(row[keep - W:], np.arange(S - W, S))
        assert np.all(idx_g[bh, keep:] == -5)
    kk, vv = k_out.reshape(BH, cap, D), v_out.reshape(BH, cap, D)
    for bh in range(BH):
        keep = keep_rows[bh // H]
        t = torch.as_tensor(idx_g[bh, :keep], device=DEV).long()
        assert torch.equal(kk[bh, :keep], pre["k"].reshape(BH, S, D)[bh, t])
        assert torch.equal(vv[bh, :keep], pre["v"].reshape(BH, S, D)[bh, t])
        assert bool((kk[bh, keep:] == 7.0).all()) and bool((vv[bh, keep:] == 7.0).all())


def _prune_decode_rows(wl, pre, keep_rows, k_out, v_out, idx, sample, steps):
    """Prune and decode the evicted caches with per-row lengths; the oracle
    runs each sampled head on its own kept tokens."""
    R, H, G, W = wl.rows, wl.Hkv, wl.G, wl.W
    BH, cap = R * H, k_out.shape[2]
    T = spark_lambda_to_T(wl.lam)
    kr = torch.tensor(keep_rows, dtype=torch.int32, device=DEV)
    kc = KCache.empty(R, H, cap, D, T, k_out.dtype)
    kc.lens = kr
    wsp = workspace(spark_workspace_bytes(SPARK_OP_PRUNE, R, H, G, cap, D, T, 0))
    spark_prune(k_out, pre["q_obs"], G, W, kc, wsp)
    torch.cuda.synchronize()
    assert spark_device_status(wsp) == 0
    st_g = kc.stats.cpu().numpy().reshape(BH, 4)
    assert np.array_equal(st_g[:, 0], np.array([keep_rows[b // H] * (D - T) for b in range(BH)], np.float64))
    m_g_all, v_g_all = mask_np(kc), unpack_vals(kc)
    q_np = to_np(pre["q_obs"]).reshape(BH * G, W, D)
    kv = to_np(k_out).reshape(BH, cap, D)
    vvals = to_np(v_out).reshape(BH, cap, D)
    ref = {}
    for bh in sample:
        keep = keep_rows[bh // H]
        qn = oracle.qnorm(q_np[bh * G:(bh + 1) * G], G)
        m_o, v_o, s_o = oracle.prune(kv[bh:bh + 1, :keep], qn, T)
        rep = compare_masks(m_g_all[bh:bh + 1, :keep], m_o, kv[bh:bh + 1, :keep], qn, T)
        assert rep["mismatch"] == rep["near_tie"] and rep["mismatch"] <= 1e-4 * rep["tokens"], rep
        ok = np.all(m_g_all[bh, :keep] == m_o[0], axis=-1)
        assert np.array_equal(v_g_all[bh, :keep][ok].view(np.uint32), v_o[0][ok].view(np.uint32))
        np.testing.assert_allclose(st_g[bh, 1:], s_o[0, 1:], rtol=STATS_RTOL, atol=0)
        ref[bh] = (qn, m_o, v_o, s_o)
    capt = wl.tail_cap
    kt = torch.zeros((R, H, capt, D), dtype=k_out.dtype, device=DEV)
    vt = torch.zeros_like(kt)
    wsd = workspace(spark_workspace_bytes(SPARK_OP_DECODE, R, H, G, cap, D, T, capt))
    out = torch.empty((R, H * G, D), dtype=torch.float32, device=DEV)
    for step in range(steps):
        stp = make_decode_step(wl, step, DEV)
        spark_tail_append(stp["k_new"], stp["v_new"], kt, vt, R, H, D, capt, step)
        spark_decode_attn(stp["q"], kc, v_out, kt, vt, capt, step + 1, G, out, wsd)
    torch.cuda.synchronize()
    assert spark_device_status(wsd) == 0
    n_tail = steps
    q_last = to_np(make_decode_step(wl, steps - 1, DEV)["q"]).reshape(BH * G, D)
    for bh in sample:
        keep = keep_rows[bh // H]
        qn, m_o, v_o, s_o = ref[bh]
        o_ref = oracle.decode(q_last[bh * G:(bh + 1) * G], m_o, v_o, qn, s_o, vvals[bh:bh + 1, :keep],
                              to_np(kt).reshape(BH, capt, D)[bh:bh + 1], to_np(vt).reshape(BH, capt, D)[bh:bh + 1],
                              n_tail, G)
        assert_out_close(out.reshape(BH * G, D)[bh * G:(bh + 1) * G].cpu().numpy(), o_ref, f"row head {bh}")


def test_pyramid_rows_small():
    """Two layers x two batch rows, budgets 300 / 100 (beta 0.5 around 200),
    then pruning at lambda 0.5 and 5 decode steps."""
    wl = scaled(WORKLOADS["evict"], B=2, L=2, Hkv=2, S=600, keep=0, W=16, G=4, lam=0.5, seed=31)
    pre = make_prefill(wl, DEV)
    keep_rows = _row_budgets(wl, 200, 0.5)
    assert keep_rows == [300, 300, 100, 100]
    k_out, v_out, idx, kr, ws = _evict_rows(wl, pre, keep_rows)
    sample = list(range(wl.BH))
    _check_rows(wl, pre, keep_rows, k_out, v_out, idx, ws, sample)
    _prune_decode_rows(wl, pre, keep_rows, k_out, v_out, idx, sample, steps=5)


def test_pyramid_long_context_32_layers():
    """The long-context shape (32 layers x 8 kv heads, S = 131072, lambda
    0.8) with a PyramidKV budget of 2048 tokens per head on average (beta
    0.5: 3072 in the first layer down to 1024 in the last): one eviction over
    all 256 (layer, kv head) rows, then pruning and one decode step over
    rows of 32 different lengths; sampled heads against the oracle, every
    gather, length and pruned count checked."""
    wl = scaled(WORKLOADS["long"], keep=0)
    pre = make_prefill(wl, DEV)
    keep_rows = _row_budgets(wl, 2048, 0.5)
    assert keep_rows[0] == 3072 and keep_rows[-1] == 1024 and sum(keep_rows) == 2048 * wl.rows
    k_out, v_out, idx, kr, ws = _evict_rows(wl, pre, keep_rows)
    sample = [0, 101, 255]
    _check_rows(wl, pre, keep_rows, k_out, v_out, idx, ws, sample)
    _prune_decode_rows(wl, pre, keep_rows, k_out, v_out, idx, sample, steps=1)


def test_bad_row_budget_and_length_flagged():
    """A budget below the window evicts nothing for its row and raises
    SPARK_ERR_ARG in the status word; a length past S is clamped and flagged."""
    wl = scaled(WORKLOADS["evict"], B=1, L=2, Hkv=2, S=300, keep=0, W=16, G=4, seed=32)
    pre = make_prefill(wl, DEV)
    R, H, S, G, W = wl.rows, wl.Hkv, wl.S, wl.G, wl.W
    cap = 120
    k_out = torch.full((R, H, cap, D), 7.0, dtype=pre["k"].dtype, device=DEV)
    v_out = torch.full_like(k_out, 7.0)
    idx = torch.full((R, H, cap), -5, dtype=torch.int32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_SNAPKV, R, H, G, S, D, 0, 0))
    kr = torch.tensor([120, 8], dtype=torch.int32, device=DEV)  # row 1: below W = 16
    spark_snapkv_evict_rows(pre["k"], pre["v"], pre["q_obs"], G, W, kr, cap, wl.pool, k_out, v_out, idx, ws)
    assert spark_device_status(ws) == 1  # SPARK_ERR_ARG
    assert bool((idx[1] == -5).all()) and bool((k_out[1] == 7.0).all())
    assert bool((idx[0] >= 0).all())
    T = 64
    kc = KCache.empty(R, H, cap, D, T, k_out.dtype)
    kc.lens = torch.tensor([cap, cap + 5], dtype=torch.int32, device=DEV)
    wsp = workspace(spark_workspace_bytes(SPARK_OP_PRUNE, R, H, G, cap, D, T, 0))
    spark_prune(k_out, pre["q_obs"], G, W, kc, wsp)
    assert spark_device_status(wsp) == 1
    assert np.all(kc.stats.cpu().numpy().reshape(-1, 4)[:, 0] == cap * (D - T))
