"""GPU parity of SparK-g grouped pruning (spark_prune_grouped) against the
oracle's prune_grouped on the same seeded inputs: masks and kept values bit
for bit (near-ties inside a group are counted and must stay under 0.01 %),
statistics to fp32-partial rounding, and decode over the grouped cache within
the attention tolerance."""
import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (KCache, spark_device_status, spark_group_budget, spark_prune_grouped,
                                        spark_workspace_bytes, workspace, SPARK_OP_PRUNE)
from channel_pruned_decode_b200.synth import WORKLOADS, make_decode_step, make_prefill, scaled
from tests._parity import assert_out_close, mask_np, to_np, unpack_vals
from tests.test_gpu_parity import STATS_RTOL, _decode_gpu

pytestmark = pytest.mark.gpu
D = 128
DEV = "cuda"
RATES = {1: [0.5], 2: [0.25, 0.75], 4: [0.25, 0.5, 0.75, 1.0], 5: [0.1, 0.3, 0.5, 0.7, 0.9],
         8: [0.0, 0.125, 0.25, 0.5, 0.5, 0.75, 0.875, 1.0]}


def run_grouped(k, q_obs, G, W, Tg):
    R, Hkv, S, _ = k.shape
    kc = KCache.empty(R, Hkv, S, D, sum(Tg), k.dtype, device=k.device)
    ws = workspace(spark_workspace_bytes(SPARK_OP_PRUNE, R, Hkv, G, S, D, sum(Tg), 0))
    spark_prune_grouped(k, q_obs, G, W, Tg, kc, ws)
    torch.cuda.synchronize()
    return kc


def _near_tie(w, gid, Tg, bits_g, bits_o):
    """A mismatching token is a near-tie when, in a group whose kept sets
    differ, the Tq-th and (Tq+1)-th saliencies are within 1e-6 relative."""
    for q, Tq in enumerate(Tg):
        sel = gid == q
        if np.array_equal(bits_g[sel], bits_o[sel]):
            continue
        srt = np.sort(w[sel])[::-1]
        if not (0 < Tq < sel.sum()):
            return False
        a, b = float(srt[Tq - 1]), float(srt[Tq])
        if not (a == 0 or abs(a - b) <= 1e-6 * abs(a)):
            return False
    return True


def check_grouped(kc, k_np, q_np, G, Tg, what):
    BH, S = kc.B * kc.Hkv, kc.S
    qn = oracle.qnorm(q_np.reshape(BH * G, -1, D), G)
    assert np.array_equal(kc.qn.cpu().numpy().reshape(BH, D).view(np.uint32), qn.view(np.uint32))
    k3 = k_np.reshape(BH, S, D)
    m_o, v_o, s_o = oracle.prune_grouped(k3, qn, Tg)
    m_g = mask_np(kc)
    gid = oracle.group_of_channel(qn, len(Tg))
    diff = np.argwhere(np.any(m_g != m_o, axis=-1))
    for bh, t in diff:
        w = (qn[bh] * np.abs(k3[bh, t])).astype(np.float32)
        bg = ((m_g[bh, t][:, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(D)
        bo = ((m_o[bh, t][:, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(D)
        assert _near_tie(w, gid[bh], Tg, bg, bo), f"{what}: non-tie mismatch at {(bh, t)}"
    assert len(diff) <= max(1e-4 * BH * S, 1), f"{what}: {len(diff)} near-tie mismatches"
    ok = np.all(m_g == m_o, axis=-1)
    v_g = unpack_vals(kc)
    assert np.array_equal(v_g[ok].view(np.uint32), v_o[ok].view(np.uint32)), f"{what}: values differ"
    s_g = kc.stats.cpu().numpy().reshape(BH, 4)
    assert np.array_equal(s_g[:, 0], s_o[:, 0]), f"{what}: N_pruned"
    np.testing.assert_allclose(s_g[:, 1:], s_o[:, 1:], rtol=STATS_RTOL, atol=0, err_msg=what)
    return qn, m_o, v_o, s_o


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("S,g", [(1, 4), (33, 4), (1000, 5), (2049, 8), (300, 1), (777, 2), (0, 4)])
def test_grouped_parity_and_decode(dtype, S, g):
    wl = scaled(WORKLOADS["tiny"], S=S, dtype="f32" if dtype == torch.float32 else "bf16", Hkv=3,
                seed=31 + S + g)
    pre = make_prefill(wl, DEV)
    Tg = spark_group_budget(D, RATES[g])
    assert Tg == oracle.group_budget(D, RATES[g])
    kc = run_grouped(pre["k"], pre["q_obs"], wl.G, wl.W, Tg)
    qn, m, vals, st = check_grouped(kc, to_np(pre["k"]), to_np(pre["q_obs"]), wl.G, Tg, f"S={S} g={g}")
    BH = wl.rows * wl.Hkv
    q = make_decode_step(wl, 5, DEV)["q"]
    out = _decode_gpu(q, kc, pre["v"], None, None, 0, 0, wl.G)
    o_ref = oracle.decode(to_np(q).reshape(BH * wl.G, D), m, vals, qn, st,
                          to_np(pre["v"]).reshape(BH, S, D), G=wl.G)
    assert_out_close(out.cpu().numpy().reshape(BH * wl.G, D), o_ref, f"grouped decode S={S} g={g}")


@pytest.mark.parametrize("k_exp,spread", [(-30, 0), (20, 0), (0, 30)])
def test_grouped_extremes(k_exp, spread):
    g = torch.Generator(device=DEV).manual_seed(7 + k_exp + spread)
    R, Hkv, G, W, S = 1, 2, 4, 16, 400
    ch = torch.randint(-spread, spread + 1, (D,), generator=g, device=DEV).float() if spread else \
        torch.zeros(D, device=DEV)
    k = (torch.randn((R, Hkv, S, D), generator=g, device=DEV) * torch.exp2(ch + k_exp)).to(torch.bfloat16)
    q_obs = torch.randn((R, Hkv * G, W, D), generator=g, device=DEV).to(torch.bfloat16)
    for rates in (RATES[4], RATES[8]):
        Tg = spark_group_budget(D, rates)
        kc = run_grouped(k, q_obs, G, W, Tg)
        check_grouped(kc, to_np(k), to_np(q_obs), G, Tg, f"extremes k2^{k_exp} spread {spread} g={len(Tg)}")


@pytest.mark.parametrize("rates", [[0.0, 0.03, 0.97, 1.0], [0.5, 0.5, 0.5, 0.5], [0.97, 0.97, 0.97, 0.97],
                                   [0.03, 0.1, 0.2, 0.3], [1.0, 1.0, 1.0, 0.0], [0.0, 0.0, 0.0, 0.0]])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_grouped_four_groups_budgets(rates, dtype):
    # four groups of 32 channels (one per lane of a quad): budgets from 0 to
    # 32 per group, over several 32-token groups and a ragged tail
    wl = scaled(WORKLOADS["tiny"], S=2083, dtype="f32" if dtype == torch.float32 else "bf16", Hkv=2,
                seed=int(sum(rates) * 100))
    pre = make_prefill(wl, DEV)
    Tg = spark_group_budget(D, rates)
    kc = run_grouped(pre["k"], pre["q_obs"], wl.G, wl.W, Tg)
    check_grouped(kc, to_np(pre["k"]), to_np(pre["q_obs"]), wl.G, Tg, f"four groups {Tg}")


@pytest.mark.parametrize("g", [4, 2])
def test_grouped_row_lengths(g):
    # per-row prompt lengths (spark_kcache.lens): each row's own tokens are
    # pruned as if the row were that long, and nothing past it is written
    wl = scaled(WORKLOADS["tiny"], B=3, S=700, Hkv=2, dtype="bf16", seed=71 + g)
    pre = make_prefill(wl, DEV)
    R, Hkv, S = wl.rows, wl.Hkv, wl.S
    lens = [700, 333, 1]
    Tg = spark_group_budget(D, RATES[g])
    kc = KCache.empty(R, Hkv, S, D, sum(Tg), pre["k"].dtype, device=DEV)
    kc.mask.fill_(0x55555555)
    kc.lens = torch.tensor(lens, dtype=torch.int32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_PRUNE, R, Hkv, wl.G, S, D, sum(Tg), 0))
    spark_prune_grouped(pre["k"], pre["q_obs"], wl.G, wl.W, Tg, kc, ws)
    torch.cuda.synchronize()
    assert spark_device_status(ws) == 0
    m_g, v_g = mask_np(kc), unpack_vals(kc)
    s_g = kc.stats.cpu().numpy().reshape(R * Hkv, 4)
    k3 = to_np(pre["k"]).reshape(R * Hkv, S, D)
    q3 = to_np(pre["q_obs"]).reshape(R * Hkv * wl.G, wl.W, D)
    qn_all = oracle.qnorm(q3, wl.G)
    for bh in range(R * Hkv):
        n = lens[bh // Hkv]
        qn = qn_all[bh:bh + 1]
        m_o, v_o, s_o = oracle.prune_grouped(k3[bh:bh + 1, :n], qn, Tg)
        gid = oracle.group_of_channel(qn, len(Tg))[0]
        for t in np.argwhere(np.any(m_g[bh, :n] != m_o[0], axis=-1)).ravel():
            w = (qn[0] * np.abs(k3[bh, t])).astype(np.float32)
            bg = ((m_g[bh, t][:, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(D)
            bo = ((m_o[0, t][:, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(D)
            assert _near_tie(w, gid, Tg, bg, bo), f"row head {bh}: non-tie mismatch at token {t}"
        ok = np.all(m_g[bh, :n] == m_o[0], axis=-1)
        assert np.array_equal(v_g[bh, :n][ok].view(np.uint32), v_o[0][ok].view(np.uint32))
        assert s_g[bh, 0] == s_o[0, 0] == n * (D - sum(Tg))
        np.testing.assert_allclose(s_g[bh, 1:], s_o[0, 1:], rtol=STATS_RTOL, atol=0)
        assert np.all(m_g[bh, n:] == 0x55555555), f"row head {bh}: mask written past the row's length"


def test_grouped_ties_integer_keys():
    # integer keys and window queries: exact saliency ties everywhere, and
    # equal window-query norms across group boundaries
    g = torch.Generator(device=DEV).manual_seed(12)
    R, Hkv, G, W, S = 1, 2, 4, 8, 500
    k = torch.randint(-3, 4, (R, Hkv, S, D), generator=g, device=DEV).to(torch.bfloat16)
    q_obs = torch.randint(-1, 2, (R, Hkv * G, W, D), generator=g, device=DEV).to(torch.bfloat16)
    for rates in (RATES[2], RATES[4], RATES[5]):
        Tg = spark_group_budget(D, rates)
        kc = run_grouped(k, q_obs, G, W, Tg)
        check_grouped(kc, to_np(k), to_np(q_obs), G, Tg, f"ties g={len(Tg)}")


def test_grouped_llama_layer_sampled_heads():
    # Llama-3.1-8B layer shape (8 kv heads, S=32768, bf16) with the pages'
    # g = 4 rates; the oracle checks two whole heads
    wl = WORKLOADS["llama1l"]
    pre = make_prefill(wl, DEV)
    Tg = spark_group_budget(D, RATES[4])
    kc = run_grouped(pre["k"], pre["q_obs"], wl.G, wl.W, Tg)
    sel = [0, 5]
    k_np = to_np(pre["k"].reshape(wl.BH, wl.S, D)[sel])
    q_np = to_np(pre["q_obs"].reshape(wl.BH, wl.G, wl.W, D)[sel])
    qn = oracle.qnorm(q_np.reshape(-1, wl.W, D), wl.G)
    m_o, v_o, s_o = oracle.prune_grouped(k_np, qn, Tg)
    m_g = mask_np(kc)[sel]
    bad = np.any(m_g != m_o, axis=-1)
    assert bad.sum() <= 1e-4 * bad.size, int(bad.sum())
    v_g = unpack_vals(kc)[sel]
    ok = ~bad
    assert np.array_equal(v_g[ok].view(np.uint32), v_o[ok].view(np.uint32))
    s_g = kc.stats.cpu().numpy().reshape(wl.BH, 4)[sel]
    np.testing.assert_allclose(s_g[:, 1:], s_o[:, 1:], rtol=STATS_RTOL, atol=0)
    assert spark_device_status(workspace(256)) == 0
