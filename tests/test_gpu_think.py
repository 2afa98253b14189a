"""GPU parity of the ThinK comparator (spark_prune_think) against the
oracle's think_prune on the same seeded inputs: the shared head mask (a swap
is allowed only between channels whose fp64 scores tie to 1e-12), the kept
values bit for bit, the statistics, and decode over the ThinK cache within
the attention tolerance."""
import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (KCache, spark_prune_think, spark_workspace_bytes, workspace,
                                        SPARK_OP_THINK)
from channel_pruned_decode_b200.synth import WORKLOADS, make_decode_step, make_prefill, scaled
from tests._parity import assert_out_close, mask_np, to_np, unpack_vals
from tests.test_gpu_parity import _decode_gpu

pytestmark = pytest.mark.gpu
D = 128
DEV = "cuda"


def run_think(k, q_obs, G, W, T):
    R, Hkv, S, _ = k.shape
    kc = KCache.empty(R, Hkv, S, D, T, k.dtype, device=k.device)
    ws = workspace(spark_workspace_bytes(SPARK_OP_THINK, R, Hkv, G, S, D, T, 0))
    spark_prune_think(k, q_obs, G, W, kc, ws)
    torch.cuda.synchronize()
    return kc


def check_think(kc, k_np, q_np, G, T, what):
    BH, S = kc.B * kc.Hkv, kc.S
    qn = oracle.qnorm(q_np.reshape(BH * G, -1, D), G)
    k3 = k_np.reshape(BH, S, D)
    m_o, v_o, s_o = oracle.think_prune(k3, qn, T)
    s_g = kc.stats.cpu().numpy().reshape(BH, 4)
    assert np.array_equal(s_g, s_o), what
    if S == 0:
        return qn, m_o, v_o, s_o
    m_g = mask_np(kc)
    assert np.all(m_g == m_g[:, :1]), f"{what}: mask not shared by the tokens"
    for bh in range(BH):
        if np.array_equal(m_g[bh, 0], m_o[bh, 0]):
            continue
        score = qn[bh].astype(np.float64) * np.sqrt((k3[bh].astype(np.float64) ** 2).sum(0))
        bg = ((m_g[bh, 0][:, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(D).astype(bool)
        bo = ((m_o[bh, 0][:, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(D).astype(bool)
        a, b = score[bg & ~bo], score[bo & ~bg]
        assert np.allclose(np.sort(a), np.sort(b), rtol=1e-12, atol=0), f"{what}: non-tie channel swap"
    ok = np.all(m_g == m_o, axis=-1)
    assert np.array_equal(unpack_vals(kc)[ok].view(np.uint32), v_o[ok].view(np.uint32)), what
    return qn, m_o, v_o, s_o


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("S,T,G", [(1, 26, 4), (33, 64, 4), (1000, 26, 2), (257, 0, 4), (300, 128, 1),
                                   (2049, 90, 8), (0, 26, 4)])
def test_think_parity_and_decode(dtype, S, T, G):
    wl = scaled(WORKLOADS["tiny"], S=S, G=G, Hkv=3, dtype="f32" if dtype == torch.float32 else "bf16",
                seed=300 + S + T)
    pre = make_prefill(wl, DEV)
    kc = run_think(pre["k"], pre["q_obs"], G, wl.W, T)
    qn, m, vals, st = check_think(kc, to_np(pre["k"]), to_np(pre["q_obs"]), G, T, f"think S={S} T={T}")
    BH = wl.rows * wl.Hkv
    q = make_decode_step(wl, 1, DEV)["q"]
    out = _decode_gpu(q, kc, pre["v"], None, None, 0, 0, G)
    o_ref = oracle.decode(to_np(q).reshape(BH * G, D), m, vals, qn, st, to_np(pre["v"]).reshape(BH, S, D), G=G)
    assert_out_close(out.cpu().numpy().reshape(BH * G, D), o_ref, f"think decode S={S} T={T}")


def test_think_llama_layer():
    wl = WORKLOADS["llama1l"]
    pre = make_prefill(wl, DEV)
    kc = run_think(pre["k"], pre["q_obs"], wl.G, wl.W, 26)
    check_think(kc, to_np(pre["k"]), to_np(pre["q_obs"]), wl.G, 26, "think llama layer")
