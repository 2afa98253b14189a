"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Masks, kept values and window norms are compared bit for
bit (near-tie mismatches are counted and must stay under 0.01 %); statistics
to fp64/fp32-partial rounding; attention outputs within max-abs 2e-3 and
relative 1e-2."""
import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (KCache, SparkError, spark_decode_attn, spark_device_status,
                                        spark_lambda_to_T, spark_prune, spark_tail_append,
                                        spark_workspace_bytes, workspace, SPARK_OP_DECODE,
                                        SPARK_OP_PRUNE)
from channel_pruned_decode_b200.synth import WORKLOADS, make_decode_step, make_prefill, scaled
from tests._parity import (assert_out_close, compare_masks, mask_np, run_prune, to_np,
                           unpack_vals)

pytestmark = pytest.mark.gpu

D = 128
DEV = "cuda"
STATS_RTOL = 2e-6   # fp32 per-lane partials summed in fp64 vs a plain fp64 sum


def _oracle_prefill(k_np, q_np, G, T):
    qn = oracle.qnorm(q_np, G)
    m, v, s = oracle.prune(k_np, qn, T)
    return qn, m, v, s


def _check_prune(kc, k_np, q_np, G, T, what):
    BH, S = kc.B * kc.Hkv, kc.S
    qn_o, m_o, v_o, s_o = _oracle_prefill(k_np.reshape(BH, S, D), q_np.reshape(BH * G, -1, D), G, T)
    qn_g = kc.qn.cpu().numpy().reshape(BH, D)
    assert np.array_equal(qn_g.view(np.uint32), qn_o.view(np.uint32)), f"{what}: qn not bit-exact"
    m_g = mask_np(kc)
    rep = compare_masks(m_g, m_o, k_np.reshape(BH, S, D), qn_o, T)
    assert rep["mismatch"] == rep["near_tie"], f"{what}: non-tie mask mismatches {rep}"
    assert rep["mismatch"] <= 1e-4 * max(rep["tokens"], 1), f"{what}: {rep}"
    ok = np.all(m_g == m_o, axis=-1)
    v_g = unpack_vals(kc)
    assert np.array_equal(v_g[ok].view(np.uint32), v_o[ok].view(np.uint32)), f"{what}: vals differ"
    s_g = kc.stats.cpu().numpy().reshape(BH, 4)
    assert np.array_equal(s_g[:, 0], s_o[:, 0]), f"{what}: N_pruned"
    np.testing.assert_allclose(s_g[:, 1:], s_o[:, 1:], rtol=STATS_RTOL, atol=0, err_msg=what)
    return qn_o, m_o, v_o, s_o


def _decode_gpu(q, kc, v, kt, vt, cap, n_tail, G):
    R, Hq, _ = q.shape
    out = torch.empty((R, Hq, D), dtype=torch.float32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, kc.B, kc.Hkv, G, kc.S, D, kc.T, cap))
    spark_decode_attn(q, kc, v, kt, vt, cap, n_tail, G, out, ws)
    torch.cuda.synchronize()
    assert spark_device_status(ws) == 0
    return out


# ------------------------------------------------------------ tiny (fp32)
def test_tiny_full_parity():
    wl = WORKLOADS["tiny"]
    T = spark_lambda_to_T(wl.lam)
    assert T == 64
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, T)
    torch.cuda.synchronize()
    k_np, q_np, v_np = to_np(pre["k"]), to_np(pre["q_obs"]), to_np(pre["v"])
    qn, m, vals, st = _check_prune(kc, k_np, q_np, wl.G, T, "tiny")
    step = make_decode_step(wl, 0, DEV)
    cap = wl.tail_cap
    kt = torch.zeros((wl.rows, wl.Hkv, cap, D), dtype=wl.torch_dtype, device=DEV)
    vt = torch.zeros_like(kt)
    spark_tail_append(step["k_new"], step["v_new"], kt, vt, wl.rows, wl.Hkv, D, cap, 0)
    out = _decode_gpu(step["q"], kc, pre["v"], kt, vt, cap, 1, wl.G)
    BH = wl.rows * wl.Hkv
    o_ref = oracle.decode(to_np(step["q"]).reshape(BH * wl.G, D), m, vals, qn, st,
                          v_np.reshape(BH, -1, D), to_np(kt).reshape(BH, cap, D),
                          to_np(vt).reshape(BH, cap, D), 1, wl.G)
    assert_out_close(out.cpu().numpy().reshape(BH * wl.G, D), o_ref, "tiny decode")


# --------------------------------------------- edge shapes, small, fp32 + bf16
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("S,T,G,n_tail", [
    (1, 26, 4, 0), (33, 26, 4, 3), (1000, 64, 4, 0), (257, 0, 4, 2), (300, 128, 4, 0),
    (777, 1, 2, 5), (640, 127, 1, 0), (129, 90, 8, 64), (0, 26, 4, 7), (2049, 26, 4, 256),
])
def test_edge_shapes(dtype, S, T, G, n_tail):
    wl = scaled(WORKLOADS["tiny"], S=S, G=G, dtype="f32" if dtype == torch.float32 else "bf16",
                Hkv=3, seed=17 + S + T)
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], G, wl.W, T)
    torch.cuda.synchronize()
    BH = wl.rows * wl.Hkv
    k_np, q_np, v_np = to_np(pre["k"]), to_np(pre["q_obs"]), to_np(pre["v"])
    qn, m, vals, st = _check_prune(kc, k_np, q_np, G, T, f"edge S={S} T={T}")
    cap = max(n_tail, 8)
    kt = torch.zeros((wl.rows, wl.Hkv, cap, D), dtype=dtype, device=DEV)
    vt = torch.zeros_like(kt)
    for i in range(n_tail):
        stp = make_decode_step(wl, i, DEV)
        spark_tail_append(stp["k_new"], stp["v_new"], kt, vt, wl.rows, wl.Hkv, D, cap, i)
    q = make_decode_step(wl, 99, DEV)["q"]
    out = _decode_gpu(q, kc, pre["v"], kt, vt, cap, n_tail, G)
    o_ref = oracle.decode(to_np(q).reshape(BH * G, D), m, vals, qn, st, v_np.reshape(BH, S, D),
                          to_np(kt).reshape(BH, cap, D), to_np(vt).reshape(BH, cap, D), n_tail, G)
    assert_out_close(out.cpu().numpy().reshape(BH * G, D), o_ref, f"edge S={S} T={T} G={G}")


def test_ties_and_zero_norm_channels():
    # integer-valued keys (many exact saliency ties) and window queries that
    # are zero on some channels (qn_j = 0: saliency 0, recovered key 0)
    g = torch.Generator(device=DEV).manual_seed(5)
    R, Hkv, G, W, S = 1, 2, 4, 8, 700
    k = torch.randint(-3, 4, (R, Hkv, S, D), generator=g, device=DEV).to(torch.bfloat16)
    v = torch.randn((R, Hkv, S, D), generator=g, device=DEV).to(torch.bfloat16)
    q_obs = torch.randint(-2, 3, (R, Hkv * G, W, D), generator=g, device=DEV).to(torch.bfloat16)
    q_obs[..., ::7] = 0
    for T in (26, 64, 100):
        kc = run_prune(k, q_obs, G, W, T)
        torch.cuda.synchronize()
        qn, m, vals, st = _check_prune(kc, to_np(k), to_np(q_obs), G, T, f"ties T={T}")
        q = torch.randn((R, Hkv * G, D), generator=g, device=DEV).to(torch.bfloat16)
        out = _decode_gpu(q, kc, v, None, None, 0, 0, G)
        o_ref = oracle.decode(to_np(q).reshape(-1, D), m, vals, qn, st, to_np(v).reshape(R * Hkv, S, D),
                              G=G)
        assert_out_close(out.cpu().numpy().reshape(-1, D), o_ref, f"ties T={T}")


@pytest.mark.parametrize("k_exp,q_exp,spread", [(-30, 0, 0), (-12, 0, 0), (20, 0, 0), (40, 0, 0),
                                                 (0, -40, 0), (0, 30, 0), (0, 0, 30), (-20, 10, 12)])
def test_key_magnitude_extremes(k_exp, q_exp, spread):
    # keys and window queries scaled by powers of two (and, with `spread`, a
    # random per-channel exponent in [-spread, spread]): saliencies far below,
    # inside and far above the 16-bit search keys' normal range, which pushes
    # the selection into its underflow, overflow and exact-tie paths
    g = torch.Generator(device=DEV).manual_seed(100 + k_exp + 3 * q_exp + spread)
    R, Hkv, G, W, S = 1, 2, 4, 16, 520
    ch = torch.randint(-spread, spread + 1, (D,), generator=g, device=DEV).float() if spread else \
        torch.zeros(D, device=DEV)
    k = (torch.randn((R, Hkv, S, D), generator=g, device=DEV) * torch.exp2(ch + k_exp)).to(torch.bfloat16)
    q_obs = (torch.randn((R, Hkv * G, W, D), generator=g, device=DEV) * 2.0 ** q_exp).to(torch.bfloat16)
    for T in (1, 26, 64, 127):
        kc = run_prune(k, q_obs, G, W, T)
        torch.cuda.synchronize()
        _check_prune(kc, to_np(k), to_np(q_obs), G, T, f"extremes k2^{k_exp} q2^{q_exp} spread {spread} T={T}")


def test_lambda0_matches_dense_sdpa():
    # T = D keeps every channel: the GPU decode must equal plain attention
    wl = scaled(WORKLOADS["llama1l"], S=3000, Hkv=2, seed=9)
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, D)
    q = make_decode_step(wl, 0, DEV)["q"]
    out = _decode_gpu(q, kc, pre["v"], None, None, 0, 0, wl.G)
    kk = pre["k"].float().repeat_interleave(wl.G, dim=1)
    vv = pre["v"].float().repeat_interleave(wl.G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q.float()[:, :, None], kk, vv)[:, :, 0]
    assert_out_close(out.cpu().numpy(), ref.cpu().numpy(), "lambda=0 vs sdpa")


def test_deterministic_reruns():
    wl = scaled(WORKLOADS["llama1l"], S=5000, Hkv=4, seed=3)
    pre = make_prefill(wl, DEV)
    T = spark_lambda_to_T(0.8)
    outs = []
    for _ in range(2):
        kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, T)
        q = make_decode_step(wl, 0, DEV)["q"]
        out = _decode_gpu(q, kc, pre["v"], None, None, 0, 0, wl.G)
        outs.append((kc.mask.clone(), kc.vals.clone(), kc.stats.clone(), out))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


def test_runtime_argument_errors():
    kc = KCache.empty(1, 2, 64, D, 32, torch.bfloat16, device=DEV)
    k = torch.zeros((1, 2, 64, D), dtype=torch.bfloat16, device=DEV)
    q_obs = torch.zeros((1, 8, 4, D), dtype=torch.bfloat16, device=DEV)
    small = workspace(4096)
    with pytest.raises(SparkError):
        spark_prune(k, q_obs, 4, 4, kc, workspace(16)[:8], None)
    with pytest.raises(SparkError):
        spark_prune(k[..., 1:], q_obs, 4, 4, kc, small, None)  # misaligned key pointer


# ------------------------------------------------- pages' workload shapes
def _multi_step(wl, check_steps, sample_bh=None):
    """Prune once, then `wl.steps` decode steps appending unpruned keys; the
    oracle checks the listed steps (on all or a sample of (row, kv head))."""
    T = spark_lambda_to_T(wl.lam)
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, T)
    torch.cuda.synchronize()
    BH, S, G = wl.BH, wl.S, wl.G
    sel_np = np.arange(BH) if sample_bh is None else np.asarray(sample_bh)
    sel = torch.as_tensor(sel_np, device=DEV)
    kv = pre["k"].reshape(BH, S, D)
    qv = pre["q_obs"].reshape(BH * G, wl.W, D)
    sub = KCache(1, len(sel_np), S, D, T, kc.dtype, kc.mask.reshape(BH, S, 4)[sel][None],
                 kc.vals.reshape(BH, -1)[sel][None], kc.qn.reshape(BH, D)[sel][None],
                 kc.stats.reshape(BH, 4)[sel][None])
    qsel = torch.as_tensor(np.concatenate([np.arange(b * G, (b + 1) * G) for b in sel_np]), device=DEV)
    qn, m, vals, st = _check_prune(sub, to_np(kv[sel]), to_np(qv[qsel]), G, T, wl.name)
    # every token of every head keeps exactly T channels
    mk = kc.mask.view(torch.int32)
    pc = sum(torch.bitwise_and(torch.bitwise_right_shift(mk, b), 1).sum(-1) for b in range(32))
    assert int(pc.min()) == T and int(pc.max()) == T

    cap = wl.tail_cap
    kt = torch.zeros((wl.rows, wl.Hkv, cap, D), dtype=wl.torch_dtype, device=DEV)
    vt = torch.zeros_like(kt)
    ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, wl.rows, wl.Hkv, G, S, D, T, cap))
    out = torch.empty((wl.rows, wl.Hq, D), dtype=torch.float32, device=DEV)
    v_np = to_np(pre["v"].reshape(BH, S, D)[sel])
    for step in range(wl.steps):
        stp = make_decode_step(wl, step, DEV)
        spark_tail_append(stp["k_new"], stp["v_new"], kt, vt, wl.rows, wl.Hkv, D, cap, step)
        spark_decode_attn(stp["q"], kc, pre["v"], kt, vt, cap, step + 1, G, out, ws)
        if step in check_steps:
            torch.cuda.synchronize()
            o_ref = oracle.decode(to_np(stp["q"].reshape(BH * G, D)[qsel]), m, vals, qn, st, v_np,
                                  to_np(kt.reshape(BH, cap, D)[sel]), to_np(vt.reshape(BH, cap, D)[sel]),
                                  step + 1, G)
            got = out.reshape(BH * G, D)[qsel].cpu().numpy()
            assert_out_close(got, o_ref, f"{wl.name} step {step}")
    torch.cuda.synchronize()
    assert spark_device_status(ws) == 0
    return kc, pre, T


def _check_all_heads(kc, pre, wl, T, threads=None):
    """The oracle's prune of every (row, kv head), one head at a time on a
    thread pool (the oracle's C calls release the GIL): window norms bit for
    bit, masks bit-exact outside counted near-ties, kept values bit-exact,
    N exact and the pruned-saliency sums within STATS_RTOL."""
    import concurrent.futures as cf
    import os

    BH, S, G = wl.BH, wl.S, wl.G
    qn_all = oracle.qnorm(to_np(pre["q_obs"]).reshape(BH * G, wl.W, D), G)
    assert np.array_equal(kc.qn.cpu().numpy().reshape(BH, D).view(np.uint32), qn_all.view(np.uint32))
    st_g = kc.stats.cpu().numpy().reshape(BH, 4)
    assert np.all(st_g[:, 0] == float(S) * (D - T))
    kv, mk = pre["k"].reshape(BH, S, D), kc.mask.reshape(BH, S, 4)

    def one(h):
        k_np = kv[h:h + 1].float().cpu().numpy()
        m_o, v_o, s_o = oracle.prune(k_np, qn_all[h:h + 1], T)
        m_g = mk[h:h + 1].cpu().numpy().view(np.uint32)
        rep = compare_masks(m_g, m_o, k_np, qn_all[h:h + 1], T)
        sub = KCache(1, 1, S, D, T, kc.dtype, kc.mask.reshape(BH, S, 4)[h][None], kc.vals.reshape(BH, -1)[h][None],
                     kc.qn.reshape(BH, D)[h][None], kc.stats.reshape(BH, 4)[h][None])
        ok = np.all(m_g == m_o, axis=-1)
        v_bad = int((~np.all(unpack_vals(sub)[ok] == v_o[ok], axis=-1)).sum())
        rel = np.abs(st_g[h, 1:3] - s_o[0, 1:3]) / np.maximum(np.abs(s_o[0, 1:3]), 1e-300)
        return rep, v_bad, float(rel.max())

    with cf.ThreadPoolExecutor(max_workers=threads or min(16, os.cpu_count() or 1)) as ex:
        res = list(ex.map(one, range(BH)))
    tokens = sum(r[0]["tokens"] for r in res)
    mism = sum(r[0]["mismatch"] for r in res)
    near = sum(r[0]["near_tie"] for r in res)
    assert mism == near and mism <= 1e-4 * tokens, (mism, near, tokens)
    assert sum(r[1] for r in res) == 0
    worst = max(r[2] for r in res)
    assert worst <= STATS_RTOL, worst


def test_llama_single_layer_64_steps():
    _multi_step(WORKLOADS["llama1l"], check_steps={0, 1, 31, 63})


@pytest.mark.parametrize("name", ["lsweep_0.3", "lsweep_0.5", "lsweep_0.8"])
def test_lambda_sweep_128_steps(name):
    wl = WORKLOADS[name]
    _multi_step(wl, check_steps={0, 127}, sample_bh=[0, 9, 27, 63])


def test_long_context_32_layers():
    # full-size prune + one decode step over all 32 layers; the decode output is
    # checked on a sample of (layer, kv head) pairs, the prune on all of them
    wl = WORKLOADS["long"]
    kc, pre, T = _multi_step(wl, check_steps={0}, sample_bh=[0, 37, 130, 255])
    # the prune of every one of the 256 (layer, kv head) pairs against the
    # oracle: qn bits, masks, kept values and statistics
    _check_all_heads(kc, pre, wl, T)


# ------------------------------------------ sampling recoveries (F table)
@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("dtype,S,T,G,n_tail", [(torch.bfloat16, 1000, 26, 4, 3), (torch.float32, 257, 64, 2, 0),
                                                (torch.bfloat16, 64, 0, 4, 1), (torch.bfloat16, 300, 127, 8, 0)])
def test_sampling_recovery_parity(mode, dtype, S, T, G, n_tail):
    wl = scaled(WORKLOADS["tiny"], S=S, G=G, dtype="f32" if dtype == torch.float32 else "bf16", Hkv=3,
                seed=101 + S + T + mode)
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], G, wl.W, T)
    torch.cuda.synchronize()
    BH = wl.rows * wl.Hkv
    qn, m, vals, st = _check_prune(kc, to_np(pre["k"]), to_np(pre["q_obs"]), G, T, "sampling")
    cap = max(n_tail, 4)
    kt = torch.zeros((wl.rows, wl.Hkv, cap, D), dtype=dtype, device=DEV)
    vt = torch.zeros_like(kt)
    for i in range(n_tail):
        stp = make_decode_step(wl, i, DEV)
        spark_tail_append(stp["k_new"], stp["v_new"], kt, vt, wl.rows, wl.Hkv, D, cap, i)
    q = make_decode_step(wl, 7, DEV)["q"]
    seed = 0x1234_5678_9ABC
    out = torch.empty((wl.rows, wl.Hq, D), dtype=torch.float32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, wl.rows, wl.Hkv, G, S, D, T, cap))
    spark_decode_attn(q, kc, pre["v"], kt, vt, cap, n_tail, G, out, ws, recovery=mode, seed=seed)
    torch.cuda.synchronize()
    assert spark_device_status(ws) == 0
    o_ref = oracle.decode_f(to_np(q).reshape(BH * G, D), m, vals, qn, st, to_np(pre["v"]).reshape(BH, S, D),
                            to_np(kt).reshape(BH, cap, D), to_np(vt).reshape(BH, cap, D), n_tail, G,
                            mode=mode, seed=seed)
    assert_out_close(out.cpu().numpy().reshape(BH * G, D), o_ref, f"F={mode} S={S} T={T}")
    # the draw depends on the seed: another seed changes the output
    out2 = torch.empty_like(out)
    spark_decode_attn(q, kc, pre["v"], kt, vt, cap, n_tail, G, out2, ws, recovery=mode, seed=seed + 1)
    torch.cuda.synchronize()
    if T < D:
        assert not torch.equal(out, out2)


@pytest.mark.parametrize("mode", [1, 2])
def test_sampling_recovery_llama_layer(mode):
    wl = scaled(WORKLOADS["llama1l"], S=8192)
    T = spark_lambda_to_T(wl.lam)
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, T)
    BH, S, G = wl.BH, wl.S, wl.G
    q = make_decode_step(wl, 0, DEV)["q"]
    out = torch.empty((wl.rows, wl.Hq, D), dtype=torch.float32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, wl.rows, wl.Hkv, G, S, D, T, 0))
    spark_decode_attn(q, kc, pre["v"], None, None, 0, 0, G, out, ws, recovery=mode, seed=42)
    torch.cuda.synchronize()
    qn = oracle.qnorm(to_np(pre["q_obs"]).reshape(BH * G, -1, D), G)
    m, vals, st = oracle.prune(to_np(pre["k"]).reshape(BH, S, D), qn, T)
    o_ref = oracle.decode_f(to_np(q).reshape(BH * G, D), m, vals, qn, st, to_np(pre["v"]).reshape(BH, S, D),
                            G=G, mode=mode, seed=42)
    assert_out_close(out.cpu().numpy().reshape(BH * G, D), o_ref, f"llama layer F={mode}")
