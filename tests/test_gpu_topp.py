"""GPU parity of SparK-p (spark_prune_topp / spark_decode_attn_topp) against
the oracle's prune_topp on the same seeded inputs.  The oracle sums the
cumulative saliency in fp64 (reading R19); the GPU may decide a token's
boundary in other arithmetic, so a token's kept set may differ from the
oracle's only at a counted near-tie: the GPU's set is still a greedy prefix
and the exact cumulative saliency at the differing boundary lies within fp32
rounding of the target (2^-23 * D * total).  Such tokens must stay under
0.01 %.  Kept values (zero padding included) are compared bit for bit on
every other token, the pruned count and saliency sums through the
statistics, and decode within the attention tolerance.  Full-size heads are
checked on sampled tokens."""
import numpy as np
import pytest
import torch

import oracle
from channel_pruned_decode_b200 import (KCache, spark_decode_attn, spark_decode_attn_topp, spark_device_status,
                                        spark_prune_topp, spark_topp_vals_used, spark_workspace_bytes, workspace,
                                        SPARK_F_GAUSSIAN, SPARK_OP_DECODE, SPARK_OP_TOPP)
from channel_pruned_decode_b200.synth import WORKLOADS, make_decode_step, make_prefill, scaled
from tests._parity import assert_out_close, mask_np, run_prune, to_np
from tests.test_gpu_parity import STATS_RTOL

pytestmark = pytest.mark.gpu
D = 128
DEV = "cuda"


def run_topp(k, q_obs, G, W, p, Tcap):
    R, Hkv, S, _ = k.shape
    kc = KCache.empty_topp(R, Hkv, S, D, Tcap, k.dtype, device=k.device)
    ws = workspace(spark_workspace_bytes(SPARK_OP_TOPP, R, Hkv, G, S, D, Tcap, 0))
    spark_prune_topp(k, q_obs, G, W, p, kc, ws)
    torch.cuda.synchronize()
    assert spark_device_status(ws) == 0
    return kc


def unpack_topp(kc):
    """The compact SparK-p value stream (group offsets in 32-element rows) as
    [B*Hkv, S, Tcap] fp32, zero past each token's kept values; also checks
    the layout: each group's slot count is its longest kept set, unused
    slots hold 0, and the last offset is the number of rows used."""
    BH, S, Tcap = kc.B * kc.Hkv, kc.S, kc.T
    ng = (S + 31) // 32
    goff = kc.goff.cpu().numpy().view(np.uint32).astype(np.int64)
    assert goff.shape == (BH * ng + 1,) and goff[0] == 0 and np.all(np.diff(goff) >= 0)
    vals = kc.vals.reshape(-1)[: int(goff[-1]) * 32].float().cpu().numpy()
    m = mask_np(kc)
    cnt = np.zeros((BH, ng * 32), np.int64)
    if S:
        cnt[:, :S] = np.unpackbits(np.ascontiguousarray(m).view(np.uint8), axis=-1).sum(-1)
    out = np.zeros((BH, ng * 32, Tcap), np.float32)
    for i in range(BH * ng):
        bh, g = divmod(i, ng)
        r0, r1 = int(goff[i]), int(goff[i + 1])
        c = cnt[bh, g * 32:(g + 1) * 32]
        assert r1 - r0 == c.max(), (i, r1 - r0, c.max())
        blk = vals[r0 * 32:r1 * 32].reshape(r1 - r0, 32).T
        slot = np.arange(r1 - r0)[None, :]
        assert not np.any(blk[slot >= c[:, None]]), f"group {i}: nonzero unused slots"
        out[bh, g * 32:(g + 1) * 32, :r1 - r0] = blk
    return out[:, :S]


def topp_near_ties(m_g, m_o, k_np, qn_np, p, Tcap):
    """Tokens whose GPU kept set differs from the oracle's, and how many of
    them are counted near-ties (see the module docstring).  A differing token
    that is not a greedy prefix, or not near a tie, is never counted."""
    diff = np.argwhere(np.any(m_g != m_o, axis=-1))
    near = 0
    for bh, t in diff:
        w = (qn_np[bh] * np.abs(k_np[bh, t])).astype(np.float32).astype(np.float64)
        order = sorted(range(D), key=lambda j: (-w[j], j))
        kept = [j for j in range(D) if (int(m_g[bh, t, j // 32]) >> (j % 32)) & 1]
        n_g = len(kept)
        if sorted(order[:n_g]) != kept or n_g > Tcap:
            continue
        total = float(np.sum(w))
        target = float(np.float32(p)) * total
        tol = 2.0 ** -23 * D * total
        pre = np.concatenate([[0.0], np.cumsum(w[order])])
        n_o = int(np.searchsorted(pre >= target, True)) if total > 0 else 0
        if n_g < min(n_o, Tcap) and target - pre[n_g] <= tol:
            near += 1
        elif n_g > n_o and pre[n_g - 1] - target <= tol:
            near += 1
    return len(diff), near


def check_topp(kc, k_np, q_np, G, p, what):
    BH, S, Tcap = kc.B * kc.Hkv, kc.S, kc.T
    qn = oracle.qnorm(q_np.reshape(BH * G, -1, D), G)
    assert np.array_equal(kc.qn.cpu().numpy().reshape(BH, D).view(np.uint32), qn.view(np.uint32)), what
    m_o, v_o, s_o = oracle.prune_topp(k_np.reshape(BH, S, D), qn, p, Tcap)
    s_g = kc.stats.cpu().numpy().reshape(BH, 4)
    if S == 0:
        assert np.array_equal(s_g[:, 0], s_o[:, 0]), f"{what}: pruned count"
        return qn, m_o, v_o, s_o
    m_g = mask_np(kc)
    n_diff, near = topp_near_ties(m_g, m_o, k_np.reshape(BH, S, D), qn, p, Tcap)
    assert n_diff == near, f"{what}: {n_diff - near} of {n_diff} differing tokens are not near-ties"
    assert n_diff <= 1e-4 * BH * S, f"{what}: {n_diff} near-tie tokens of {BH * S}"
    ok = np.all(m_g == m_o, axis=-1)
    v_g = unpack_topp(kc)
    if Tcap > 0:
        assert np.array_equal(v_g[ok].view(np.uint32), v_o[ok].view(np.uint32)), f"{what}: vals"
    if n_diff == 0:
        assert np.array_equal(s_g[:, 0], s_o[:, 0]), f"{what}: pruned count"
        np.testing.assert_allclose(s_g[:, 1:], s_o[:, 1:], rtol=STATS_RTOL, atol=0, err_msg=what)
    return qn, m_o, v_o, s_o


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("S,p,Tcap", [(1, 0.99, 128), (33, 0.99, 128), (1000, 0.99, 128), (2049, 0.9, 96),
                                      (700, 0.99, 40), (300, 0.5, 128), (257, 1.0, 128), (129, 0.0, 64),
                                      (100, 0.99, 0), (0, 0.99, 64)])
def test_topp_parity_and_decode(dtype, S, p, Tcap):
    G = 4
    wl = scaled(WORKLOADS["tiny"], S=S, G=G, Hkv=3, dtype="f32" if dtype == torch.float32 else "bf16",
                seed=700 + S + Tcap)
    pre = make_prefill(wl, DEV)
    what = f"topp S={S} p={p} Tcap={Tcap} {dtype}"
    kc = run_topp(pre["k"], pre["q_obs"], G, wl.W, p, Tcap)
    qn, m, vals, st = check_topp(kc, to_np(pre["k"]), to_np(pre["q_obs"]), G, p, what)
    BH = wl.rows * wl.Hkv
    q = make_decode_step(wl, 1, DEV)["q"]
    out = torch.empty((wl.rows, wl.Hkv * G, D), dtype=torch.float32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, wl.rows, wl.Hkv, G, S, D, Tcap, 0))
    spark_decode_attn_topp(q, kc, pre["v"], None, None, 0, 0, G, out, ws)
    torch.cuda.synchronize()
    o_ref = oracle.decode(to_np(q).reshape(BH * G, D), m, vals, qn, st, to_np(pre["v"]).reshape(BH, S, D), G=G)
    assert_out_close(out.cpu().numpy().reshape(BH * G, D), o_ref, what + " decode")


def test_topp_extreme_tokens():
    """All-zero tokens, single dominant channels, saliencies spanning many
    octaves and exact ties."""
    G, S, Hkv = 2, 512, 2
    wl = scaled(WORKLOADS["tiny"], S=S, G=G, Hkv=Hkv, dtype="bf16", seed=91)
    pre = make_prefill(wl, DEV)
    k = pre["k"].float()
    k[0, 0, 0:40] = 0.0                                  # no saliency at all
    k[0, 0, 40:80] = 0.0
    k[0, 0, 40:80, 7] = 3.0                              # one channel holds everything
    k[0, 1, 0:64] *= torch.logspace(-20, 20, D, base=2.0, device=DEV)   # many octaves
    k[0, 1, 64:128] = torch.round(k[0, 1, 64:128] * 2) / 2              # many exact ties
    k = k.to(torch.bfloat16)
    for p, Tcap in ((0.99, 128), (0.999, 50), (1.0, 128)):
        kc = run_topp(k, pre["q_obs"], G, wl.W, p, Tcap)
        check_topp(kc, to_np(k), to_np(pre["q_obs"]), G, p, f"extreme p={p} Tcap={Tcap}")
        # the groups whose tokens keep one channel or none take 1 or 0 slots
        goff = kc.goff.cpu().numpy().view(np.uint32).astype(np.int64)
        assert goff[1] - goff[0] == 0 and goff[2] - goff[1] == 1
        assert spark_topp_vals_used(kc) < Hkv * S * Tcap * 2


def test_topp_concentrated_saliency_stores_less():
    """Keys whose saliency sits in a few channels per token (the concentrated
    case SparK-p is made for): the compact stream holds about the kept
    values, far below the capacity layout, and still matches the oracle."""
    G, S, Hkv = 4, 4096, 2
    wl = scaled(WORKLOADS["tiny"], S=S, G=G, Hkv=Hkv, dtype="bf16", seed=93)
    pre = make_prefill(wl, DEV)
    g = torch.Generator(device=DEV).manual_seed(93)
    k = pre["k"].float() * 1e-3
    hot = torch.randint(0, D, (1, Hkv, S, 6), generator=g, device=DEV)
    k.scatter_(-1, hot, torch.randn(hot.shape, generator=g, device=DEV) * 10)
    k = k.to(torch.bfloat16)
    kc = run_topp(k, pre["q_obs"], G, wl.W, 0.99, 128)
    check_topp(kc, to_np(k), to_np(pre["q_obs"]), G, 0.99, "concentrated")
    used = spark_topp_vals_used(kc)
    m = mask_np(kc)
    kept = int(np.unpackbits(np.ascontiguousarray(m).view(np.uint8), axis=-1).sum())
    assert kept * 2 <= used <= 4 * kept * 2 and used < Hkv * S * 128 * 2 / 8


def test_topp_decode_gaussian_and_tail():
    """Sampling F and the dense tail over a SparK-p cache."""
    G = 4
    wl = scaled(WORKLOADS["tiny"], S=777, G=G, Hkv=2, dtype="bf16", seed=44)
    pre = make_prefill(wl, DEV)
    kc = run_topp(pre["k"], pre["q_obs"], G, wl.W, 0.99, 100)
    qn, m, vals, st = check_topp(kc, to_np(pre["k"]), to_np(pre["q_obs"]), G, 0.99, "topp tail")
    BH = wl.rows * wl.Hkv
    cap, n_tail = 16, 5
    kt = torch.randn((wl.rows, wl.Hkv, cap, D), device=DEV).to(torch.bfloat16)
    vt = torch.randn((wl.rows, wl.Hkv, cap, D), device=DEV).to(torch.bfloat16)
    q = make_decode_step(wl, 2, DEV)["q"]
    for rec in (0, SPARK_F_GAUSSIAN):
        out = torch.empty((wl.rows, wl.Hkv * G, D), dtype=torch.float32, device=DEV)
        ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, wl.rows, wl.Hkv, G, wl.S, D, kc.T, cap))
        spark_decode_attn_topp(q, kc, pre["v"], kt, vt, cap, n_tail, G, out, ws, recovery=rec, seed=5)
        torch.cuda.synchronize()
        args = (to_np(q).reshape(BH * G, D), m, vals, qn, st, to_np(pre["v"]).reshape(BH, wl.S, D),
                to_np(kt).reshape(BH, cap, D), to_np(vt).reshape(BH, cap, D), n_tail, G)
        o_ref = oracle.decode(*args) if rec == 0 else oracle.decode_f(*args, mode=rec, seed=5)
        assert_out_close(out.cpu().numpy().reshape(BH * G, D), o_ref, f"topp decode F={rec}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T,G", [(1, 4), (26, 4), (26, 1), (26, 8), (47, 2), (64, 4), (127, 8)])
def test_topp_decode_equals_plain_decode_on_full_masks(dtype, T, G):
    """On a plain SparK cache (exactly T bits per token) the SparK-p decode,
    which always steps through the channels in order, gives the same bits as
    spark_decode_attn, which walks the T kept bits of each token for T < 48:
    the kept channels meet the same FMAs in the same order."""
    wl = scaled(WORKLOADS["llama1l"], S=3000, Hkv=3, G=G, dtype=dtype, seed=T + G)
    pre = make_prefill(wl, DEV)
    kc = run_prune(pre["k"], pre["q_obs"], wl.G, wl.W, T)
    q = make_decode_step(wl, 0, DEV)["q"]
    # the plain cache read through group offsets that give every group T slots
    BH, ng = wl.rows * wl.Hkv, (wl.S + 31) // 32
    kc.goff = (torch.arange(BH * ng + 1, device=DEV, dtype=torch.int64) * T).to(torch.int32)
    outs = []
    for fn in (spark_decode_attn, spark_decode_attn_topp):
        out = torch.empty((wl.rows, wl.Hkv * wl.G, D), dtype=torch.float32, device=DEV)
        ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, wl.rows, wl.Hkv, wl.G, wl.S, D, T, 0))
        fn(q, kc, pre["v"], None, None, 0, 0, wl.G, out, ws)
        torch.cuda.synchronize()
        assert spark_device_status(ws) == 0
        outs.append(out)
    assert torch.equal(outs[0], outs[1])


def test_topp_full_size_sampled():
    """One layer of the long-context workload (8 heads x 131072 tokens) in
    the launch configuration of the benchmark: sampled tokens against the
    oracle, every mask within the capacity, and the compact value stream
    smaller than the capacity layout."""
    wl = scaled(WORKLOADS["long"], L=1)
    pre = make_prefill(wl, DEV)
    Tcap = 96
    kc = run_topp(pre["k"], pre["q_obs"], wl.G, wl.W, 0.99, Tcap)
    BH, S = wl.rows * wl.Hkv, wl.S
    qn = oracle.qnorm(to_np(pre["q_obs"]).reshape(BH * wl.G, -1, D), wl.G)
    m_g = mask_np(kc)
    pc = np.zeros(m_g.shape[:2], np.int64)
    for wd in range(4):
        x = m_g[..., wd].astype(np.uint64)
        pc += np.array([bin(int(v)).count("1") for v in x.ravel()]).reshape(x.shape)
    assert pc.max() <= Tcap
    st = kc.stats.cpu().numpy().reshape(BH, 4)
    assert np.array_equal(st[:, 0], (D - pc).sum(1).astype(np.float64))
    rng = np.random.default_rng(1)
    vals_g = unpack_topp(kc)
    k_np = to_np(pre["k"]).reshape(BH, S, D)
    n_diff = n_near = 0
    for bh in range(BH):
        ts = np.sort(rng.choice(S, 4096, replace=False))
        m_o, v_o, _ = oracle.prune_topp(k_np[bh, ts][None], qn[bh:bh + 1], 0.99, Tcap)
        d, nr = topp_near_ties(m_g[bh, ts][None], m_o, k_np[bh, ts][None], qn[bh:bh + 1], 0.99, Tcap)
        n_diff, n_near = n_diff + d, n_near + nr
        ok = np.all(m_g[bh, ts] == m_o[0], axis=-1)
        assert np.array_equal(vals_g[bh, ts][ok].view(np.uint32), v_o[0][ok].view(np.uint32)), f"head {bh}"
    assert n_diff == n_near and n_diff <= 1e-4 * BH * 4096, (n_diff, n_near)
    # the compact stream: each group holds its longest kept set (here nearly
    # every group has a token cut at the cap, so it is close to the capacity)
    used = spark_topp_vals_used(kc)
    assert used == int(kc.goff[-1].item()) * 32 * 2 and used <= BH * S * Tcap * 2


@pytest.mark.parametrize("G", [1, 2, 8])
def test_topp_group_sizes(G):
    """The variable-count decode walk for every supported GQA group size (the
    odd size takes the scalar FMA path, the others packed head pairs)."""
    wl = scaled(WORKLOADS["tiny"], S=600, G=G, Hkv=2, dtype="bf16", seed=810 + G)
    pre = make_prefill(wl, DEV)
    kc = run_topp(pre["k"], pre["q_obs"], G, wl.W, 0.9, 100)
    qn, m, vals, st = check_topp(kc, to_np(pre["k"]), to_np(pre["q_obs"]), G, 0.9, f"topp G={G}")
    BH = wl.rows * wl.Hkv
    q = make_decode_step(wl, 3, DEV)["q"]
    out = torch.empty((wl.rows, wl.Hkv * G, D), dtype=torch.float32, device=DEV)
    ws = workspace(spark_workspace_bytes(SPARK_OP_DECODE, wl.rows, wl.Hkv, G, wl.S, D, kc.T, 0))
    spark_decode_attn_topp(q, kc, pre["v"], None, None, 0, 0, G, out, ws)
    torch.cuda.synchronize()
    o_ref = oracle.decode(to_np(q).reshape(BH * G, D), m, vals, qn, st, to_np(pre["v"]).reshape(BH, wl.S, D), G=G)
    assert_out_close(out.cpu().numpy().reshape(BH * G, D), o_ref, f"topp decode G={G}")
