"""Pins for the CPU oracle: each checks it against something other than
itself -- closed forms, brute force, invariants the SparK pages state, or a
library routine for a special case.  No GPU needed.

Pages: "KV Cache 还能再砍一刀：SparK 在通道维度上做了一件被忽略多年的事"
(paper walkthrough) sections 3.1-3.3 and Fig. 3; AMD blog "AAAI 2026 AMD论文
Spark方法揭秘" (decode = standard full attention after recovery).
"""
import itertools

import numpy as np
import pytest
import torch

import oracle

D = 128


def _rng(seed):
    return np.random.default_rng(seed)


def _outlier(rng, shape, scale_shape):
    s = np.exp(rng.standard_normal(scale_shape)).astype(np.float32)
    return (rng.standard_normal(shape).astype(np.float32) * s).astype(np.float32)


# --------------------------------------------------------------- lambda -> T
def test_lambda_to_T_values():
    # T = round((1 - lambda) * D): 0.3 -> 89.6 -> 90, 0.5 -> 64, 0.8 -> 25.6 -> 26
    assert oracle.lambda_to_T(0.3, D) == 90
    assert oracle.lambda_to_T(0.5, D) == 64
    assert oracle.lambda_to_T(0.8, D) == 26
    assert oracle.lambda_to_T(0.0, D) == 128
    assert oracle.lambda_to_T(1.0, D) == 0
    assert oracle.lambda_to_T(-0.1, D) == -1
    assert oracle.lambda_to_T(1.5, D) == -1
    assert oracle.lambda_to_T(float("nan"), D) == -1


# ----------------------------------------------------------------- qnorm
def test_qnorm_all_ones_closed_form():
    G, W = 4, 16
    q = np.ones((2 * G, W, D), np.float32)
    qn = oracle.qnorm(q, G)
    assert qn.shape == (2, D)
    assert np.all(qn == np.float32(np.sqrt(G * W)))


def test_qnorm_pythagorean_and_group_isolation():
    G, W = 4, 8
    q = np.zeros((3 * G, W, D), np.float32)
    # kv head 1: entries 3 and 4 in different (g, t) cells of channel 5 -> 5
    q[1 * G + 0, 2, 5] = 3.0
    q[1 * G + 3, 7, 5] = -4.0
    # kv head 1, channel 9: a single entry -> its magnitude
    q[1 * G + 2, 0, 9] = -2.5
    # kv heads 0 and 2 carry huge values that must not leak into head 1
    q[0 * G:1 * G] = 1e6
    q[2 * G:3 * G] = -1e6
    qn = oracle.qnorm(q, G)
    assert qn[1, 5] == 5.0
    assert qn[1, 9] == 2.5
    assert np.all(np.delete(qn[1], [5, 9]) == 0.0)
    assert np.all(qn[0] > 1e6)


def test_qnorm_sums_every_window_row_and_group_head():
    # each (g, t) cell contributes 1 in its own channel set: qn^2 counts them
    G, W = 4, 16
    q = np.zeros((G, W, D), np.float32)
    for g in range(G):
        for t in range(W):
            q[g, t, (g * W + t) % D] = 1.0
            q[g, t, D - 1] = 1.0
    qn = oracle.qnorm(q, G)
    assert qn[0, D - 1] == np.float32(np.sqrt(G * W))
    assert np.all(qn[0, : G * W] == 1.0)


# ------------------------------------------------------- top-T brute force
def _lex_first_optimum(w, T):
    """Brute force over all C(D, T) subsets of the relaxed objective
    max sum_j w_j z_j, sum z = T; among optima the lexicographically first
    index set (the lower-index tie rule)."""
    best, best_set = None, None
    for sub in itertools.combinations(range(len(w)), T):  # lexicographic order
        val = sum(int(w[j]) for j in sub)                   # exact integers
        if best is None or val > best:
            best, best_set = val, sub
    return set(best_set)


@pytest.mark.parametrize("T", range(0, 9))
def test_topT_bruteforce_D8(orc, T):
    rng = _rng(100 + T)
    Dt, S = 8, 300
    # integer-valued keys with many ties; qn a power of two keeps w exact
    k = rng.integers(-3, 4, size=(1, S, Dt)).astype(np.float32)
    qn = np.full((1, Dt), 2.0, np.float32)
    qn[0, 5] = 4.0
    mask, vals, stats = oracle.prune(k, qn, T, lib=orc)
    for t in range(S):
        w = (np.abs(k[0, t]) * qn[0]).astype(np.int64)
        want = _lex_first_optimum(w, T)
        got = {j for j in range(Dt) if (mask[0, t, 0] >> j) & 1}
        assert got == want, (t, w, got, want)
        assert mask[0, t, 0] >> Dt == 0


def test_topT_bruteforce_D8_distinct_floats(orc):
    rng = _rng(7)
    Dt, S, T = 8, 200, 4
    k = rng.standard_normal((1, S, Dt)).astype(np.float32)
    qn = np.exp(rng.standard_normal((1, Dt))).astype(np.float32)
    mask, _, _ = oracle.prune(k, qn, T, lib=orc)
    for t in range(S):
        w = (qn[0] * np.abs(k[0, t])).astype(np.float32).astype(np.float64)
        best = max(itertools.combinations(range(Dt), T), key=lambda s: sum(w[j] for j in s))
        got = {j for j in range(Dt) if (mask[0, t, 0] >> j) & 1}
        assert got == set(best)


# ------------------------------------------- mask / packed-value invariants
@pytest.mark.parametrize("T", [0, 1, 26, 64, 90, 127, 128])
def test_popcount_and_values_bit_exact(orc, T):
    rng = _rng(T)
    BH, S = 3, 97
    k = _outlier(rng, (BH, S, D), (BH, 1, D))
    qn = np.exp(rng.standard_normal((BH, D))).astype(np.float32)
    mask, vals, stats = oracle.prune(k, qn, T, lib=orc)
    bits = np.unpackbits(mask.view(np.uint8), axis=-1, bitorder="little").astype(bool)
    assert np.all(bits.sum(-1) == T)                 # sum z = T per token
    for bh in range(BH):
        for t in range(S):
            kept = k[bh, t][bits[bh, t]]             # ascending channel order
            assert np.array_equal(kept.view(np.uint32), vals[bh, t].view(np.uint32))
    # N_pruned = S * (D - T) for every head
    assert np.all(stats[:, 0] == S * (D - T))


def test_kept_channels_dominate_pruned(orc):
    # optimality of top-T for the relaxed objective: every kept saliency is
    # >= every pruned saliency of the same token
    rng = _rng(3)
    BH, S, T = 2, 64, 26
    k = _outlier(rng, (BH, S, D), (BH, 1, D))
    qn = np.exp(rng.standard_normal((BH, D))).astype(np.float32)
    mask, _, _ = oracle.prune(k, qn, T, lib=orc)
    bits = np.unpackbits(mask.view(np.uint8), axis=-1, bitorder="little").astype(bool)
    w = (qn[:, None, :] * np.abs(k)).astype(np.float32)
    for bh in range(BH):
        for t in range(S):
            assert w[bh, t][bits[bh, t]].min() >= w[bh, t][~bits[bh, t]].max()


def test_stats_partition_identity(orc):
    # pruned + kept saliency = all saliency; mean over the pruned set
    rng = _rng(11)
    BH, S, T = 2, 200, 64
    k = _outlier(rng, (BH, S, D), (BH, 1, D))
    qn = np.exp(rng.standard_normal((BH, D))).astype(np.float32)
    mask, vals, stats = oracle.prune(k, qn, T, lib=orc)
    bits = np.unpackbits(mask.view(np.uint8), axis=-1, bitorder="little").astype(bool)
    w = (qn[:, None, :] * np.abs(k)).astype(np.float32).astype(np.float64)
    for bh in range(BH):
        kept_sum = 0.0
        for t in range(S):
            ch = np.nonzero(bits[bh, t])[0]
            kept_sum += float(np.sum((qn[bh, ch] * np.abs(vals[bh, t])).astype(np.float32)
                                     .astype(np.float64)))
        total = float(w[bh].sum())
        assert stats[bh, 1] + kept_sum == pytest.approx(total, rel=1e-12)
        assert stats[bh, 3] == pytest.approx(stats[bh, 1] / stats[bh, 0], rel=1e-15)
        assert stats[bh, 2] >= stats[bh, 1] ** 2 / stats[bh, 0] * (1 - 1e-12)  # Cauchy-Schwarz


def test_full_keep_has_no_stats(orc):
    rng = _rng(5)
    k = rng.standard_normal((1, 10, D)).astype(np.float32)
    qn = np.ones((1, D), np.float32)
    _, vals, stats = oracle.prune(k, qn, D, lib=orc)
    assert np.array_equal(vals, k)
    assert np.all(stats == 0.0)


# ------------------------------------------------------------- recovery
def test_recovery_back_solve_invariant(orc):
    # qn_j * k~_j = mu_pruned on every pruned entry; qn_j = 0 gives k~ = 0
    rng = _rng(13)
    BH, S, T = 2, 50, 26
    k = _outlier(rng, (BH, S, D), (BH, 1, D))
    qn = np.exp(rng.standard_normal((BH, D))).astype(np.float32)
    qn[1, 17] = 0.0
    mask, vals, stats = oracle.prune(k, qn, T, lib=orc)
    bits = np.unpackbits(mask.view(np.uint8), axis=-1, bitorder="little").astype(bool)
    for bh in range(BH):
        Kt = oracle.recover_keys(mask, vals, qn, stats, bh, lib=orc)
        mu = stats[bh, 3]
        pr = ~bits[bh]
        prod = Kt * qn[bh].astype(np.float64)[None, :]
        ok = pr & (qn[bh] > 0)[None, :]
        assert np.allclose(prod[ok], mu, rtol=1e-14, atol=0)
        assert np.all(Kt[:, qn[bh] == 0][pr[:, qn[bh] == 0]] == 0.0)
        assert np.array_equal(Kt[bits[bh]], k[bh][bits[bh]].astype(np.float64))


# ---------------------------------------------------------------- decode
def _sdpa_fp64(q, k, v, G):
    """torch scaled_dot_product_attention in fp64 (library special case)."""
    BHG, Dd = q.shape
    qq = torch.from_numpy(q.astype(np.float64)).view(-1, G, 1, Dd)          # [BH, G, 1, D]
    kk = torch.from_numpy(k.astype(np.float64))[:, None].expand(-1, G, -1, -1)
    vv = torch.from_numpy(v.astype(np.float64))[:, None].expand(-1, G, -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)
    return o.reshape(BHG, Dd).numpy()


@pytest.mark.parametrize("n_tail", [0, 5])
def test_lambda0_is_dense_attention(orc, n_tail):
    rng = _rng(21 + n_tail)
    BH, G, S, cap = 3, 4, 77, 8
    k = _outlier(rng, (BH, S, D), (BH, 1, D))
    v = _outlier(rng, (BH, S, D), (BH, 1, D))
    q = _outlier(rng, (BH * G, D), (BH * G, D))
    kt = _outlier(rng, (BH, cap, D), (BH, 1, D))
    vt = _outlier(rng, (BH, cap, D), (BH, 1, D))
    qn = np.exp(rng.standard_normal((BH, D))).astype(np.float32)
    mask, vals, stats = oracle.prune(k, qn, D, lib=orc)
    out = oracle.decode(q, mask, vals, qn, stats, v, kt, vt, n_tail, G, lib=orc)
    kf = np.concatenate([k, kt[:, :n_tail]], axis=1)
    vf = np.concatenate([v, vt[:, :n_tail]], axis=1)
    ref = _sdpa_fp64(q, kf, vf, G)
    np.testing.assert_allclose(out, ref.astype(np.float32), rtol=1e-6, atol=1e-6)


def test_all_pruned_gives_mean_of_values(orc):
    # T = 0: every key is recovered to mu/qn_j, identical for all tokens, so
    # the softmax is uniform and out = mean of V
    rng = _rng(31)
    BH, G, S = 2, 4, 40
    k = _outlier(rng, (BH, S, D), (BH, 1, D))
    v = _outlier(rng, (BH, S, D), (BH, 1, D))
    q = _outlier(rng, (BH * G, D), (BH * G, D))
    qn = np.exp(rng.standard_normal((BH, D))).astype(np.float32)
    mask, vals, stats = oracle.prune(k, qn, 0, lib=orc)
    assert np.all(stats[:, 3] > 0)
    out = oracle.decode(q, mask, vals, qn, stats, v, G=G, lib=orc)
    ref = np.repeat(v.astype(np.float64).mean(axis=1), G, axis=0)
    np.testing.assert_allclose(out, ref, rtol=1e-5, atol=1e-6)


def test_all_pruned_score_is_closed_form(orc):
    # T = 0 with one extra dense tail token: score of a prefix token is
    # mu * sum_j q_j / qn_j / sqrt(D); two-token softmax in closed form
    rng = _rng(41)
    G = 1
    k = rng.standard_normal((1, 1, D)).astype(np.float32)
    v = rng.standard_normal((1, 1, D)).astype(np.float32)
    kt = rng.standard_normal((1, 1, D)).astype(np.float32)
    vt = rng.standard_normal((1, 1, D)).astype(np.float32)
    q = rng.standard_normal((1, D)).astype(np.float32)
    qn = np.exp(rng.standard_normal((1, D))).astype(np.float32)
    mask, vals, stats = oracle.prune(k, qn, 0, lib=orc)
    mu = float(stats[0, 3])
    s0 = mu * float(np.sum(q[0].astype(np.float64) / qn[0].astype(np.float64))) / np.sqrt(D)
    s1 = float(np.dot(q[0].astype(np.float64), kt[0, 0].astype(np.float64))) / np.sqrt(D)
    p0 = 1.0 / (1.0 + np.exp(s1 - s0))
    ref = p0 * v[0, 0].astype(np.float64) + (1 - p0) * vt[0, 0].astype(np.float64)
    out = oracle.decode(q, mask, vals, qn, stats, v, kt, vt, 1, G, lib=orc)
    np.testing.assert_allclose(out[0], ref, rtol=1e-6, atol=1e-7)


def test_single_token_returns_its_value(orc):
    rng = _rng(51)
    k = rng.standard_normal((2, 1, D)).astype(np.float32)
    v = rng.standard_normal((2, 1, D)).astype(np.float32)
    q = rng.standard_normal((8, D)).astype(np.float32)
    qn = np.exp(rng.standard_normal((2, D))).astype(np.float32)
    mask, vals, stats = oracle.prune(k, qn, 26, lib=orc)
    out = oracle.decode(q, mask, vals, qn, stats, v, G=4, lib=orc)
    assert np.array_equal(out, np.repeat(v[:, 0], 4, axis=0))


def test_empty_context_is_zero(orc):
    qn = np.ones((2, D), np.float32)
    k = np.zeros((2, 0, D), np.float32)
    mask, vals, stats = oracle.prune(k, qn, 26, lib=orc)
    q = np.ones((8, D), np.float32)
    out = oracle.decode(q, mask, vals, qn, stats, k, G=4, lib=orc)
    assert out.shape == (8, D) and np.all(out == 0.0)


def test_query_scale_invariance(orc):
    # doubling the window queries doubles qn and mu exactly: masks, values and
    # the recovered keys (mu / qn) -- hence the output -- are unchanged
    rng = _rng(61)
    BH, G, W, S, T = 2, 4, 16, 60, 26
    q_obs = _outlier(rng, (BH * G, W, D), (BH * G, 1, D))
    k = _outlier(rng, (BH, S, D), (BH, 1, D))
    v = _outlier(rng, (BH, S, D), (BH, 1, D))
    q = _outlier(rng, (BH * G, D), (BH * G, D))
    outs = []
    for f in (1.0, 2.0):
        qn = oracle.qnorm(q_obs * np.float32(f), G, lib=orc)
        m, vl, st = oracle.prune(k, qn, T, lib=orc)
        outs.append((m, vl, st, oracle.decode(q, m, vl, qn, st, v, G=G, lib=orc)))
    assert np.array_equal(outs[0][0], outs[1][0])
    assert np.array_equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][2][:, 3] * 2, outs[1][2][:, 3])
    assert np.array_equal(outs[0][3], outs[1][3])


def test_token_permutation_equivariance(orc):
    rng = _rng(71)
    BH, G, S, T = 2, 4, 90, 64
    k = _outlier(rng, (BH, S, D), (BH, 1, D))
    v = _outlier(rng, (BH, S, D), (BH, 1, D))
    q = _outlier(rng, (BH * G, D), (BH * G, D))
    qn = np.exp(rng.standard_normal((BH, D))).astype(np.float32)
    perm = rng.permutation(S)
    m1, v1, s1 = oracle.prune(k, qn, T, lib=orc)
    m2, v2, s2 = oracle.prune(k[:, perm], qn, T, lib=orc)
    assert np.array_equal(m1[:, perm], m2)
    assert np.array_equal(v1[:, perm], v2)
    np.testing.assert_allclose(s1, s2, rtol=1e-13)
    o1 = oracle.decode(q, m1, v1, qn, s1, v, G=G, lib=orc)
    o2 = oracle.decode(q, m2, v2, qn, s2, v[:, perm], G=G, lib=orc)
    np.testing.assert_allclose(o1, o2, rtol=1e-6, atol=1e-7)
