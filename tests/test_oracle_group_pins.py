"""Pins of the oracle's SparK-g pruning (reading R15 of the oracle: channel
groups by window-query norm rank, one per-token top-T budget per group), each
against something other than the oracle's own code: brute force over subsets,
closed forms, the plain top-T special case, and invariants."""
import itertools

import numpy as np
import pytest

import oracle


def _groups(qn, g):
    D = len(qn)
    order = sorted(range(D), key=lambda j: (-float(qn[j]), j))
    gid = np.zeros(D, int)
    for k in range(g):
        for r in range(k * D // g, (k + 1) * D // g):
            gid[order[r]] = k
    return gid


def test_budget_closed_forms():
    # [W] 5.2: g = 4 with pruning rates (0.25, 0.5, 0.75, 1.0) on 32-channel groups
    assert oracle.group_budget(128, [0.25, 0.5, 0.75, 1.0]) == [24, 16, 8, 0]
    assert oracle.group_budget(128, [0.0] * 4) == [32] * 4
    assert oracle.group_budget(128, [1.0] * 8) == [0] * 8
    # g = 5: group sizes 25, 26, 25, 26, 26 (rank cuts at k*128/5)
    assert oracle.group_budget(128, [0.0] * 5) == [25, 26, 25, 26, 26]
    # halves round away from zero: 0.5 * 25 = 12.5 -> 13
    assert oracle.group_budget(128, [0.5] * 5) == [13, 13, 13, 13, 13]


def test_groups_follow_query_norm_rank():
    qn = np.array([[3.0, 9.0, 1.0, 9.0, 5.0, 0.0, 7.0, 2.0]], np.float32)
    gid = oracle.group_of_channel(qn, 2)[0]
    # ranks by (qn desc, j asc): 1, 3, 6, 4 | 0, 7, 2, 5
    assert list(gid) == [1, 0, 1, 0, 0, 1, 0, 1]
    gid4 = oracle.group_of_channel(qn, 4)[0]
    assert list(gid4) == [2, 0, 3, 0, 1, 3, 1, 2]
    # equal norms across a group boundary: the lower channel takes the
    # higher-ranked group
    tied = np.array([[5.0, 1.0, 5.0, 5.0]], np.float32)
    assert list(oracle.group_of_channel(tied, 2)[0]) == [0, 1, 0, 1]
    rng = np.random.default_rng(3)
    qr = rng.random((3, 128)).astype(np.float32)
    for g in (1, 2, 4, 5, 8):
        got = oracle.group_of_channel(qr, g)
        for b in range(3):
            assert np.array_equal(got[b], _groups(qr[b], g))


def test_one_group_is_plain_top_t():
    rng = np.random.default_rng(1)
    k = rng.standard_normal((3, 70, 128)).astype(np.float32)
    qn = np.abs(rng.standard_normal((3, 128))).astype(np.float32)
    for T in (0, 1, 26, 64, 127, 128):
        a = oracle.prune(k, qn, T)
        b = oracle.prune_grouped(k, qn, [T])
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


@pytest.mark.parametrize("Tg", [(2, 1), (0, 3), (4, 0), (1, 1), (3, 4)])
def test_brute_force_small(Tg):
    # D = 8, g = 2: the kept set maximises sum w with |kept & group k| = Tg[k];
    # among optima (integer saliencies make ties common) the smallest channel
    # indices win
    rng = np.random.default_rng(sum(Tg) + 7)
    D, g = 8, 2
    qn = np.array([[5.0, 1.0, 4.0, 2.0, 8.0, 3.0, 7.0, 6.0]], np.float32)
    gid = _groups(qn[0], g)
    for trial in range(40):
        k = rng.integers(-3, 4, (1, 1, D)).astype(np.float32)
        w = [float(np.float32(qn[0, j]) * np.float32(abs(k[0, 0, j]))) for j in range(D)]
        best, best_set = None, None
        for sub in itertools.combinations(range(D), sum(Tg)):
            if any(sum(1 for j in sub if gid[j] == q) != Tg[q] for q in range(g)):
                continue
            val = sum(w[j] for j in sub)
            if best is None or val > best or (val == best and list(sub) < best_set):
                best, best_set = val, list(sub)
        m, v, _ = oracle.prune_grouped(k, qn, list(Tg))
        got = [j for j in range(D) if (int(m[0, 0, 0]) >> j) & 1]
        assert got == best_set, (trial, w, got, best_set)
        assert np.array_equal(v[0, 0], k[0, 0, got])


def test_counts_values_and_statistics():
    rng = np.random.default_rng(5)
    BH, S, D = 2, 90, 128
    k = (rng.standard_normal((BH, S, D)) * np.exp(rng.standard_normal(D))).astype(np.float32)
    qn = np.abs(rng.standard_normal((BH, D))).astype(np.float32)
    Tg = oracle.group_budget(D, [0.25, 0.5, 0.75, 1.0])
    m, v, st = oracle.prune_grouped(k, qn, Tg)
    bits = ((m[..., None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(BH, S, D).astype(bool)
    w = (qn[:, None, :] * np.abs(k)).astype(np.float32)
    for b in range(BH):
        gid = _groups(qn[b], 4)
        for q in range(4):
            sel = gid == q
            assert np.all(bits[b][:, sel].sum(1) == Tg[q])
            # inside a group every kept saliency dominates every pruned one
            kept = np.where(bits[b][:, sel], w[b][:, sel], np.inf).min(1)
            pruned = np.where(~bits[b][:, sel], w[b][:, sel], -np.inf).max(1)
            assert np.all(kept >= pruned)
        # packed values: the kept keys in ascending channel order, bit for bit
        for t in range(S):
            assert np.array_equal(v[b, t].view(np.uint32), k[b, t, bits[b, t]].view(np.uint32))
        pw = w[b][~bits[b]].astype(np.float64)
        assert st[b, 0] == S * (D - sum(Tg))
        np.testing.assert_allclose(st[b, 1], pw.sum(), rtol=1e-12)
        np.testing.assert_allclose(st[b, 2], (pw * pw).sum(), rtol=1e-12)
        np.testing.assert_allclose(st[b, 3], pw.sum() / pw.size, rtol=1e-12)


def test_channel_permutation_equivariance():
    rng = np.random.default_rng(11)
    k = rng.standard_normal((1, 40, 128)).astype(np.float32)
    qn = (rng.permutation(128).astype(np.float32) + 1.0)[None]  # distinct norms
    perm = rng.permutation(128)
    Tg = [20, 10, 5, 1]
    m, _, _ = oracle.prune_grouped(k, qn, Tg)
    mp, _, _ = oracle.prune_grouped(k[..., perm], qn[:, perm], Tg)
    bits = ((m[..., None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(1, 40, 128)
    bp = ((mp[..., None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(1, 40, 128)
    assert np.array_equal(bits[..., perm], bp)
