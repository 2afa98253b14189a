"""Pins of the oracle's ThinK comparator (reading R18: one channel mask per
(b, h), channels ranked by qn_j * ||k^j||_2, no recovery), against brute
force, closed forms and numpy restatements."""
import itertools

import numpy as np
import pytest

import oracle

D = 128


def _bits(m, D):
    return ((m[..., None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(*m.shape[:-1], D).astype(bool)


@pytest.mark.parametrize("T", [0, 1, 26, 64, 127, 128])
def test_mask_is_shared_and_values_exact(T):
    rng = np.random.default_rng(T + 3)
    k = (rng.standard_normal((2, 50, D)) * np.exp(rng.standard_normal(D))).astype(np.float32)
    qn = np.abs(rng.standard_normal((2, D))).astype(np.float32)
    m, v, st = oracle.think_prune(k, qn, T)
    b = _bits(m, D)
    for h in range(2):
        assert np.all(b[h] == b[h, 0])               # one mask for every token
        assert b[h, 0].sum() == T
        for t in range(50):
            assert np.array_equal(v[h, t].view(np.uint32), k[h, t, b[h, t]].view(np.uint32))
        assert list(st[h]) == [50.0 * (D - T), 0.0, 0.0, 0.0]


def test_brute_force_channel_set():
    # D = 8: the kept set maximises the sum of the channel scores over all
    # size-T subsets; equal scores -> smallest indices
    rng = np.random.default_rng(9)
    D8 = 8
    for trial in range(30):
        k = rng.integers(-2, 3, (1, 6, D8)).astype(np.float32)
        qn = rng.integers(0, 3, (1, D8)).astype(np.float32)
        score = [float(qn[0, j]) * float(np.sqrt(np.sum(k[0, :, j].astype(np.float64) ** 2))) for j in range(D8)]
        for T in (1, 3, 5):
            best, best_set = None, None
            for sub in itertools.combinations(range(D8), T):
                val = sum(score[j] for j in sub)
                if best is None or val > best + 1e-12 or (abs(val - best) <= 1e-12 and list(sub) < best_set):
                    best, best_set = val, list(sub)
            m, _, _ = oracle.think_prune(k, qn, T)
            got = [j for j in range(D8) if (int(m[0, 0, 0]) >> j) & 1]
            assert got == best_set, (trial, T, score, got, best_set)


def test_channel_scaling_and_token_order():
    rng = np.random.default_rng(4)
    k = rng.standard_normal((1, 40, D)).astype(np.float32)
    qn = (rng.random((1, D)) + 0.5).astype(np.float32)
    m0, _, _ = oracle.think_prune(k, qn, 64)
    # boosting one pruned channel's keys by 1000 moves it into the kept set
    pruned = np.flatnonzero(~_bits(m0, D)[0, 0])
    k2 = k.copy()
    k2[..., pruned[0]] *= 1000.0
    m2, _, _ = oracle.think_prune(k2, qn, 64)
    assert _bits(m2, D)[0, 0, pruned[0]]
    # the column norm ignores token order
    perm = rng.permutation(40)
    m3, _, _ = oracle.think_prune(k[:, perm], qn, 64)
    assert np.array_equal(m3[0, 0], m0[0, 0])


def test_decode_is_attention_over_kept_channels():
    # no recovery: scores use the kept channels only
    rng = np.random.default_rng(6)
    G, S = 2, 37
    k = rng.standard_normal((1, S, D)).astype(np.float32)
    v = rng.standard_normal((1, S, D)).astype(np.float32)
    qo = rng.standard_normal((G, 8, D)).astype(np.float32)
    q = rng.standard_normal((G, D)).astype(np.float32)
    qn = oracle.qnorm(qo, G)
    m, vals, st = oracle.think_prune(k, qn, 40)
    keep = _bits(m, D)[0, 0]
    out = oracle.decode(q, m, vals, qn, st, v, G=G)
    for g in range(G):
        s = (k[0][:, keep].astype(np.float64) @ q[g, keep].astype(np.float64)) / np.sqrt(D)
        p = np.exp(s - s.max())
        p /= p.sum()
        np.testing.assert_allclose(out[g], (p @ v[0].astype(np.float64)).astype(np.float32), rtol=1e-6, atol=1e-7)
