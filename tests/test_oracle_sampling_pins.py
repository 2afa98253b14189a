"""Pins for the sampling recoveries of the oracle (F table of the SparK
walkthrough, section 3.3: Gaussian N(mu, sigma^2) and Exponential Exp(1/mu);
reading R14: one Philox4x32-10 draw per pruned entry).  The generator is
pinned to its published known-answer vectors; the samplers to the moments of
the distributions they claim; Degenerate to the closed-form path."""
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for ln in open(GOLD):
        if ln.strip() and not ln.startswith("#"):
            v = [int(x, 16) for x in ln.split()]
            rows.append((v[:4], v[4:6], v[6:10]))
    return rows


@pytest.mark.parametrize("row", range(3))
def test_philox_known_answers(row):
    ctr, key, want = _kat()[row]
    assert list(oracle.philox4x32_10(ctr, key)) == want


def _draws(mode, st, n, seed=7):
    return np.array([oracle.sample_score(mode, st, seed, 3, t, t % 128) for t in range(n)])


def test_gaussian_moments():
    mu, sigma = 2.5, 0.75
    st = np.array([1000.0, 1000.0 * mu, 1000.0 * (sigma ** 2 + mu ** 2), mu])
    x = _draws(oracle.GAUSSIAN, st, 60000)
    assert abs(x.mean() - mu) < 5 * sigma / np.sqrt(len(x))
    assert abs(x.std() - sigma) < 0.02 * sigma
    # symmetric: third standardised moment near zero, kurtosis near 3
    z = (x - x.mean()) / x.std()
    assert abs((z ** 3).mean()) < 0.05 and abs((z ** 4).mean() - 3.0) < 0.1


def test_exponential_moments():
    mu = 1.7
    st = np.array([10.0, 10.0 * mu, 0.0, mu])
    x = _draws(oracle.EXPONENTIAL, st, 60000)
    assert np.all(x > 0)
    assert abs(x.mean() - mu) < 5 * mu / np.sqrt(len(x))
    assert abs(x.std() - mu) < 0.03 * mu  # Exp: sd = mean


def test_degenerate_is_mu_and_seed_free():
    st = np.array([5.0, 6.0, 9.0, 1.2])
    assert oracle.sample_score(oracle.DEGENERATE, st, 1, 0, 0, 0) == 1.2
    assert oracle.sample_score(oracle.DEGENERATE, st, 99, 4, 8, 9) == 1.2


def test_draws_depend_on_every_counter_field():
    st = np.array([10.0, 10.0, 20.0, 1.0])
    base = oracle.sample_score(oracle.EXPONENTIAL, st, 5, 2, 3, 4)
    assert oracle.sample_score(oracle.EXPONENTIAL, st, 5, 2, 3, 4) == base
    for args in [(6, 2, 3, 4), (5, 3, 3, 4), (5, 2, 4, 4), (5, 2, 3, 5), (5 + (1 << 32), 2, 3, 4),
                 (5, 2 + (1 << 32), 3, 4)]:
        assert oracle.sample_score(oracle.EXPONENTIAL, st, *args) != base


def _case(seed=0, T=26, BH=2, S=40, G=4):
    rng = np.random.default_rng(seed)
    k = (rng.standard_normal((BH, S, 128)) * np.exp(rng.standard_normal((BH, 1, 128)))).astype(np.float32)
    v = rng.standard_normal((BH, S, 128)).astype(np.float32)
    q = rng.standard_normal((BH * G, 128)).astype(np.float32)
    qn = np.exp(rng.standard_normal((BH, 128))).astype(np.float32)
    m, vals, st = oracle.prune(k, qn, T)
    return q, m, vals, qn, st, v, G


def test_degenerate_mode_matches_closed_form_path():
    q, m, vals, qn, st, v, G = _case()
    assert np.array_equal(oracle.decode_f(q, m, vals, qn, st, v, G=G, mode=oracle.DEGENERATE, seed=3),
                          oracle.decode(q, m, vals, qn, st, v, G=G))
    assert np.array_equal(oracle.recover_keys_f(m, vals, qn, st, 1, oracle.DEGENERATE, 3),
                          oracle.recover_keys(m, vals, qn, st, 1))


@pytest.mark.parametrize("mode", [oracle.GAUSSIAN, oracle.EXPONENTIAL])
def test_sampled_keys_back_solve_the_draw(mode):
    # kept entries are untouched; pruned entries satisfy qn_j * k~_j = w~
    q, m, vals, qn, st, v, G = _case(seed=4)
    bits = np.unpackbits(m.view(np.uint8), axis=-1, bitorder="little").astype(bool)
    Kt = oracle.recover_keys_f(m, vals, qn, st, 0, mode, 11)
    Kd = oracle.recover_keys(m, vals, qn, st, 0)
    assert np.array_equal(Kt[bits[0]], Kd[bits[0]])
    for t in (0, 17, 39):
        for j in np.nonzero(~bits[0, t])[0][:5]:
            w = oracle.sample_score(mode, st[0], 11, 0, t, int(j))
            assert Kt[t, j] * np.float64(qn[0, j]) == pytest.approx(w, rel=1e-14)
