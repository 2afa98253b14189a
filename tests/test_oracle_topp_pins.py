"""Pins for the SparK-p oracle (per-token top-p channel selection, reading
R19 of the oracle: the shortest greedy prefix of channels whose cumulative
saliency, summed in fp64 in greedy order, reaches p times the token's total,
capped at Tcap).

Source: "KV Cache 还能再砍一刀：SparK ..." section 5.2 (SparK-p: every token
keeps the fewest channels whose cumulative saliency reaches 99 %), with the
greedy order and tie rule of section 3.1.  Each pin fixes a part of the
oracle from outside it: a brute-force minimum over all channel subsets on
exact (integer) saliencies, closed forms for p = 0 / p = 1 / all-zero
tokens, the cap against plain top-T pruning, hand-built cases whose exact
sums an fp32 accumulation would get wrong, and invariants on random data
checked with exact rational sums.
"""
import itertools

import numpy as np
import pytest

import oracle


def _popc(mrow):
    return sum(bin(int(x)).count("1") for x in mrow)


def _kept(mrow, D):
    return [j for j in range(D) if (int(mrow[j // 32]) >> (j % 32)) & 1]


def test_brute_force_minimum_subset_exact_sums():
    """D = 8, small-integer saliencies (every fp32 sum exact, so order is
    irrelevant): the kept set is a smallest subset whose sum reaches p of the
    total, and of the smallest ones the first in (saliency desc, channel asc)
    order."""
    rng = np.random.default_rng(11)
    D = 8
    for trial in range(300):
        k = rng.integers(0, 6, size=(1, 1, D)).astype(np.float32)
        k *= rng.choice([-1.0, 1.0], size=k.shape).astype(np.float32)
        qn = np.ones((1, D), np.float32)
        p = float(rng.choice([0.25, 0.5, 0.75, 0.875, 1.0]))
        m, v, st = oracle.prune_topp(k, qn, p, D)
        w = np.abs(k[0, 0]).astype(np.int64)
        total = int(w.sum())
        target = p * total  # exact in binary for these p
        best = None
        for size in range(D + 1):
            cands = [c for c in itertools.combinations(range(D), size) if w[list(c)].sum() >= target]
            if cands:
                # the greedy-order-first subset of that size: compare the
                # (saliency desc, channel asc) rank lists lexicographically
                rank = {j: r for r, j in enumerate(sorted(range(D), key=lambda j: (-w[j], j)))}
                best = min(cands, key=lambda c: sorted(rank[j] for j in c))
                break
        assert _kept(m[0, 0], D) == sorted(best), (trial, w, p)


def test_closed_forms():
    rng = np.random.default_rng(3)
    D, S = 128, 6
    k = (rng.integers(-7, 8, size=(2, S, D))).astype(np.float32)
    qn = np.ones((2, D), np.float32)
    # p = 0: the empty prefix already reaches 0
    m, v, st = oracle.prune_topp(k, qn, 0.0, D)
    assert not m.any() and not v.any()
    assert np.all(st[:, 0] == S * D)
    # p = 1 on integer saliencies (exact sums): exactly the nonzero channels
    m, v, st = oracle.prune_topp(k, qn, 1.0, D)
    for b in range(2):
        for t in range(S):
            assert _kept(m[b, t], D) == [j for j in range(D) if k[b, t, j] != 0]
    # an all-zero token keeps nothing, whatever p
    z = np.zeros((1, 2, D), np.float32)
    m, v, st = oracle.prune_topp(z, np.ones((1, D), np.float32), 0.99, D)
    assert not m.any() and st[0, 0] == 2 * D and st[0, 3] == 0.0


def test_cumulative_sums_are_exact():
    """Hand-built tokens whose exact cumulative saliency an fp32 running sum
    would lose: the kept count follows the exact sums."""
    D = 128
    qn = np.ones((1, D), np.float32)
    # (a) a 1.0 and 63 saliencies of 2^-25 (channels 1..63).  Exactly, the
    # total is 1 + 63 * 2^-25 and with p = 1 every one of the 64 nonzero
    # channels is needed; an fp32 running sum from 1.0 loses every 2^-25 term
    # (half an ulp of 1 is 2^-24) and would keep one channel.
    k = np.zeros((1, 1, D), np.float32)
    k[0, 0, 0] = 1.0
    k[0, 0, 1:64] = 2.0 ** -25
    m, v, st = oracle.prune_topp(k, qn, 1.0, D)
    assert _kept(m[0, 0], D) == list(range(64))
    # (b) 1.0 in channel 0, 2^-24 in channels 64 and 96: the exact total
    # 1 + 2^-23 needs all three; the two equal saliencies go in channel order
    k = np.zeros((1, 1, D), np.float32)
    k[0, 0, 0] = 1.0
    k[0, 0, 64] = 2.0 ** -24
    k[0, 0, 96] = 2.0 ** -24
    m, v, st = oracle.prune_topp(k, qn, 1.0, D)
    assert _kept(m[0, 0], D) == [0, 64, 96]
    # (c) p = 0.75 with saliencies 4, 1, 1, 1, 1 (total 8, target 6): the
    # prefix {4, 1, 1} reaches 6 exactly (>= counts equality); the three
    # equal ones taken in channel order
    k = np.zeros((1, 1, D), np.float32)
    k[0, 0, [3, 10, 20, 30, 40]] = [1.0, 4.0, 1.0, 1.0, 1.0]
    m, v, st = oracle.prune_topp(k, qn, 0.75, D)
    assert _kept(m[0, 0], D) == [3, 10, 20]


def test_capacity_cut_equals_top_T():
    """Tokens whose prefix is longer than Tcap keep exactly the top-Tcap set
    of plain SparK pruning (a separate oracle routine)."""
    rng = np.random.default_rng(5)
    BH, S, D, Tcap = 2, 64, 128, 40
    k = rng.standard_normal((BH, S, D)).astype(np.float32)
    qn = np.abs(rng.standard_normal((BH, D))).astype(np.float32)
    m_full, _, _ = oracle.prune_topp(k, qn, 0.99, D)
    m_cap, v_cap, _ = oracle.prune_topp(k, qn, 0.99, Tcap)
    m_top, v_top, _ = oracle.prune(k, qn, Tcap)
    n_cut = 0
    for b in range(BH):
        for t in range(S):
            if _popc(m_full[b, t]) > Tcap:
                n_cut += 1
                assert np.array_equal(m_cap[b, t], m_top[b, t])
                assert np.array_equal(v_cap[b, t], v_top[b, t])
            else:
                assert np.array_equal(m_cap[b, t], m_full[b, t])
    assert n_cut > 0


def _exact(w, idx):
    """Exact rational sum of the fp32 values w[idx]."""
    from fractions import Fraction
    return sum((Fraction(float(w[j])) for j in idx), Fraction(0))


def test_invariants_lognormal_tokens():
    """Random tokens shaped like the workloads (per-channel log-normal
    scales): the kept set is a greedy prefix, its mass reaches the target and
    one channel less does not; values and statistics follow the mask."""
    rng = np.random.default_rng(9)
    BH, S, D, p = 2, 48, 128, 0.99
    scale = np.exp(rng.standard_normal((BH, 1, D))).astype(np.float32)
    k = (rng.standard_normal((BH, S, D)).astype(np.float32) * scale).astype(np.float32)
    qn = np.abs(rng.standard_normal((BH, D))).astype(np.float32) * 3
    m, v, st = oracle.prune_topp(k, qn, p, D)
    counts = []
    for b in range(BH):
        sw = 0.0
        for t in range(S):
            w = (qn[b] * np.abs(k[b, t])).astype(np.float32)
            order = sorted(range(D), key=lambda j: (-float(w[j]), j))
            kept = _kept(m[b, t], D)
            n = len(kept)
            counts.append(n)
            assert sorted(order[:n]) == kept
            # with exact sums: the prefix reaches p of the total and one
            # channel less does not (the fp64 sums of the oracle agree with
            # the exact ones away from 1e-12 relative near-ties, none here)
            from fractions import Fraction
            target = Fraction(float(np.float32(p))) * _exact(w, range(D))
            assert _exact(w, order[:n]) >= target
            if n > 0:
                assert _exact(w, order[:n - 1]) < target
            assert np.array_equal(v[b, t, :n].view(np.uint32), k[b, t, kept].view(np.uint32))
            assert not v[b, t, n:].any()
            sw += float(np.sum(w.astype(np.float64)[[j for j in range(D) if j not in kept]]))
        assert st[b, 0] == sum(D - c for c in counts[b * S:(b + 1) * S])
        assert st[b, 1] == pytest.approx(sw, rel=1e-12)
    # the data are not degenerate: counts vary and stay well inside (0, D)
    assert 10 < np.mean(counts) < 120 and len(set(counts)) > 5
