"""Pins of the oracle's V-channel pruning (reading R16: top-T_v value channels
by |v| per token, pruned value entries recovered as 0), against numpy
restatements, closed forms and special cases."""
import numpy as np
import pytest

import oracle

D = 128


def _np_topk_mask(x, T):
    # stable order: larger |x| first, lower channel first on ties
    order = np.lexsort((np.arange(x.shape[-1]), -np.abs(x)))
    keep = np.zeros(x.shape[-1], bool)
    keep[order[:T]] = True
    return keep


@pytest.mark.parametrize("Tv", [0, 1, 13, 64, 100, 128])
def test_value_mask_is_top_tv_by_magnitude(Tv):
    rng = np.random.default_rng(Tv + 1)
    v = rng.integers(-4, 5, (2, 40, D)).astype(np.float32)  # many magnitude ties
    vm, vv, _ = oracle.prune_values(v, Tv)
    bits = ((vm[..., None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(2, 40, D).astype(bool)
    for b in range(2):
        for t in range(40):
            assert np.array_equal(bits[b, t], _np_topk_mask(v[b, t], Tv))
            assert np.array_equal(vv[b, t], v[b, t][bits[b, t]])


def test_recovered_values_are_kept_or_zero():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((1, 30, D)).astype(np.float32)
    vm, vv, _ = oracle.prune_values(v, 50)
    vh = oracle.recover_values(vm, vv, 0)
    keep = np.stack([_np_topk_mask(v[0, t], 50) for t in range(30)])
    assert np.array_equal(vh[keep], v[0][keep].astype(np.float64))
    assert np.all(vh[~keep] == 0.0)
    assert np.all(np.abs(v[0])[keep].reshape(30, 50).min(1) >= np.abs(np.where(keep, 0, v[0])).max(1))


def _case(seed, S=57, G=2, BH=2):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((BH, S, D)).astype(np.float32)
    v = rng.standard_normal((BH, S, D)).astype(np.float32)
    qo = rng.standard_normal((BH * G, 8, D)).astype(np.float32)
    q = rng.standard_normal((BH * G, D)).astype(np.float32)
    return k, v, qo, q


def test_full_value_budget_is_plain_decode():
    k, v, qo, q = _case(3)
    qn = oracle.qnorm(qo, 2)
    m, vals, st = oracle.prune(k, qn, 26)
    vm, vv, _ = oracle.prune_values(v, D)
    a = oracle.decode(q, m, vals, qn, st, v, G=2)
    b = oracle.decode_kv(q, m, vals, qn, st, vm, vv, G=2)
    assert np.array_equal(a, b)


def test_zero_value_budget_gives_zero_output():
    k, v, qo, q = _case(4)
    qn = oracle.qnorm(qo, 2)
    m, vals, st = oracle.prune(k, qn, 64)
    vm, vv, _ = oracle.prune_values(v, 0)
    assert np.all(oracle.decode_kv(q, m, vals, qn, st, vm, vv, G=2) == 0.0)


def test_closed_form_with_unpruned_keys():
    # T = D for the keys: the scores are exact dot products, so the output is
    # softmax(q K^T / sqrt(D)) @ V^ with V^ the numpy top-T_v masking of V
    k, v, qo, q = _case(5, S=33, G=2, BH=1)
    qn = oracle.qnorm(qo, 2)
    m, vals, st = oracle.prune(k, qn, D)
    Tv = 40
    vm, vv, _ = oracle.prune_values(v, Tv)
    got = oracle.decode_kv(q, m, vals, qn, st, vm, vv, G=2)
    vhat = np.stack([np.where(_np_topk_mask(v[0, t], Tv), v[0, t], 0.0) for t in range(33)]).astype(np.float64)
    for g in range(2):
        s = k[0].astype(np.float64) @ q[g].astype(np.float64) / np.sqrt(D)
        p = np.exp(s - s.max())
        p /= p.sum()
        np.testing.assert_allclose(got[g], (p @ vhat).astype(np.float32), rtol=1e-6, atol=1e-7)


def test_value_scale_equivariance():
    k, v, qo, q = _case(6)
    qn = oracle.qnorm(qo, 2)
    m, vals, st = oracle.prune(k, qn, 26)
    vm, vv, _ = oracle.prune_values(v, 64)
    vm2, vv2, _ = oracle.prune_values(2.0 * v, 64)
    assert np.array_equal(vm, vm2)
    a = oracle.decode_kv(q, m, vals, qn, st, vm, vv, G=2)
    b = oracle.decode_kv(q, m, vals, qn, st, vm2, vv2, G=2)
    assert np.array_equal(2.0 * a, b)
