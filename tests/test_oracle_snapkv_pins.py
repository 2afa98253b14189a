"""Pins for the SnapKV-style eviction pre-pass of the oracle (readings R11-R13:
the pages name SnapKV as the base SparK stacks on but give no detail of it).
Checked against torch's fp64 softmax (library special case), closed forms for
the pooling and the selection, and the identity at keep = S."""
import numpy as np
import pytest
import torch

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _scores_torch(q_obs, k, G, W):
    """Summed causal window-attention probabilities on prefix tokens, with
    torch.softmax in fp64."""
    BHG, W_, D = q_obs.shape
    BH, S, _ = k.shape
    P = S - W
    q = torch.from_numpy(q_obs.astype(np.float64)).view(BH, G * W, D)
    kk = torch.from_numpy(k.astype(np.float64))
    logits = q @ kk.transpose(1, 2) / np.sqrt(D)                 # [BH, G*W, S]
    pos = torch.arange(W).repeat(G) + P                          # row -> position
    causal = torch.arange(S)[None, :] <= pos[:, None]
    logits = logits.masked_fill(~causal[None], float("-inf"))
    probs = torch.softmax(logits, dim=-1)
    return probs[:, :, :P].sum(1).numpy()


def test_scores_match_torch_softmax():
    rng = _rng(1)
    BH, G, W, S, D = 2, 4, 8, 70, 128
    q = (rng.standard_normal((BH * G, W, D)) * 0.3).astype(np.float32)
    k = rng.standard_normal((BH, S, D)).astype(np.float32)
    got = oracle.snapkv_scores(q, k, G)
    want = _scores_torch(q, k, G, W)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-13)


def test_scores_mass_bound():
    # every row's probabilities sum to 1, so the prefix mass is < G*W
    rng = _rng(2)
    BH, G, W, S = 1, 4, 16, 100
    q = rng.standard_normal((BH * G, W, 128)).astype(np.float32)
    k = rng.standard_normal((BH, S, 128)).astype(np.float32)
    sc = oracle.snapkv_scores(q, k, G)
    assert np.all(sc >= 0) and sc.sum() < G * W


def test_uniform_keys_give_closed_form_scores():
    # identical keys: row p attends uniformly over p+1 keys, so a prefix
    # token's score is sum_{g,w} 1/(P+w+1)
    BH, G, W, S = 1, 2, 4, 20
    P = S - W
    q = np.ones((BH * G, W, 128), np.float32)
    k = np.ones((BH, S, 128), np.float32)
    sc = oracle.snapkv_scores(q, k, G)
    want = G * sum(1.0 / (P + w + 1) for w in range(W))
    np.testing.assert_allclose(sc, want, rtol=1e-13)


def test_pool_closed_form():
    s = np.zeros((1, 20))
    s[0, 10] = 5.0
    s[0, 0] = 2.0
    p = oracle.snapkv_pool(s, 7)
    want = np.zeros(20)
    want[7:14] = 5.0
    want[0:4] = 2.0
    assert np.array_equal(p[0], want)
    assert np.array_equal(oracle.snapkv_pool(s, 1), s)


def test_select_identity_and_order():
    rng = _rng(3)
    BH, S, W = 2, 50, 8
    pooled = rng.random((BH, S - W))
    idx = oracle.snapkv_select(pooled, S, W, S)
    assert np.array_equal(idx, np.tile(np.arange(S), (BH, 1)))
    idx = oracle.snapkv_select(pooled, S, W, 20)
    for b in range(BH):
        top = np.argsort(-pooled[b], kind="stable")[:12]
        assert np.array_equal(idx[b, :12], np.sort(top))
        assert np.array_equal(idx[b, 12:], np.arange(S - W, S))


def test_select_ties_go_to_lower_index():
    pooled = np.full((1, 30), 0.25)
    pooled[0, 17] = 1.0
    idx = oracle.snapkv_select(pooled, 38, 8, 13)
    assert np.array_equal(idx[0], np.array([0, 1, 2, 3, 17] + list(range(30, 38))))
