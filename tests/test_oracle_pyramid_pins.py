"""Pins for the oracle's PyramidKV layer budgets (reading R20: the budget of
layer l of L falls linearly with depth around the mean budget M, from
M (1 + beta) at the first layer to M (1 - beta) at the last, rounded half away
from zero, clamped to [W, S]).

Source: "KV Cache 还能再砍一刀：SparK ..." sections 4.1 and 4.2 (SparK stacked
on PyramidKV, a layer-wise eviction budget; the pages give no schedule).  The
pins are closed forms at chosen shapes, the symmetry around the mean that the
linear reading implies (so the budgets of all layers sum to L * M exactly),
monotonicity, the clamp, and the C library's own copy of the rule."""
import pytest

import oracle
from channel_pruned_decode_b200 import binding as B


def test_closed_forms():
    # 32 layers around a mean of 2048 with beta = 1/2: 3072 down to 1024 in
    # steps of 2048 / 31 (rounded)
    k = oracle.pyramid_keep(32, 2048, 0.5, 32, 8192)
    assert k[0] == 3072 and k[31] == 1024 and k[15] == 2081 and k[16] == 2015
    # two layers: M (1 + beta), M (1 - beta); three: the middle one keeps M
    assert oracle.pyramid_keep(2, 100, 0.25, 1, 1000) == [125, 75]
    assert oracle.pyramid_keep(3, 100, 0.25, 1, 1000) == [125, 100, 75]
    # four layers, fractions 1, 1/3, -1/3, -1: 150, 116.67, 83.33, 50
    assert oracle.pyramid_keep(4, 100, 0.5, 1, 1000) == [150, 117, 83, 50]
    # one layer, or beta = 0: the mean everywhere
    assert oracle.pyramid_keep(1, 321, 0.7, 1, 1000) == [321]
    assert oracle.pyramid_keep(9, 128, 0.0, 32, 4096) == [128] * 9


@pytest.mark.parametrize("L,M,beta", [(32, 2048, 0.5), (24, 128, 0.3), (7, 999, 0.9), (80, 512, 0.125)])
def test_symmetry_sum_and_order(L, M, beta):
    k = oracle.pyramid_keep(L, M, beta, 1, 10 ** 6)
    assert all(k[l] + k[L - 1 - l] == 2 * M for l in range(L))   # rounding is odd-symmetric
    assert sum(k) == L * M
    assert all(a >= b for a, b in zip(k, k[1:]))


def test_clamped_to_window_and_prompt():
    k = oracle.pyramid_keep(8, 100, 0.9, 40, 150)
    assert min(k) == 40 and max(k) == 150
    assert k == sorted(k, reverse=True)


def test_library_copy_matches():
    for L, M, beta, W, S in [(32, 2048, 0.5, 32, 8192), (24, 128, 0.3, 32, 4096), (8, 100, 0.9, 40, 150),
                             (1, 64, 0.5, 32, 64), (5, 77, 0.45, 16, 1000)]:
        assert B.spark_pyramid_keep(L, M, beta, W, S) == oracle.pyramid_keep(L, M, beta, W, S)
