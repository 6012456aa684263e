"""Pins of the oracle's global mixed-precision search (MLSys 2026 talk notes
on MixLLM, notes.yuuk.io, §グローバル混合精度探索 and its Algorithm 1): the
channel salience S_c = mean_d |g_d^T (c_q - c_0) + (g_d^T (c_q - c_0))^2 / 2|
and the global top-T selection.  Each expected value is a closed form on a
constructed channel whose quantization error is known exactly, so a wrong
sign of c_q - c_0, a dropped or mis-scaled second-order term, a missing
absolute value or mean, or the wrong group's scale fails one of them.
"""
import numpy as np
import pytest

import oracle

S_GRID = 2.0 ** -6  # a power of two: the grid values and their scale are exact


def grid_group(rng):
    """128 weights on the 4-bit grid of scale S_GRID and zero point 8: codes
    0 and 15 present, so lo = -8 s, hi = 7 s, (hi - lo) / 15 = s exactly."""
    q = rng.integers(0, 16, 128)
    q[0], q[1] = 0, 15
    return ((q - 8) * S_GRID).astype(np.float32), q


def test_channel_on_the_grid_has_zero_salience():
    rng = np.random.default_rng(0)
    W = np.stack([np.concatenate([grid_group(rng)[0] for _ in range(3)]) for _ in range(2)])
    G = rng.normal(0, 1, (5, 2, W.shape[1])).astype(np.float32)
    assert (oracle.channel_salience(W, G) == 0.0).all()


def test_zero_gradients_give_zero_salience():
    rng = np.random.default_rng(1)
    W = rng.normal(0, 0.02, (3, 256)).astype(np.float32)
    assert (oracle.channel_salience(W, np.zeros((4, 3, 256), np.float32)) == 0.0).all()


@pytest.mark.parametrize("eps", [0.25 * S_GRID, -0.375 * S_GRID, 0.125 * S_GRID])
def test_one_perturbed_weight_closed_form(eps):
    """One interior weight moved by eps (< s/2, so its code and the group's
    range do not change): c_q - c_0 = -eps at that index, 0 elsewhere.  With
    g_d = lam_d * e_j, t_d = -lam_d * eps and S = mean |t + t^2 / 2|."""
    rng = np.random.default_rng(2)
    w, q = grid_group(rng)
    j = 5
    while q[j] in (0, 15):
        j += 1
    w = w.copy()
    w[j] += np.float32(eps)
    lams = np.array([1.0, -2.0, 40.0, -3000.0], np.float64)
    G = np.zeros((lams.size, 1, 128), np.float32)
    G[:, 0, j] = lams.astype(np.float32)
    t = -lams * float(np.float32(eps))  # c_q - c_0 = -eps
    expected = np.mean(np.abs(t + 0.5 * t * t))
    S = oracle.channel_salience(w[None, :], G)
    assert S[0] == pytest.approx(expected, rel=1e-12)
    # the second-order term matters: at lam = -3000 it dominates the first
    assert abs(t[3] + 0.5 * t[3] ** 2) > 2 * abs(t[3])


def test_each_group_uses_its_own_scale_and_the_dot_product_spans_the_row():
    """Two groups with scales s and 4s; a moved weight in each: the error of
    group 1 is its own eps (it is on group 1's grid), and g summing both
    positions gives t = -(eps0 + eps1)."""
    rng = np.random.default_rng(3)
    w0, q0 = grid_group(rng)
    w1, q1 = grid_group(rng)
    w1 = (w1 * 4).astype(np.float32)  # scale 4s, zero point 8
    i0 = next(i for i in range(2, 128) if q0[i] not in (0, 15))
    i1 = next(i for i in range(2, 128) if q1[i] not in (0, 15))
    e0, e1 = np.float32(0.25 * S_GRID), np.float32(-1.5 * S_GRID)  # |e1| < 4s/2
    w = np.concatenate([w0, w1])
    w[i0] += e0
    w[128 + i1] += e1
    G = np.zeros((1, 1, 256), np.float32)
    G[0, 0, i0] = 1.0
    G[0, 0, 128 + i1] = 1.0
    t = -(float(e0) + float(e1))
    assert oracle.channel_salience(w[None, :], G)[0] == pytest.approx(abs(t + 0.5 * t * t), rel=1e-12)


def test_channels_are_independent():
    rng = np.random.default_rng(4)
    W = rng.normal(0, 0.02, (6, 256)).astype(np.float32)
    G = rng.normal(0, 1, (3, 6, 256)).astype(np.float32)
    S = oracle.channel_salience(W, G)
    perm = rng.permutation(6)
    assert np.array_equal(oracle.channel_salience(W[perm], G[:, perm]), S[perm])
    # and duplicating every sample leaves the mean unchanged
    assert np.allclose(oracle.channel_salience(W, np.concatenate([G, G])), S, rtol=1e-14)


def test_top_t_ties_and_bounds():
    S = np.array([3, 1, 3, 2, 3], np.float32)
    assert oracle.select_top_t(S, 2).tolist() == [1, 0, 1, 0, 0]
    assert oracle.select_top_t(S, 4).tolist() == [1, 0, 1, 1, 1]
    assert oracle.select_top_t(S, 0).tolist() == [0] * 5
    assert oracle.select_top_t(S, 5).tolist() == [1] * 5


def test_top_t_selects_the_largest():
    rng = np.random.default_rng(5)
    S = rng.exponential(1.0, 1000).astype(np.float32)
    for T in (1, 100, 999):
        is8 = oracle.select_top_t(S, T).astype(bool)
        assert is8.sum() == T
        assert S[is8].min() >= S[~is8].max()
