"""Pins of the oracle's head backward (oracle/head_backward.py): central finite
differences of its own loss, and properties the pages fix ("The Mathematics
of Karpathy's nanochat", §Logit Softcap: the derivative vanishes for
saturated logits; §RMS Normalization: the norm is scale-invariant;
§Cross-Entropy Loss: the mean over valid targets)."""
import numpy as np
import pytest

from oracle import head_backward as HB


def _case(seed, M=5, C=8, V=11, scale=1.0):
    g = np.random.default_rng(seed)
    x = g.standard_normal((M, C)) * 1.7
    w = g.standard_normal((V, C)) * scale
    y = g.integers(0, V, size=M)
    y[1] = -1
    return x, w, y


@pytest.mark.parametrize("seed,scale", [(0, 1.0), (1, 4.0), (2, 0.3)])
def test_gradients_match_central_differences(seed, scale):
    x, w, y = _case(seed, scale=scale)
    dx, dw, loss = HB.head_backward(x, w, y)
    assert abs(loss - HB.head_forward(x, w, y)) < 1e-14
    h = 1e-6
    for (i, j) in [(0, 0), (2, 5), (4, 7), (1, 3)]:
        xp, xm = x.copy(), x.copy()
        xp[i, j] += h
        xm[i, j] -= h
        fd = (HB.head_forward(xp, w, y) - HB.head_forward(xm, w, y)) / (2 * h)
        assert abs(fd - dx[i, j]) < 1e-8 * max(1.0, abs(fd)), (i, j, fd, dx[i, j])
    for (v, j) in [(0, 0), (y[0], 2), (10, 7), (y[3], 5)]:
        wp, wm = w.copy(), w.copy()
        wp[v, j] += h
        wm[v, j] -= h
        fd = (HB.head_forward(x, wp, y) - HB.head_forward(x, wm, y)) / (2 * h)
        assert abs(fd - dw[v, j]) < 1e-8 * max(1.0, abs(fd)), (v, j, fd, dw[v, j])


def test_ignored_rows_get_no_gradient_and_mean_is_over_valid_rows():
    x, w, y = _case(3)
    dx, dw, loss = HB.head_backward(x, w, y)
    assert np.all(dx[1] == 0.0)
    # the same rows without the ignored one: same loss, same gradients
    keep = y >= 0
    dx2, dw2, loss2 = HB.head_backward(x[keep], w, y[keep])
    assert abs(loss - loss2) < 1e-14
    assert np.allclose(dx[keep], dx2, atol=1e-15) and np.allclose(dw, dw2, atol=1e-15)
    # no valid target: NaN loss, zero gradients
    dx3, dw3, loss3 = HB.head_backward(x, w, np.full(len(y), -1))
    assert np.isnan(loss3) and not dx3.any() and not dw3.any()


def test_saturated_logits_stop_the_gradient():
    # |z| >> c: tanh saturates and d zhat / d z -> 0, so no gradient reaches
    # x or W_U (the page's "implicit gradient clipping")
    x, w, y = _case(4, scale=1e4)
    dx, dw, _ = HB.head_backward(x, w, y)
    assert np.max(np.abs(dx)) < 1e-12 and np.max(np.abs(dw)) < 1e-12


def test_norm_scale_invariance_makes_dx_orthogonal_to_x():
    # with eps = 0, RMSNorm(a x) = RMSNorm(x) for a > 0, so dL/dx . x = 0 per row
    x, w, y = _case(5)
    dx, _, _ = HB.head_backward(x, w, y, eps=0.0)
    assert np.max(np.abs(np.sum(dx * x, axis=-1))) < 1e-14 * np.max(np.abs(dx)) * 10 + 1e-16


def test_logit_gradient_rows_sum_to_zero():
    # sum over v of (softmax - one-hot) = 0; with the softcap inactive (tiny
    # logits, tanh' ~ 1), sum_v dW_U[v] = sum_t (sum_v dz_tv) xn_t ~ 0
    # (at W_U ~ 1e-7 the tanh^2 term is ~1e-16; at 1e-4 it would be ~1e-9)
    x, w, y = _case(6, scale=1e-7)
    _, dw, _ = HB.head_backward(x, w, y)
    assert np.max(np.abs(dw.sum(axis=0))) < 1e-12 * np.max(np.abs(dw))
