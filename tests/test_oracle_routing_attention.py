"""Pins of the oracle's pass-2 routing attention (oracle/routing_attention.py)
against the separately pinned plain attention of the base model and the
identity the "looped nanochat" card states: the additive logit prior equals
ordinary attention on augmented-width queries and keys."""
import math

import numpy as np
import pytest

from oracle import nanochat_fwd as O
from oracle import routing_attention as R


def _inputs(seed, T=20, H=4, Hkv=2, D=16):
    g = np.random.default_rng(seed)
    f = lambda h: g.standard_normal((T, h, D))
    return f(H), f(Hkv), f(Hkv), f(H), f(Hkv)


def test_softplus():
    assert R.softplus(0.0) == pytest.approx(math.log(2.0), abs=1e-15)
    assert R.softplus(50.0) == pytest.approx(50.0, abs=1e-15)
    assert R.softplus(-50.0) == pytest.approx(math.exp(-50.0), rel=1e-12)
    assert R.softplus(800.0) == 800.0          # no overflow


@pytest.mark.parametrize("window", [20, 7, 1])
def test_closed_gate_is_the_base_attention(window):
    # g = softplus(-inf) = 0: the prior vanishes
    q2, k2, v2, q1, k1 = _inputs(1)
    got = R.routing_attention(q2, k2, v2, q1, k1, -800.0, window)
    ref = O.attention(q2, k2, v2, window, 16 ** -0.5)
    assert np.max(np.abs(got - ref)) < 1e-13


@pytest.mark.parametrize("gate_logit,window", [(0.0, 20), (1.7, 7), (-2.3, 3)])
def test_prior_equals_augmented_width_attention(gate_logit, window):
    # [q2, g q1] . [k2, k1] = q2.k2 + g q1.k1 at width 2D, same 1/sqrt(D) scale
    q2, k2, v2, q1, k1 = _inputs(2)
    g = R.softplus(gate_logit)
    qa = np.concatenate([q2, g * q1], axis=-1)
    ka = np.concatenate([k2, k1], axis=-1)
    va = np.concatenate([v2, np.zeros_like(v2)], axis=-1)   # output width of the plain oracle = q width
    ref = O.attention(qa, ka, va, window, 16 ** -0.5)[..., :16]
    got = R.routing_attention(q2, k2, v2, q1, k1, gate_logit, window)
    assert np.max(np.abs(got - ref)) < 1e-13


def test_prior_alone_when_pass2_features_vanish():
    # q2 = 0: the logits are g q1.k1 / sqrt(D), i.e. the base attention on
    # (sqrt(g) q1, sqrt(g) k1)
    q2, k2, v2, q1, k1 = _inputs(3)
    g = R.softplus(0.9)
    got = R.routing_attention(np.zeros_like(q2), k2, v2, q1, k1, 0.9, 20)
    ref = O.attention(math.sqrt(g) * q1, math.sqrt(g) * k1, v2, 20, 16 ** -0.5)
    assert np.max(np.abs(got - ref)) < 1e-13
