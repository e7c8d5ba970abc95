"""Pins of the oracle's sampling step (oracle/sampling.py) against the page's
worked example and against closed forms: "The Mathematics of Karpathy's
nanochat", §Inference: Generating Text, §Sampling Controls."""
import math

import numpy as np
import pytest

from decoder_only_transformer_fwd_b200 import synth
from oracle import sampling as S

from golden_io import load


def test_worked_example_greedy():
    g = load("sampling_example.txt")
    assert S.sample_next(np.array(g["logits"]), 0.0, None, 0.7) == g["greedy"]
    # top-1 leaves only the greedy token, whatever the temperature and u
    for tau in (0.8, 1.0, 3.0):
        for u in (0.0, 0.5, 0.999):
            assert S.sample_next(np.array(g["logits"]), tau, 1, u) == g["greedy"]


def test_greedy_takes_first_of_equal_maxima():
    z = np.zeros(50)
    z[17] = z[42] = 5.0
    assert S.greedy(z) == 17
    assert S.sample_next(z, 0.0, 3, 0.99) == 17


def test_uniform_logits_draw_floor_u_v():
    # equal weights: the cumulative probability of index i is (i + 1) / V
    V = 10
    z = np.full(V, 2.5)
    for j in range(V):
        assert S.sample_next(z, 1.0, None, (j + 0.5) / V) == j
    assert S.sample_next(z, 0.7, None, 0.0) == 0
    assert S.sample_next(z, 0.7, None, 0.999) == V - 1


@pytest.mark.parametrize("tau", [0.5, 1.0, 2.0])
def test_two_point_distribution(tau):
    # z1 - z0 = tau ln 3 gives P = (1/4, 3/4)
    z = np.array([0.0, tau * math.log(3.0)])
    assert S.sample_next(z, tau, None, 0.2) == 0
    assert S.sample_next(z, tau, None, 0.3) == 1
    lo, hi = S.draw_interval(z, tau, None, 0)
    assert abs(lo) < 1e-15 and abs(hi - 0.25) < 1e-12


def test_top_k_keeps_every_tie_at_the_threshold():
    z = np.array([1.0, 3.0, 3.0, 2.0, 3.0])
    # the 2nd largest value is 3 (ties counted): indices 1, 2, 4 survive with equal weight
    assert S.sample_next(z, 1.0, 2, 0.2) == 1
    assert S.sample_next(z, 1.0, 2, 0.5) == 2
    assert S.sample_next(z, 1.0, 2, 0.9) == 4
    kept = np.isfinite(S.top_k_filter(z, 2))
    assert kept.tolist() == [False, True, True, False, True]
    # k = 4: threshold 2, index 0 dropped
    assert np.isfinite(S.top_k_filter(z, 4)).tolist() == [False, True, True, True, True]
    # k >= V and k = 0 keep everything
    assert np.isfinite(S.top_k_filter(z, 5)).all() and np.isfinite(S.top_k_filter(z, 0)).all()


def test_top3_closed_form():
    # z = 5..1, tau = 1, k = 3: P = (1, e^-1, e^-2) / (1 + e^-1 + e^-2)
    z = np.array([5.0, 4.0, 3.0, 2.0, 1.0])
    d = 1 + math.exp(-1) + math.exp(-2)
    c0, c1 = 1 / d, (1 + math.exp(-1)) / d      # 0.66524, 0.90997
    assert S.sample_next(z, 1.0, 3, c0 - 1e-3) == 0
    assert S.sample_next(z, 1.0, 3, c0 + 1e-3) == 1
    assert S.sample_next(z, 1.0, 3, c1 - 1e-3) == 1
    assert S.sample_next(z, 1.0, 3, c1 + 1e-3) == 2
    assert S.sample_next(z, 1.0, 3, 0.99999) == 2


def test_temperature_frequencies_follow_exp_z_over_tau():
    z = np.array([0.0, 1.0, 2.0])
    tau = 2.0
    n = 30000
    counts = np.zeros(3)
    for j in range(n):
        counts[S.sample_next(z, tau, None, (j + 0.5) / n)] += 1
    w = np.array([1.0, math.exp(0.5), math.exp(1.0)])
    assert np.max(np.abs(counts / n - w / w.sum())) <= 2.0 / n


def test_temperature_limits():
    z = synth.sampling_logits(5, 1, 300)[0].astype(np.float64)
    top = 123
    z[top] = np.max(z) + 1.0
    # tau -> 0 concentrates on the argmax (the others weigh exp(-1000) = 0 in
    # fp64); tau -> inf flattens to uniform
    for u in (0.0, 0.4, 0.9999):
        assert S.sample_next(z, 1e-3, None, u) == top
    p = S.probabilities(z, 1e6, None)
    assert np.max(np.abs(p - 1.0 / 300)) < 1e-6


def test_seeded_rows_draws_stay_in_their_interval():
    z = synth.sampling_logits(9, 4, 2000, ties=5).astype(np.float64)
    u = synth.uniforms(9, 4)
    for b in range(4):
        for tau, k in ((0.8, 50), (1.0, 0), (1.3, 5)):
            v = S.sample_next(z[b], tau, k, float(u[b]))
            lo, hi = S.draw_interval(z[b], tau, k, v)
            assert lo <= u[b] < hi
            assert np.isfinite(S.top_k_filter(z[b], k)[v])
