"""Pins of the oracle's online temperature calibration (host only).

- the update is one step along the exact derivative of the negative
  log-likelihood of the round's outcomes (checked by finite differences of a
  likelihood written out here term by term);
- its fixed point: outcomes for which that derivative vanishes leave T_j as
  it is, and positions nobody reached keep theirs;
- its direction: over-confident positions (predicted survival above the
  observed) get a higher temperature, under-confident ones a lower one;
- repeated rounds whose outcomes are drawn from a logistic model with a known
  temperature T* move the temperatures to T*;
- which observations count: only requests that reached and verified j.
"""
import math

import numpy as np
import pytest
import scipy.optimize
import scipy.special

import oracle


def _nll(theta, c, y):
    tot = 0.0
    for ci, yi in zip(c, y):
        p = 1.0 / (1.0 + math.exp(-ci * theta))
        tot -= yi * math.log(p) + (1 - yi) * math.log(1.0 - p)
    return tot


def test_step_is_the_likelihood_gradient():
    rng = np.random.default_rng(1)
    B, K = 40, 5
    conf = rng.normal(1.0, 1.5, size=(B, K))
    temps = 1 + 0.1 * np.arange(1, K + 1)
    L = rng.integers(0, K + 1, size=B)
    acc = np.minimum(rng.integers(0, K + 1, size=B), L)
    eta = 0.05
    new = oracle.calibrate(conf, temps, L, acc, eta, 1e-3, 1e3)
    for j in range(1, K + 1):
        reached = [b for b in range(B) if acc[b] >= j - 1 and L[b] >= j]
        if not reached:
            assert new[j - 1] == temps[j - 1]
            continue
        c = [conf[b, j - 1] for b in reached]
        y = [1.0 if acc[b] >= j else 0.0 for b in reached]
        th = 1.0 / temps[j - 1]
        h = 1e-6
        grad = (_nll(th + h, c, y) - _nll(th - h, c, y)) / (2 * h) / len(reached)
        assert abs(1.0 / new[j - 1] - (th - eta * grad)) < 1e-8


def test_fixed_point_and_unreached_positions():
    # at theta = 1, an accepted observation with c = 1 contributes
    # sigmoid(1) - 1 to the gradient and a rejected one with c = x contributes
    # x sigmoid(x); choosing x with x sigmoid(x) = 1 - sigmoid(1) makes the
    # gradient vanish, so T_1 = 1 must not move
    x = scipy.optimize.brentq(lambda v: v * scipy.special.expit(v) - (1.0 - scipy.special.expit(1.0)), 0.0, 2.0)
    conf = np.array([[1.0, 0.3], [x, 0.7]])
    temps = np.array([1.0, 1.3])
    L = np.array([1, 1])            # position 2 is verified by nobody
    acc = np.array([1, 0])
    new = oracle.calibrate(conf, temps, L, acc, 0.5, 1e-3, 1e3)
    assert abs(new[0] - 1.0) < 1e-12
    assert new[1] == 1.3


def test_direction_over_and_under_confident():
    conf = np.full((20, 1), 2.0)
    temps = np.array([1.0])
    L = np.ones(20, np.int64)
    over = oracle.calibrate(conf, temps, L, np.zeros(20, np.int64), 0.1, 1e-3, 1e3)   # all rejected
    under = oracle.calibrate(conf, temps, L, np.ones(20, np.int64), 0.1, 1e-3, 1e3)   # all accepted
    assert over[0] > 1.0 > under[0]


def test_clamp():
    conf = np.full((4, 1), 3.0)
    new = oracle.calibrate(conf, np.array([1.0]), np.ones(4, np.int64), np.zeros(4, np.int64), 100.0, 0.5, 4.0)
    assert new[0] == 4.0
    new = oracle.calibrate(conf, np.array([1.0]), np.ones(4, np.int64), np.ones(4, np.int64), 100.0, 0.5, 4.0)
    assert new[0] == 0.5


def test_converges_to_the_generating_temperature():
    rng = np.random.default_rng(7)
    B, K = 256, 3
    t_true = np.array([0.6, 1.8, 3.0])
    temps = np.ones(K)
    late = []
    for it in range(1000):
        conf = rng.normal(1.0, 2.0, size=(B, K))
        L = np.full(B, K)
        # outcomes: position j survives with sigmoid(c / T*_j) given the earlier ones did
        u = rng.random(size=(B, K))
        surv = u < 1.0 / (1.0 + np.exp(-conf / t_true))
        acc = np.array([int(np.argmin(np.append(s, False))) for s in surv])
        temps = oracle.calibrate(conf, temps, L, acc, 0.5, 0.05, 20.0)
        if it >= 400:
            late.append(temps)
    # the steps are noisy (one round's outcomes each); their average settles at T*
    mean = np.mean(late, axis=0)
    assert np.all(np.abs(mean - t_true) / t_true < 0.08), mean


def test_only_reached_and_verified_requests_count():
    # request 0 rejected position 1: it never reached position 2, so its
    # confidence there must not move T_2 (however extreme it is)
    conf = np.array([[1.0, 50.0], [1.0, 1.0]])
    temps = np.array([1.0, 1.0])
    L = np.array([2, 2])
    a = oracle.calibrate(conf, temps, L, np.array([0, 2]), 0.1, 1e-3, 1e3)
    conf2 = conf.copy()
    conf2[0, 1] = -50.0
    b = oracle.calibrate(conf2, temps, L, np.array([0, 2]), 0.1, 1e-3, 1e3)
    assert a[1] == b[1]
    # a request with L_b = 1 never verified position 2
    c = oracle.calibrate(conf, temps, np.array([1, 2]), np.array([1, 2]), 0.1, 1e-3, 1e3)
    d = oracle.calibrate(conf2, temps, np.array([1, 2]), np.array([1, 2]), 0.1, 1e-3, 1e3)
    assert c[1] == d[1]
