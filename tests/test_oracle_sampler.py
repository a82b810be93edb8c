"""Pins for the sampler pieces of the oracle (Euler step, CFG combine, shifted sigma schedule)."""
import math

import numpy as np
import pytest

from oracle import krea2_oracle as O


def test_shift_mu_endpoints_and_1024sq():
    # the pages' shift parameters: 0.5 at 256 image tokens, 1.15 at 6400
    assert abs(O.shift_mu(256) - 0.5) < 1e-15
    assert abs(O.shift_mu(6400) - 1.15) < 1e-15
    # 1024^2 -> 64 x 64 = 4096 tokens: 0.5 + 0.65 * 3840 / 6144
    assert abs(O.shift_mu(4096) - (0.5 + 0.65 * 3840 / 6144)) < 1e-15


def test_shifted_sigmas_properties():
    for steps, mu in ((28, O.shift_mu(4096)), (8, 1.15)):
        s = O.shifted_sigmas(steps, mu)
        assert s.shape == (steps + 1,)
        assert s[0] == 1.0 and s[-1] == 0.0          # the shift keeps sigma = 1 fixed
        assert np.all(np.diff(s) < 0)                # strictly decreasing
        assert np.all(s[:-1] >= np.linspace(1, 1 / steps, steps) - 1e-15)  # mu > 0 shifts towards noise
    # mu = 0 is no shift at all
    np.testing.assert_allclose(O.shifted_sigmas(10, 0.0)[:-1], np.linspace(1, 0.1, 10), rtol=1e-14)
    # hand value: sigma = 0.5, mu = ln 3 -> 3 / (3 + 1) = 0.75
    s = O.shifted_sigmas(2, math.log(3.0))
    assert abs(s[1] - 0.75) < 1e-15


def test_cfg_combine():
    rng = np.random.default_rng(0)
    c, u = rng.standard_normal((2, 3, 5))
    np.testing.assert_array_equal(O.cfg_combine(c, u, 0.0), c)   # guidance off
    np.testing.assert_allclose(O.cfg_combine(c, u, 4.5), 5.5 * c - 4.5 * u, rtol=1e-14)
    np.testing.assert_array_equal(O.cfg_combine(c, c, 4.5), c)    # identical branches


def test_euler_integrates_a_straight_path_exactly():
    # a constant velocity field (flow matching's straight path x_sigma = x0 + sigma * v) is
    # integrated exactly from sigma = 1 to 0 by the Euler steps, whatever the schedule
    rng = np.random.default_rng(1)
    x0, v = rng.standard_normal((2, 4, 7))
    s = O.shifted_sigmas(28, O.shift_mu(4096))
    x = x0 + v
    for i in range(28):
        x = O.euler_step(x, v, s[i], s[i + 1])
    np.testing.assert_allclose(x, x0, rtol=1e-12, atol=1e-12)
