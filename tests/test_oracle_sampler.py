"""Pins for the sampler pieces of the oracle (Euler step, CFG combine, shifted sigma schedule)."""
import math

import numpy as np
import pytest

import krea2_inputs as KI
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


# ---- the loop itself (sample_loop) and the backbone wiring of sample

def _point_mass_velocity(targets):
    """Exact flow-matching velocity towards a point mass: on the straight path x_sigma =
    (1 - sigma) a + sigma z the velocity is z - a = (x - a) / sigma, here as a field of x."""
    return lambda x, sigma, branch: (x - targets[branch]) / sigma


def test_loop_lands_on_the_guided_point_mass_exactly():
    # Euler on (x - a) / sigma keeps x_i - a = sigma_i (z - a), whatever the schedule, and lands on a
    # at sigma = 0. With guidance g the combined field is (x - c) / sigma, c = (1 + g) a - g b.
    rng = np.random.default_rng(7)
    z, a, b = rng.standard_normal((3, 5, 4))
    g = 4.5
    for sig in (O.shifted_sigmas(28, O.shift_mu(4096)), O.shifted_sigmas(8, 1.15)):
        out = O.sample_loop(z, sig, g, _point_mass_velocity((a, b)))
        np.testing.assert_allclose(out, (1 + g) * a - g * b, rtol=1e-10, atol=1e-10)
        # negative control: cond and uncond swapped lands elsewhere
        assert np.max(np.abs(out - ((1 + g) * b - g * a))) > 1.0
        # without guidance the unconditional target plays no part
        np.testing.assert_allclose(O.sample_loop(z, sig, 0.0, _point_mass_velocity((a, b))), a,
                                   rtol=1e-10, atol=1e-10)


def test_loop_feeds_step_i_the_timestep_sigma_i():
    # a probe model that returns its timestep: the result is x0 + sum (s[i+1] - s[i]) * s[i];
    # feeding s[i+1] instead would give x0 + sum (s[i+1] - s[i]) * s[i+1]
    sig = O.shifted_sigmas(8, 1.15)
    x0 = np.zeros(3)
    calls = []

    def probe(x, sigma, branch):
        calls.append((sigma, branch))
        return np.full_like(x, sigma)
    out = O.sample_loop(x0, sig, 0.0, probe)
    want = sum((sig[i + 1] - sig[i]) * sig[i] for i in range(8))
    wrong = sum((sig[i + 1] - sig[i]) * sig[i + 1] for i in range(8))
    np.testing.assert_allclose(out, want, rtol=1e-14)
    assert abs(want - wrong) > 0.05
    assert calls == [(sig[i], 0) for i in range(8)]        # no unconditional call without guidance
    calls.clear()
    O.sample_loop(x0, sig, 4.5, probe)
    assert calls == [(sig[i], br) for i in range(8) for br in (0, 1)]


def test_sample_runs_the_conditional_prompt_on_the_guided_branch():
    # one step of the backbone-driven loop written out with the (separately pinned) backbone:
    # x1 = x0 + (s1 - s0) * ((1 + g) v(text_cond) - g v(text_uncond)) at timestep s0
    d = KI.TINY
    T, gh, gw, g = 8, 4, 4, 4.5
    N = gh * gw
    x0 = KI.latents(d, 1, N)[0].astype(np.float64)
    tc, tu = KI.text_states(d, 1, T, key=0)[0], KI.text_states(d, 1, T, key=1)[0]
    mc, mu = KI.mask_from_lengths(T, [8])[0], KI.mask_from_lengths(T, [3])[0]
    pos = KI.position_ids(T, gh, gw)
    mw = KI.model_weights(d)
    bw = lambda i: KI.block_weights(d, i)
    sig = [0.9, 0.6]
    args = (pos, sig, g, mw, bw, d.n_layers, d.H, d.Hkv, d.D, d.axes, d.theta, d.eps, d.t_dim)

    def v(text, mask):
        return O.backbone_forward(x0[None], text[None], pos, mask[None], np.array([sig[0]]), mw, bw, d.n_layers,
                                  d.H, d.Hkv, d.D, d.axes, d.theta, d.eps, d.t_dim)[0]
    want = x0 + (sig[1] - sig[0]) * ((1 + g) * v(tc, mc) - g * v(tu, mu))
    out = O.sample(x0, tc, tu, mc, mu, *args)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)
    swapped = O.sample(x0, tu, tc, mu, mc, *args)
    assert np.max(np.abs(swapped - want)) > 1e-3
