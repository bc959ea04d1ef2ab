"""Pins for the guidance + DDIM oracle: a hand-worked step, the special cases of the guidance
weight and of the alphas, the DDIM consistency property, and the noise schedule's definition."""
import json
import os

import numpy as np

import oracle
from synth_inputs import normal


def test_hand_step(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "cfg_ddim_hand.json")))
    gg = oracle.cfg(g["eps_u"], g["eps_c"], g["w"])
    np.testing.assert_allclose(gg, g["g"], atol=1e-15)
    np.testing.assert_allclose(oracle.ddim_step(g["x"], gg, g["alpha_t"], 1.0), g["x0_hat"], atol=1e-14)
    out = oracle.cfg_ddim_step(g["x"], g["eps_u"], g["eps_c"], g["w"], g["alpha_t"], g["alpha_prev"])
    np.testing.assert_allclose(out, g["x_next"], atol=1e-14)


def test_guidance_weight_special_cases():
    eu = normal((100,), 1)
    ec = normal((100,), 2)
    np.testing.assert_array_equal(oracle.cfg(eu, ec, 1.0), ec.astype(np.float64))
    np.testing.assert_array_equal(oracle.cfg(eu, ec, 0.0), eu.astype(np.float64))


def test_same_alpha_is_identity_and_alpha_one_is_x0():
    x = normal((64,), 3).astype(np.float64)
    g = normal((64,), 4).astype(np.float64)
    np.testing.assert_allclose(oracle.ddim_step(x, g, 0.3, 0.3), x, atol=1e-14)
    np.testing.assert_allclose(oracle.ddim_step(x, g, 0.3, 1.0), (x - np.sqrt(0.7) * g) / np.sqrt(0.3), atol=1e-14)


def test_ddim_consistency():
    # x_t built from (x0, e) by the forward marginal is mapped to the marginal at alpha_prev
    x0 = normal((256,), 5).astype(np.float64)
    e = normal((256,), 6).astype(np.float64)
    for a_t, a_p in [(0.01, 0.02), (0.5, 0.9), (0.99915, 1.0)]:
        x = np.sqrt(a_t) * x0 + np.sqrt(1 - a_t) * e
        out = oracle.cfg_ddim_step(x, e, e, 7.5, a_t, a_p)
        np.testing.assert_allclose(out, np.sqrt(a_p) * x0 + np.sqrt(1 - a_p) * e, atol=1e-12)


def test_scaled_linear_schedule_definition():
    b = oracle.scaled_linear_betas()
    assert b.shape == (1000,)
    np.testing.assert_allclose([b[0], b[-1]], [0.00085, 0.012], rtol=1e-13)
    d = np.diff(np.sqrt(b))
    np.testing.assert_allclose(d, d[0], rtol=1e-9)
    ac = oracle.alphas_cumprod(b)
    np.testing.assert_allclose(ac[0], 1 - 0.00085, rtol=1e-15)
    np.testing.assert_allclose(ac[1:] / ac[:-1], 1 - b[1:], rtol=1e-13)
    assert (np.diff(ac) < 0).all() and 0.004 < ac[-1] < 0.006


def test_timesteps_and_loop_schedule():
    ts = oracle.ddim_timesteps(1000, 20)
    assert list(ts) == list(range(950, -1, -50))
    sched = oracle.ddim_schedule(20)
    ac = oracle.alphas_cumprod(oracle.scaled_linear_betas())
    assert len(sched) == 20 and sched[-1] == (0, ac[0], 1.0)
    for (t, a_t, a_p), (t2, a_t2, _) in zip(sched[:-1], sched[1:]):
        assert t - t2 == 50 and a_t == ac[t] and a_p == a_t2


def test_loop_is_repeated_steps():
    sched = oracle.ddim_schedule(3, T=30)
    x = normal((10,), 7)
    pairs = [(normal((10,), 8 + i), normal((10,), 20 + i)) for i in range(3)]
    ref = x.astype(np.float64)
    for (t, a_t, a_p), (eu, ec) in zip(sched, pairs):
        ref = oracle.cfg_ddim_step(ref, eu, ec, 2.0, a_t, a_p)
    np.testing.assert_array_equal(oracle.cfg_ddim_loop(x, pairs, 2.0, sched), ref)
