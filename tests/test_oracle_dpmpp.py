"""Pins of the DPM-Solver++(2M) oracle (oracle/dpmpp.py) against facts fixed independently of it.

* The engine page's §4 states that order 1 is DDIM-equivalent: the first-order step must equal
  the DDIM update (oracle/ddim.py, itself pinned by hand-worked values).
* A constant data prediction is integrated exactly by both orders (the exponential integrator
  solves the ODE exactly when x0 does not change).
* On a data prediction that is linear in lambda the ODE has a closed-form solution; halving the
  step size must cut the error by about 4 for the second-order method and about 2 for the
  first-order one (a wrong second-order coefficient drops the observed order to 1).
* Karras sigmas: endpoints, rho = 1 spacing, and the alpha_bar <-> sigma map."""
import numpy as np
import pytest

import oracle
from synth_inputs import normal


def test_order_one_is_ddim():
    x, g = normal((4096,), 1).astype(np.float64), normal((4096,), 2).astype(np.float64)
    for a_t, a_n in [(0.05, 0.2), (0.3, 0.31), (0.7, 0.99), (0.2, 1.0)]:
        xn, _ = oracle.dpmpp_2m_step(x, g, None, a_t, a_t, a_n, 1)
        np.testing.assert_allclose(xn, oracle.ddim_step(x, g, a_t, a_n), rtol=1e-12, atol=1e-12)


def test_data_prediction_definition():
    # x = alpha x0 + sigma eps  =>  D = x0
    x0, eps = normal((1000,), 3).astype(np.float64), normal((1000,), 4).astype(np.float64)
    a = 0.37
    x = np.sqrt(a) * x0 + np.sqrt(1 - a) * eps
    np.testing.assert_allclose(oracle.data_prediction(x, eps, a), x0, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("order", [1, 2])
def test_constant_data_prediction_is_exact(order):
    x0, e = normal((512,), 5).astype(np.float64), normal((512,), 6).astype(np.float64)
    a_p, a_t, a_n = 0.1, 0.2, 0.45
    x = np.sqrt(a_t) * x0 + np.sqrt(1 - a_t) * e
    g = (x - np.sqrt(a_t) * x0) / np.sqrt(1 - a_t)  # the model's noise prediction consistent with x0
    xn, D = oracle.dpmpp_2m_step(x, g, x0, a_p, a_t, a_n, order)
    np.testing.assert_allclose(D, x0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(xn, np.sqrt(a_n) * x0 + np.sqrt(1 - a_n) * e, rtol=1e-12, atol=1e-12)


def _alpha_bar_of_lambda(l):
    return 1.0 / (1.0 + np.exp(-2.0 * l))


def _solve(n, order, c0=0.7, c1=-1.3, x_start=2.0, l0=-1.5, l1=1.5):
    """n steps, uniform in lambda, on the 'model' D(lambda) = c0 + c1 lambda; returns the final x."""
    lams = np.linspace(l0, l1, n + 1)
    x, d = np.array([x_start]), None
    for i in range(n):
        a_t, a_n = _alpha_bar_of_lambda(lams[i]), _alpha_bar_of_lambda(lams[i + 1])
        a_p = _alpha_bar_of_lambda(lams[i - 1]) if i else a_t
        D = c0 + c1 * lams[i]
        g = (x - np.sqrt(a_t) * D) / np.sqrt(1 - a_t)
        x, d = oracle.dpmpp_2m_step(x, g, d, a_p, a_t, a_n, 1 if (order == 1 or i == 0) else 2)
    return x[0]


def _exact(c0=0.7, c1=-1.3, x_start=2.0, l0=-1.5, l1=1.5):
    # x(l) = (sigma(l)/sigma(l0)) x(l0) + sigma(l) * int_{l0}^{l} e^u (c0 + c1 u) du,
    # int e^u (c0 + c1 u) du = e^u (c0 + c1 (u - 1))
    sig = lambda l: np.sqrt(1 - _alpha_bar_of_lambda(l))
    F = lambda u: np.exp(u) * (c0 + c1 * (u - 1))
    return sig(l1) / sig(l0) * x_start + sig(l1) * (F(l1) - F(l0))


def test_second_order_convergence():
    ex = _exact()
    e2 = [abs(_solve(n, 2) - ex) for n in (10, 20, 40)]
    e1 = [abs(_solve(n, 1) - ex) for n in (10, 20, 40)]
    for a, b in zip(e2, e2[1:]):
        assert 3.2 < a / b < 5.0, e2
    for a, b in zip(e1, e1[1:]):
        assert 1.7 < a / b < 2.4, e1
    assert e2[-1] < e1[-1] / 20


def test_karras_sigmas():
    s = oracle.karras_sigmas(20, 0.03, 14.6)
    assert s[0] == pytest.approx(14.6, rel=1e-14) and s[-1] == pytest.approx(0.03, rel=1e-14)
    assert (np.diff(s) < 0).all()
    np.testing.assert_allclose(oracle.karras_sigmas(5, 1.0, 3.0, rho=1.0), [3.0, 2.5, 2.0, 1.5, 1.0], rtol=1e-14)
    # rho: sigma^(1/rho) is evenly spaced
    np.testing.assert_allclose(np.diff(s ** (1 / 7.0)), np.full(19, (0.03 ** (1 / 7) - 14.6 ** (1 / 7)) / 19),
                               rtol=1e-10)


def test_alpha_bar_sigma_round_trip():
    ab = np.linspace(0.001, 0.999, 50)
    sigma = np.sqrt((1 - ab) / ab)
    np.testing.assert_allclose(oracle.alpha_bar_of_sigma(sigma), ab, rtol=1e-13)
    lo, hi = oracle.sd_sigma_range()
    assert 0.02 < lo < 0.04 and 14.0 < hi < 15.5  # SD scaled-linear schedule: ~0.029 .. ~14.6


def test_schedule_and_loop_end_on_the_data():
    sched = oracle.dpmpp_2m_schedule(20)
    assert len(sched) == 20 and sched[-1][2] == 1.0
    assert [o for *_, o in sched] == [1] + [2] * 18 + [1]
    abs_ = [a for _, a, _, _ in sched]
    assert (np.diff(abs_) > 0).all()
    # a model that always predicts the same x0 ends exactly on x0 (the last step returns D)
    x0 = normal((256,), 7).astype(np.float64)
    x = np.sqrt(sched[0][1]) * x0 + np.sqrt(1 - sched[0][1]) * normal((256,), 8).astype(np.float64)
    d = None
    for a_p, a_t, a_n, order in sched:
        g = (x - np.sqrt(a_t) * x0) / np.sqrt(1 - a_t)
        x, d = oracle.dpmpp_2m_step(x, g, d, a_p, a_t, a_n, order)
    np.testing.assert_allclose(x, x0, rtol=1e-10, atol=1e-10)
