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


# ---- third order (two history entries)

def _solve3(n, D, x_start=2.0, l0=-1.5, l1=1.5):
    """n third-order steps, uniform in lambda, on the data prediction D(lambda). The history starts
    from the model's values at two points before l0 (a lower-order warm-up would cap the global
    order at its own)."""
    h = (l1 - l0) / n
    lams = l0 + h * np.arange(-2, n + 1)  # lams[2] = l0
    x, hist = np.array([x_start]), [D(lams[0]), D(lams[1])]
    for i in range(2, n + 2):
        a_t, a_n = _alpha_bar_of_lambda(lams[i]), _alpha_bar_of_lambda(lams[i + 1])
        g = (x - np.sqrt(a_t) * D(lams[i])) / np.sqrt(1 - a_t)
        x, d = oracle.dpmpp_3m_step(x, g, hist[-1], hist[-2], _alpha_bar_of_lambda(lams[i - 2]),
                                    _alpha_bar_of_lambda(lams[i - 1]), a_t, a_n)
        hist.append(d)
    return x[0]


def _exact_F(F, x_start=2.0, l0=-1.5, l1=1.5):
    """x(l1) for the data prediction whose integral against e^u is F: (sigma1/sigma0) x0 + sigma1 (F(l1) - F(l0))."""
    sig = lambda l: np.sqrt(1 - _alpha_bar_of_lambda(l))
    return sig(l1) / sig(l0) * x_start + sig(l1) * (F(l1) - F(l0))


def test_third_order_is_exact_on_a_quadratic_data_prediction():
    # the step integrates e^lambda times the quadratic through three data predictions exactly
    c = (0.7, -1.3, 0.9)
    D = lambda l: c[0] + c[1] * l + c[2] * l * l
    F = lambda u: np.exp(u) * (c[0] + c[1] * (u - 1) + c[2] * (u * u - 2 * u + 2))  # int e^u D(u) du
    for n in (5, 17):
        assert abs(_solve3(n, D) - _exact_F(F)) < 1e-12


def test_third_order_convergence():
    D = lambda l: np.sin(2 * l)
    F = lambda u: np.exp(u) * (np.sin(2 * u) - 2 * np.cos(2 * u)) / 5  # int e^u sin(2u) du
    e3 = [abs(_solve3(n, D) - _exact_F(F)) for n in (80, 160, 320)]  # asymptotic regime
    for a, b in zip(e3, e3[1:]):
        assert 6.5 < a / b < 9.5, e3


def test_third_order_reproduces_a_linear_data_prediction_exactly_up_to_the_warm_up():
    # third-order divided differences of a linear D vanish; from the same starting point the
    # third-order step and the exact exponential integral then differ only through D1's model
    # a_p2, a_p1, a_t, a_n spaced evenly in lambda; D linear => D2 = 0 and D1 = slope * h exactly
    ls = np.array([-1.0, -0.7, -0.4, -0.1])
    ab = [_alpha_bar_of_lambda(l) for l in ls]
    Dl = lambda l: 0.3 + 0.8 * l
    x = np.array([1.25])
    g = (x - np.sqrt(ab[2]) * Dl(ls[2])) / np.sqrt(1 - ab[2])
    xn, _ = oracle.dpmpp_3m_step(x, g, Dl(ls[1]), Dl(ls[0]), ab[0], ab[1], ab[2], ab[3])
    sig = lambda l: np.sqrt(1 - _alpha_bar_of_lambda(l))
    F = lambda u: np.exp(u) * (0.3 + 0.8 * (u - 1))
    exact = sig(ls[3]) / sig(ls[2]) * x + sig(ls[3]) * (F(ls[3]) - F(ls[2]))
    np.testing.assert_allclose(xn, exact, rtol=1e-12)


def test_third_order_schedule_and_loop_end_on_the_data():
    sched = oracle.dpmpp_3m_schedule(20)
    assert [o for *_, o in sched] == [1, 2] + [3] * 17 + [1] and sched[-1][3] == 1.0
    x0 = normal((256,), 9).astype(np.float64)
    a0 = sched[0][2]
    x = np.sqrt(a0) * x0 + np.sqrt(1 - a0) * normal((256,), 10).astype(np.float64)
    eps = []
    # noise predictions consistent with the constant data prediction x0 along the run
    xs, hist = x.copy(), []
    for a_p2, a_p1, a_t, a_n, order in sched:
        g = (xs - np.sqrt(a_t) * x0) / np.sqrt(1 - a_t)
        eps.append((g, g))
        if order == 3:
            xs, d = oracle.dpmpp_3m_step(xs, g, hist[-1], hist[-2], a_p2, a_p1, a_t, a_n)
        else:
            xs, d = oracle.dpmpp_2m_step(xs, g, hist[-1] if hist else None, a_p1, a_t, a_n, order)
        hist.append(d)
    np.testing.assert_allclose(xs, x0, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(oracle.cfg_dpmpp_3m_loop(x, eps, 7.5, sched), x0, rtol=1e-10, atol=1e-10)
