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


# ---- guidance wiring and history bookkeeping of the guided steps and loops
#
# The guided steps combine the two noise predictions as eps_u + w (eps_c - eps_u) (the CFG loop of
# the engine page §7 and the deployment page's 示例说明) before the solver step. With w != 1 and
# eps_u != eps_c, the pins below build the pair so that only the correct combination gives the noise
# prediction g consistent with a known data prediction; swapping the pair gives g + a (2 - 1/w).

W = 7.5


def _guided_pair(g, seed):
    """(eps_u, eps_c) with eps_u + W (eps_c - eps_u) = g and eps_u != eps_c."""
    a = normal(np.shape(g), seed).astype(np.float64)
    return g + a, g + a * (1.0 - 1.0 / W)


def test_guided_pair_construction():
    g = normal((64,), 20).astype(np.float64)
    eu, ec = _guided_pair(g, 21)
    np.testing.assert_allclose(oracle.cfg(eu, ec, W), g, rtol=0, atol=1e-12)
    assert np.abs(oracle.cfg(ec, eu, W) - g).max() > 0.5  # the swapped order is far off


@pytest.mark.parametrize("order", [1, 2])
def test_guided_2m_step_lands_on_the_closed_form(order):
    # constant data prediction x0: the exponential integrator is exact for both orders
    x0, e = normal((512,), 22).astype(np.float64), normal((512,), 23).astype(np.float64)
    a_p, a_t, a_n = 0.1, 0.2, 0.45
    x = np.sqrt(a_t) * x0 + np.sqrt(1 - a_t) * e
    g = (x - np.sqrt(a_t) * x0) / np.sqrt(1 - a_t)
    eu, ec = _guided_pair(g, 24)
    xn, D = oracle.cfg_dpmpp_2m_step(x, eu, ec, x0, W, a_p, a_t, a_n, order)
    np.testing.assert_allclose(D, x0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(xn, np.sqrt(a_n) * x0 + np.sqrt(1 - a_n) * e, rtol=1e-12, atol=1e-12)


def test_guided_3m_step_lands_on_the_closed_form():
    x0, e = normal((512,), 25).astype(np.float64), normal((512,), 26).astype(np.float64)
    a2, a1, a_t, a_n = 0.05, 0.1, 0.2, 0.45
    x = np.sqrt(a_t) * x0 + np.sqrt(1 - a_t) * e
    g = (x - np.sqrt(a_t) * x0) / np.sqrt(1 - a_t)
    eu, ec = _guided_pair(g, 27)
    xn, D = oracle.cfg_dpmpp_3m_step(x, eu, ec, x0, x0, W, a2, a1, a_t, a_n)
    np.testing.assert_allclose(D, x0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(xn, np.sqrt(a_n) * x0 + np.sqrt(1 - a_n) * e, rtol=1e-12, atol=1e-12)


def _lam_of(ab):
    return 0.5 * np.log(ab / (1.0 - ab))


def _sig(ab):
    return np.sqrt(1.0 - ab)


def _run_guided(loop, x, sched, D_of_lambda, seed):
    """Drives `loop` with guided noise pairs that, at each step's state, are consistent with the data
    prediction D(lambda_t). The states come from the loop itself run on growing prefixes of the
    schedule (every prefix run starts from the same x); returns the full run's result and the pairs."""
    eps = []
    xs = np.array(x, np.float64)
    for i, row in enumerate(sched):
        a_t = row[1] if len(row) == 4 else row[2]  # (a_p, a_t, a_n, order) or (a_p2, a_p1, a_t, a_n, order)
        g = (xs - np.sqrt(a_t) * D_of_lambda(_lam_of(a_t))) / np.sqrt(1 - a_t)
        eps.append(_guided_pair(g, seed + i))
        xs = loop(x, eps, W, sched[: i + 1])
    return xs, eps


def test_guided_2m_loop_is_the_midpoint_exponential_integrator_on_a_linear_data_prediction():
    # For D(lambda) = c0 + c1 lambda, the second-order combination (1 + 1/(2r)) D_t - D_prev / (2r)
    # equals D at the midpoint lambda_t + h/2 exactly, so each order-2 step of a correct loop is
    #   x' = (sigma'/sigma) x + sigma' (e^lambda' - e^lambda) D(lambda + h/2),
    # and an order-1 step uses D(lambda). This needs D_prev and alpha_prev of the PREVIOUS step.
    c0, c1 = 0.4, -0.9
    D = lambda l: c0 + c1 * l
    sched = oracle.dpmpp_2m_schedule(12)[:-1]  # stop before the step to sigma = 0 (it returns D alone)
    x = normal((8,), 28).astype(np.float64)
    got, _ = _run_guided(oracle.cfg_dpmpp_2m_loop, x, sched, D, 300)
    ref = x.copy()
    for a_p, a_t, a_n, order in sched:
        l_t, l_n = _lam_of(a_t), _lam_of(a_n)
        l_mid = l_t if order == 1 else l_t + 0.5 * (l_n - l_t)
        ref = _sig(a_n) / _sig(a_t) * ref + _sig(a_n) * (np.exp(l_n) - np.exp(l_t)) * D(l_mid)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_guided_3m_loop_is_exact_after_its_warm_up_on_a_quadratic_data_prediction():
    # Orders 1 and 2 open the run; from the third step on, each order-3 step integrates
    # e^lambda D(lambda) exactly when D is quadratic and the two history entries are the data
    # predictions of the previous two steps, newest first. The exact flow is affine in x, so the
    # loop's result must equal (sigma_K / sigma_2) x_2 + sigma_K (F(lambda_K) - F(lambda_2)), where
    # x_2 is the state after the two warm-up steps and F' = e^u D(u).
    c = (0.7, -1.3, 0.9)
    D = lambda l: c[0] + c[1] * l + c[2] * l * l
    F = lambda u: np.exp(u) * (c[0] + c[1] * (u - 1) + c[2] * (u * u - 2 * u + 2))
    sched = oracle.dpmpp_3m_schedule(14)[:-1]
    assert [o for *_, o in sched] == [1, 2] + [3] * 11
    x = normal((8,), 29).astype(np.float64)
    got, eps = _run_guided(oracle.cfg_dpmpp_3m_loop, x, sched, D, 400)
    x2 = oracle.cfg_dpmpp_3m_loop(x, eps[:2], W, sched[:2])
    a2, aK = sched[2][2], sched[-1][3]
    ref = _sig(aK) / _sig(a2) * x2 + _sig(aK) * (F(_lam_of(aK)) - F(_lam_of(a2)))
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-11)
