"""Oracle: classifier-free guidance + DPM-Solver++(2M) latent update, fp64 (test infrastructure).

"从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §4 keeps, besides DDIM, a DPM-Solver++
scheduler: Karras sigmas for the timesteps, alphas_cumprod, an order (1 = DDIM-equivalent, 2 =
second order), a sample history that feeds a second-order correction of the derivative, and a
lower_order_final switch. It prints no update formula. Reading taken: the multistep
DPM-Solver++(2M) of Lu, Zhou, Bao, Chen, Li and Zhu (2022, "DPM-Solver++: Fast Solver for Guided
Sampling of Diffusion Probabilistic Models", the 2M algorithm), in the variance-preserving
parametrisation on the cumulative products alpha_bar:

    alpha = sqrt(alpha_bar), sigma = sqrt(1 - alpha_bar), lambda = log(alpha / sigma)
    D     = (x - sigma g) / alpha                      data prediction from the guided noise g
    h     = lambda_next - lambda_t
    order 1:  x' = (sigma_next / sigma_t) x - alpha_next (exp(-h) - 1) D
    order 2:  r = (lambda_t - lambda_prev) / h,
              x' = (sigma_next / sigma_t) x - alpha_next (exp(-h) - 1) ((1 + 1/(2r)) D - 1/(2r) D_prev)

where D_prev is the data prediction of the previous step (the history). Order 3 (the page's
"三阶") is the third-order multistep update of the same family on two history entries
(dpmpp_3m_step). The step to
alpha_bar = 1 (sigma = 0, the end of sampling) is taken at first order and returns D. Karras
sigmas (Karras et al. 2022, rho = 7) span the Stable Diffusion scaled-linear range and map to
alpha_bar = 1 / (1 + sigma^2).
"""
from __future__ import annotations

import numpy as np

from .ddim import alphas_cumprod, cfg, scaled_linear_betas


def lam(alpha_bar: float) -> float:
    """Half log-SNR: log(sqrt(alpha_bar) / sqrt(1 - alpha_bar)); +inf at alpha_bar = 1."""
    if alpha_bar >= 1.0:
        return np.inf
    return 0.5 * np.log(alpha_bar / (1.0 - alpha_bar))


def data_prediction(x, g, alpha_bar: float) -> np.ndarray:
    """x0 predicted from the latent and the noise prediction: (x - sigma g) / alpha."""
    return (np.asarray(x, np.float64) - np.sqrt(1.0 - alpha_bar) * np.asarray(g, np.float64)) / np.sqrt(alpha_bar)


def dpmpp_2m_step(x, g, d_prev, alpha_prev: float, alpha_t: float, alpha_next: float, order: int):
    """One DPM-Solver++ step from alpha_bar = alpha_t to alpha_next; returns (x_next, D).

    D is this step's data prediction (the history entry for the next step). order 2 needs d_prev
    and alpha_prev (the previous step's alpha_bar)."""
    x = np.asarray(x, np.float64)
    D = data_prediction(x, g, alpha_t)
    a_n, s_n, s_t = np.sqrt(alpha_next), np.sqrt(1.0 - alpha_next), np.sqrt(1.0 - alpha_t)
    if alpha_next >= 1.0:  # sigma_next = 0: exp(-h) = 0 and the step returns the data prediction
        return a_n * D, D
    h = lam(alpha_next) - lam(alpha_t)
    if order == 2:
        r = (lam(alpha_t) - lam(alpha_prev)) / h
        Dhat = (1.0 + 1.0 / (2.0 * r)) * D - (1.0 / (2.0 * r)) * np.asarray(d_prev, np.float64)
    elif order == 1:
        Dhat = D
    else:
        raise ValueError("order must be 1 or 2")
    return (s_n / s_t) * x - a_n * np.expm1(-h) * Dhat, D


def dpmpp_3m_step(x, g, d1, d2, alpha_p2: float, alpha_p1: float, alpha_t: float, alpha_next: float):
    """Third-order multistep DPM-Solver++ step; returns (x_next, D).

    d1, d2 are the data predictions of the previous two steps, taken at alpha_bar = alpha_p1 and
    alpha_p2. With m0 = D, m1 = d1, m2 = d2, h = lambda_next - lambda_t, h0 = lambda_t - lambda_p1,
    h1 = lambda_p1 - lambda_p2, r0 = h0 / h, r1 = h1 / h:
        D1_0 = (m0 - m1) / r0,  D1_1 = (m1 - m2) / r1
        D1   = D1_0 + r0 / (r0 + r1) (D1_0 - D1_1)      h * D'(lambda_t) of the quadratic through m2, m1, m0
        D2   = (D1_0 - D1_1) / (r0 + r1)                h^2 * D''/2 of that quadratic
        x'   = (sigma_next / sigma_t) x - alpha_next (e^-h - 1) m0
               + alpha_next ((e^-h - 1) / h + 1) D1 - 2 alpha_next ((e^-h - 1 + h) / h^2 - 1/2) D2
    This is the exact integral x' = (sigma_next/sigma_t) x + sigma_next int e^lambda D(lambda) dlambda
    of the quadratic that interpolates the three data predictions in lambda (the multistep
    third-order construction of DPM-Solver, Lu et al. 2022, in data-prediction form), hence
    third-order accurate."""
    x = np.asarray(x, np.float64)
    m0 = data_prediction(x, g, alpha_t)
    m1, m2 = np.asarray(d1, np.float64), np.asarray(d2, np.float64)
    a_n, s_n, s_t = np.sqrt(alpha_next), np.sqrt(1.0 - alpha_next), np.sqrt(1.0 - alpha_t)
    h = lam(alpha_next) - lam(alpha_t)
    r0 = (lam(alpha_t) - lam(alpha_p1)) / h
    r1 = (lam(alpha_p1) - lam(alpha_p2)) / h
    d1_0, d1_1 = (m0 - m1) / r0, (m1 - m2) / r1
    D1 = d1_0 + r0 / (r0 + r1) * (d1_0 - d1_1)
    D2 = (d1_0 - d1_1) / (r0 + r1)
    em = np.expm1(-h)
    xn = ((s_n / s_t) * x - a_n * em * m0 + a_n * (em / h + 1.0) * D1 - 2.0 * a_n * ((em + h) / h ** 2 - 0.5) * D2)
    return xn, m0


def cfg_dpmpp_2m_step(x, eps_u, eps_c, d_prev, w: float, alpha_prev: float, alpha_t: float, alpha_next: float,
                      order: int):
    """One guided step: DPM-Solver++ on the CFG-combined noise prediction; returns (x_next, D)."""
    return dpmpp_2m_step(x, cfg(eps_u, eps_c, w), d_prev, alpha_prev, alpha_t, alpha_next, order)


def cfg_dpmpp_3m_step(x, eps_u, eps_c, d1, d2, w: float, alpha_p2: float, alpha_p1: float, alpha_t: float,
                      alpha_next: float):
    """Guided third-order multistep step; returns (x_next, D)."""
    return dpmpp_3m_step(x, cfg(eps_u, eps_c, w), d1, d2, alpha_p2, alpha_p1, alpha_t, alpha_next)


def karras_sigmas(n: int, sigma_min: float, sigma_max: float, rho: float = 7.0) -> np.ndarray:
    """n noise levels from sigma_max down to sigma_min, evenly spaced in sigma^(1/rho)."""
    ramp = np.linspace(0.0, 1.0, n)
    lo, hi = sigma_min ** (1.0 / rho), sigma_max ** (1.0 / rho)
    return (hi + ramp * (lo - hi)) ** rho


def alpha_bar_of_sigma(sigma) -> np.ndarray:
    """Variance-preserving alpha_bar of a variance-exploding noise level: 1 / (1 + sigma^2)."""
    return 1.0 / (1.0 + np.asarray(sigma, np.float64) ** 2)


def sd_sigma_range(T: int = 1000) -> tuple[float, float]:
    """sigma = sqrt((1 - alpha_bar) / alpha_bar) at the first and last training timestep."""
    ab = alphas_cumprod(scaled_linear_betas(T=T))
    s = np.sqrt((1.0 - ab) / ab)
    return float(s[0]), float(s[-1])


def dpmpp_2m_schedule(steps: int = 20):
    """[(alpha_prev, alpha_t, alpha_next, order)] for a sampling run on Karras sigmas of the SD range.

    First step and the final step (to sigma = 0) are first order; the others second order."""
    smin, smax = sd_sigma_range()
    ab = list(alpha_bar_of_sigma(karras_sigmas(steps, smin, smax))) + [1.0]
    out = []
    for i in range(steps):
        order = 1 if i == 0 or i == steps - 1 else 2
        out.append((ab[i - 1] if i > 0 else ab[0], ab[i], ab[i + 1], order))
    return out


def cfg_dpmpp_2m_loop(x, eps_pairs, w: float, schedule):
    """Runs the guided DPM-Solver++(2M) steps of `schedule` with the given (eps_u, eps_c) per step."""
    x = np.asarray(x, np.float64)
    d = None
    for (a_p, a_t, a_n, order), (eu, ec) in zip(schedule, eps_pairs):
        x, d = cfg_dpmpp_2m_step(x, eu, ec, d, w, a_p, a_t, a_n, order)
    return x


def dpmpp_3m_schedule(steps: int = 20):
    """[(alpha_prev2, alpha_prev, alpha_t, alpha_next, order)]: orders 1, 2, then 3; last step order 1."""
    smin, smax = sd_sigma_range()
    ab = list(alpha_bar_of_sigma(karras_sigmas(steps, smin, smax))) + [1.0]
    out = []
    for i in range(steps):
        order = 1 if i == 0 or i == steps - 1 else min(i + 1, 3)
        out.append((ab[i - 2] if i >= 2 else ab[i], ab[i - 1] if i >= 1 else ab[i], ab[i], ab[i + 1], order))
    return out


def cfg_dpmpp_3m_loop(x, eps_pairs, w: float, schedule):
    """Runs a guided multistep run of orders 1-3 (schedule from dpmpp_3m_schedule)."""
    x = np.asarray(x, np.float64)
    hist = []
    for (a_p2, a_p1, a_t, a_n, order), (eu, ec) in zip(schedule, eps_pairs):
        if order == 3:
            x, d = cfg_dpmpp_3m_step(x, eu, ec, hist[-1], hist[-2], w, a_p2, a_p1, a_t, a_n)
        else:
            x, d = cfg_dpmpp_2m_step(x, eu, ec, hist[-1] if hist else None, w, a_p1, a_t, a_n, order)
        hist.append(d)
    return x
