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

where D_prev is the data prediction of the previous step (the history). The step to
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


def cfg_dpmpp_2m_step(x, eps_u, eps_c, d_prev, w: float, alpha_prev: float, alpha_t: float, alpha_next: float,
                      order: int):
    """One guided step: DPM-Solver++ on the CFG-combined noise prediction; returns (x_next, D)."""
    return dpmpp_2m_step(x, cfg(eps_u, eps_c, w), d_prev, alpha_prev, alpha_t, alpha_next, order)


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
