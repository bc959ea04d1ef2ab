"""Host-side noise-schedule tables for driving sd_cfg_ddim_step over a denoising loop.

Stable Diffusion's "scaled linear" betas: T points evenly spaced between sqrt(beta_start) and
sqrt(beta_end), squared; alpha_bar_t is the running product of (1 - beta). The sampler of
"从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" (§4, scheduler holding alphas_cumprod; the
order-1 solver is DDIM) steps through evenly strided timesteps; alpha_prev = 1 after the last
step. Plain Python floats (double precision); the kernel receives alpha_t and alpha_prev.

For sd_cfg_dpmpp_2m_step: Karras noise levels (rho = 7) between the smallest and largest sigma of
the same training schedule, sigma = sqrt((1 - alpha_bar) / alpha_bar), mapped back to
alpha_bar = 1 / (1 + sigma^2), then alpha_bar = 1 at the end; first and last steps first order.
"""
from __future__ import annotations

import math


def scaled_linear_alphas_cumprod(beta_start: float = 0.00085, beta_end: float = 0.012, T: int = 1000):
    lo, hi = beta_start ** 0.5, beta_end ** 0.5
    out, prod = [], 1.0
    for i in range(T):
        r = lo + (hi - lo) * i / (T - 1)
        prod *= 1.0 - r * r
        out.append(prod)
    return out


def ddim_schedule(steps: int = 20, T: int = 1000, beta_start: float = 0.00085, beta_end: float = 0.012):
    """[(t, alpha_t, alpha_prev)] for t = (steps-1)*T/steps, ..., T/steps, 0."""
    ac = scaled_linear_alphas_cumprod(beta_start, beta_end, T)
    stride = T // steps
    ts = [stride * i for i in range(steps - 1, -1, -1)]
    return [(t, ac[t], ac[ts[i + 1]] if i + 1 < len(ts) else 1.0) for i, t in enumerate(ts)]


def karras_alpha_bars(steps: int, rho: float = 7.0, T: int = 1000):
    """alpha_bar of `steps` Karras noise levels spanning the scaled-linear schedule, descending noise."""
    ac = scaled_linear_alphas_cumprod(T=T)
    s_lo, s_hi = math.sqrt((1 - ac[0]) / ac[0]), math.sqrt((1 - ac[-1]) / ac[-1])
    a, b = s_hi ** (1 / rho), s_lo ** (1 / rho)
    sig = [(a + (b - a) * i / (steps - 1)) ** rho for i in range(steps)]
    return [1.0 / (1.0 + x * x) for x in sig]


def dpmpp_2m_schedule(steps: int = 20):
    """[(alpha_prev, alpha_t, alpha_next, order)] for sd_cfg_dpmpp_2m_step over a whole sampling run."""
    ab = karras_alpha_bars(steps) + [1.0]
    return [(ab[i - 1] if i else ab[0], ab[i], ab[i + 1], 1 if i in (0, steps - 1) else 2) for i in range(steps)]


def dpmpp_3m_schedule(steps: int = 20):
    """[(alpha_prev2, alpha_prev, alpha_t, alpha_next, order)] for a third-order run: order 1, then 2,
    then 3, with the last step (to sigma = 0) first order. Unused history slots repeat alpha_t."""
    ab = karras_alpha_bars(steps) + [1.0]
    out = []
    for i in range(steps):
        order = 1 if i in (0, steps - 1) else min(i + 1, 3)
        out.append((ab[i - 2] if i >= 2 else ab[i], ab[i - 1] if i >= 1 else ab[i], ab[i], ab[i + 1], order))
    return out
