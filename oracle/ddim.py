"""Oracle: classifier-free guidance + deterministic DDIM latent update, fp64 (test infrastructure).

Guidance, from the CFG loop of "从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §7 and the
pseudo-code of "本地部署扩散模型架构与底层运行原理深度解析" (section 示例说明): the UNet runs once on the
batch [uncond, cond] and the two noise predictions are combined as
    g = eps_uncond + w * (eps_cond - eps_uncond).

Sampler step: the engine page §1 names the update step(z_t, noise_pred, t) as DDIM / DPM-Solver and
§4 keeps alphas_cumprod with "order 1 = DDIM"; the update itself is not printed. Reading taken
(the plainest one, and the only one consistent with a step that takes no noise input): DDIM
with eta = 0 on the cumulative products alpha_bar,
    x0_hat = (x - sqrt(1 - alpha_t) g) / sqrt(alpha_t)
    x'     = sqrt(alpha_prev) x0_hat + sqrt(1 - alpha_prev) g
with no clipping of x0_hat. Schedule for the multi-step sampling loop (not printed either): the
Stable Diffusion "scaled linear" betas, beta_i = linspace(sqrt(0.00085), sqrt(0.012), 1000)_i^2,
alpha_bar_t = prod_{i<=t} (1 - beta_i), timesteps 950, 900, ..., 0 and alpha_prev = 1 after the
last step.
"""
from __future__ import annotations

import numpy as np


def cfg(eps_u, eps_c, w: float) -> np.ndarray:
    """Guided noise prediction eps_u + w * (eps_c - eps_u) in fp64."""
    eu = np.asarray(eps_u, dtype=np.float64)
    ec = np.asarray(eps_c, dtype=np.float64)
    return eu + w * (ec - eu)


def ddim_step(x, g, alpha_t: float, alpha_prev: float) -> np.ndarray:
    """Deterministic DDIM (eta = 0) update of latent x given the guided noise prediction g."""
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    x0_hat = (x - np.sqrt(1.0 - alpha_t) * g) / np.sqrt(alpha_t)
    return np.sqrt(alpha_prev) * x0_hat + np.sqrt(1.0 - alpha_prev) * g


def cfg_ddim_step(x, eps_u, eps_c, w: float, alpha_t: float, alpha_prev: float) -> np.ndarray:
    """One guided sampler step: DDIM(eta=0) applied to the CFG-combined prediction."""
    return ddim_step(x, cfg(eps_u, eps_c, w), alpha_t, alpha_prev)


def scaled_linear_betas(beta_start: float = 0.00085, beta_end: float = 0.012, T: int = 1000) -> np.ndarray:
    """Scaled-linear schedule: square of T evenly spaced points between sqrt(beta_start) and sqrt(beta_end)."""
    return np.linspace(np.sqrt(beta_start), np.sqrt(beta_end), T, dtype=np.float64) ** 2


def alphas_cumprod(betas) -> np.ndarray:
    """alpha_bar_t = prod_{i<=t} (1 - beta_i)."""
    return np.cumprod(1.0 - np.asarray(betas, dtype=np.float64))


def ddim_timesteps(T: int = 1000, steps: int = 20) -> np.ndarray:
    """Evenly strided timesteps, descending: (steps-1)*T/steps, ..., T/steps, 0."""
    stride = T // steps
    return np.arange(steps - 1, -1, -1, dtype=np.int64) * stride


def ddim_schedule(steps: int = 20, T: int = 1000, beta_start: float = 0.00085, beta_end: float = 0.012):
    """List of (t, alpha_t, alpha_prev) for the sampling loop; alpha_prev = 1 after the final step."""
    ac = alphas_cumprod(scaled_linear_betas(beta_start, beta_end, T))
    ts = ddim_timesteps(T, steps)
    out = []
    for i, t in enumerate(ts):
        a_prev = ac[ts[i + 1]] if i + 1 < len(ts) else 1.0
        out.append((int(t), float(ac[t]), float(a_prev)))
    return out


def cfg_ddim_loop(x, eps_pairs, w: float, schedule) -> np.ndarray:
    """Run len(schedule) guided DDIM steps; eps_pairs[i] = (eps_u, eps_c) used at step i."""
    x = np.asarray(x, dtype=np.float64)
    for (t, a_t, a_prev), (eu, ec) in zip(schedule, eps_pairs):
        x = cfg_ddim_step(x, eu, ec, w, a_t, a_prev)
    return x
