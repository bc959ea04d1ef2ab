"""Oracle: GroupNorm over NCHW fp32 input, fp64 arithmetic (test infrastructure only).

"从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §3.1 reduces each group to its sum and
sum of squares, then takes mean = sum / N, var = sumsq / N - mean^2 (biased, divide by N) and
inv_std = 1 / sqrt(var + eps); the normalise-and-affine tail is elided on the page. Reading taken
here: group g of C/G consecutive channels is normalised with its own mean and inv_std and then
each channel c gets y = x_hat * gamma[c] + beta[c] (the standard GroupNorm affine).

The oracle computes the same statistics in the numerically safer two-pass form (mean first,
then the mean of squared deviations), which equals the page's one-pass form in exact arithmetic.

The engine page's §9 names GroupNorm + SiLU as one fused kernel without defining SiLU; it is taken
as the sigmoid-weighted linear unit v * sigmoid(v) (the activation after GroupNorm in the UNet's
residual blocks).
"""
from __future__ import annotations

import numpy as np


def group_stats(x, groups: int):
    """Per (batch, group) mean and biased variance of x [B, C, ...]; returns two fp64 [B, groups]."""
    x = np.asarray(x, dtype=np.float64)
    B, C = x.shape[:2]
    if C % groups:
        raise ValueError("channels must be divisible by groups")
    xs = x.reshape(B, groups, -1)  # group g = channels [g*C/G, (g+1)*C/G), all spatial positions
    mean = xs.mean(axis=2)
    var = ((xs - mean[:, :, None]) ** 2).mean(axis=2)
    return mean, var


def group_norm(x, gamma, beta, groups: int = 32, eps: float = 1e-5) -> np.ndarray:
    """y = (x - mean_g) / sqrt(var_g + eps) * gamma[c] + beta[c]; x [B, C, H, W] -> fp64 [B, C, H, W]."""
    x = np.asarray(x, dtype=np.float64)
    B, C = x.shape[:2]
    mean, var = group_stats(x, groups)
    inv_std = 1.0 / np.sqrt(var + eps)
    xs = x.reshape(B, groups, -1)
    xhat = ((xs - mean[:, :, None]) * inv_std[:, :, None]).reshape(x.shape)
    bshape = (1, C) + (1,) * (x.ndim - 2)
    g = np.asarray(gamma, dtype=np.float64).reshape(bshape)
    b = np.asarray(beta, dtype=np.float64).reshape(bshape)
    return xhat * g + b


def silu(v) -> np.ndarray:
    """v * sigmoid(v) in fp64, written with exp(-|v|) so that no exponential overflows."""
    v = np.asarray(v, dtype=np.float64)
    e = np.exp(-np.abs(v))
    sig = np.where(v >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return v * sig


def group_norm_silu(x, gamma, beta, groups: int = 32, eps: float = 1e-5) -> np.ndarray:
    """SiLU applied to the GroupNorm output (after the per-channel affine)."""
    return silu(group_norm(x, gamma, beta, groups, eps))
