"""Pins for the GroupNorm oracle: a hand-worked case, normalisation invariants, the instance-norm
and layer-norm special cases and an independent library routine. Dividing by N-1, applying the
affine per group instead of per channel, or grouping channels by c % G each fails here."""
import json
import os

import numpy as np
import torch

import oracle
from synth_inputs import normal


def test_hand_case(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "group_norm_hand.json")))
    x = np.array(g["x"])
    y = oracle.group_norm(x, np.array(g["gamma"]), np.array(g["beta"]), g["groups"], g["eps"])
    np.testing.assert_allclose(y, np.array(g["y"]), atol=1e-12)
    mean, var = oracle.group_stats(x, g["groups"])
    np.testing.assert_allclose(mean, np.array(g["mean"]), atol=1e-12)
    np.testing.assert_allclose(var, np.array(g["var"]), atol=1e-12)


def test_unit_affine_gives_zero_mean_and_unit_variance():
    x = normal((2, 64, 5, 7), 1).astype(np.float64) * 3.0 + 2.0
    eps = 1e-5
    y = oracle.group_norm(x, np.ones(64), np.zeros(64), 32, eps)
    ys = y.reshape(2, 32, -1)
    _, v = oracle.group_stats(x, 32)
    np.testing.assert_allclose(ys.mean(-1), 0.0, atol=1e-12)
    np.testing.assert_allclose(ys.var(-1), v / (v + eps), rtol=1e-12)


def test_constant_group_gives_beta():
    x = np.full((1, 8, 3, 3), 4.25)
    beta = np.arange(8) * 0.5 - 1.0
    y = oracle.group_norm(x, np.arange(8) + 1.0, beta, 4, 1e-5)
    np.testing.assert_allclose(y, np.broadcast_to(beta.reshape(1, 8, 1, 1), y.shape), atol=1e-12)


def test_instance_norm_when_groups_equal_channels():
    x = normal((2, 6, 4, 5), 2).astype(np.float64)
    y = oracle.group_norm(x, np.ones(6), np.zeros(6), 6, 1e-5)
    for b in range(2):
        for c in range(6):
            vals = x[b, c].ravel()
            m = sum(vals) / len(vals)
            var = sum((t - m) ** 2 for t in vals) / len(vals)
            np.testing.assert_allclose(y[b, c], (x[b, c] - m) / np.sqrt(var + 1e-5), atol=1e-12)


def test_layer_norm_when_one_group():
    x = normal((3, 10, 2, 2), 3).astype(np.float64)
    y = oracle.group_norm(x, np.ones(10), np.zeros(10), 1, 1e-5)
    flat = x.reshape(3, -1)
    ref = (flat - flat.mean(1, keepdims=True)) / np.sqrt(flat.var(1, keepdims=True) + 1e-5)
    np.testing.assert_allclose(y.reshape(3, -1), ref, atol=1e-12)


def test_per_channel_affine():
    x = normal((2, 8, 3, 3), 4).astype(np.float64)
    gamma = normal((8,), 5).astype(np.float64)
    beta = normal((8,), 6).astype(np.float64)
    xhat = oracle.group_norm(x, np.ones(8), np.zeros(8), 2, 1e-5)
    y = oracle.group_norm(x, gamma, beta, 2, 1e-5)
    np.testing.assert_allclose(y, xhat * gamma.reshape(1, 8, 1, 1) + beta.reshape(1, 8, 1, 1), atol=1e-12)


def test_against_torch_group_norm_float64():
    x = normal((2, 320, 8, 8), 7).astype(np.float64)
    gamma = 1 + 0.1 * normal((320,), 8).astype(np.float64)
    beta = 0.1 * normal((320,), 9).astype(np.float64)
    ref = torch.nn.functional.group_norm(torch.from_numpy(x), 32, torch.from_numpy(gamma),
                                         torch.from_numpy(beta), eps=1e-5).numpy()
    np.testing.assert_allclose(oracle.group_norm(x, gamma, beta, 32, 1e-5), ref, atol=1e-12)


def test_large_mean_is_not_cancelled():
    # |mean| >> std: the one-pass sumsq/N - mean^2 form loses the variance in low precision;
    # the oracle's two-pass fp64 form keeps it
    base = normal((1, 4, 16, 16), 10).astype(np.float64)
    x = 1e4 + 1e-2 * base
    _, v = oracle.group_stats(x, 2)
    _, v0 = oracle.group_stats(base, 2)
    np.testing.assert_allclose(v, 1e-4 * v0, rtol=1e-7)


# ---- SiLU and the fused GroupNorm + SiLU (the engine page's §9 fusion; SiLU(v) = v * sigmoid(v))

def test_silu_closed_forms():
    # sigmoid(ln 3) = 3/4 and sigmoid(-ln 3) = 1/4
    l3 = np.log(3.0)
    np.testing.assert_allclose(oracle.silu(np.array([0.0, l3, -l3])), [0.0, 0.75 * l3, -0.25 * l3], rtol=1e-15,
                               atol=0)


def test_silu_odd_part_is_identity():
    # v * s(v) - (-v) * s(-v) = v (s(v) + s(-v)) = v: catches a sign slip or sigmoid(-v) for sigmoid(v)
    v = np.linspace(-50, 50, 2001)
    np.testing.assert_allclose(oracle.silu(v) - oracle.silu(-v), v, rtol=0, atol=1e-12)


def test_silu_minimum_is_minus_omega():
    # min_v v*sigmoid(v) = -W(1/e) = -0.27846454276107380 (Lambert W), reached at v = -1 - W(1/e)
    v = np.linspace(-1.2790, -1.2780, 20001)
    y = oracle.silu(v)
    assert abs(y.min() - (-0.27846454276107380)) < 1e-12
    assert abs(v[y.argmin()] - (-1.27846454276107380)) < 1e-6


def test_silu_tails_do_not_overflow():
    y = oracle.silu(np.array([-1000.0, -40.0, 40.0, 1000.0]))
    assert np.isfinite(y).all()
    np.testing.assert_allclose(y, [0.0, -40.0 * np.exp(-40.0), 40.0, 1000.0], rtol=1e-14, atol=1e-300)


def test_silu_against_torch_float64():
    v = normal((4096,), 11).astype(np.float64) * 6
    np.testing.assert_allclose(oracle.silu(v), torch.nn.functional.silu(torch.from_numpy(v)).numpy(), rtol=1e-14,
                               atol=1e-15)


def test_group_norm_silu_constant_group_gives_silu_of_beta():
    # a constant group normalises to 0, so the output is SiLU(beta[c]): SiLU comes after the affine
    x = np.full((1, 4, 3, 3), 2.5)
    beta = np.array([-2.0, -0.5, 0.5, 3.0])
    y = oracle.group_norm_silu(x, np.full(4, 7.0), beta, 2, 1e-5)
    np.testing.assert_allclose(y, np.broadcast_to(oracle.silu(beta).reshape(1, 4, 1, 1), y.shape), rtol=1e-15)


def test_group_norm_silu_against_torch_float64():
    x = normal((2, 64, 6, 6), 12).astype(np.float64) * 3 + 1
    gamma = 1 + 0.1 * normal((64,), 13).astype(np.float64)
    beta = 0.1 * normal((64,), 14).astype(np.float64)
    tx = torch.from_numpy(x)
    ref = torch.nn.functional.silu(torch.nn.functional.group_norm(tx, 32, torch.from_numpy(gamma),
                                                                  torch.from_numpy(beta), eps=1e-5)).numpy()
    np.testing.assert_allclose(oracle.group_norm_silu(x, gamma, beta, 32, 1e-5), ref, atol=1e-12)
