"""GPU parity of sd_group_norm_silu (GroupNorm + SiLU in one launch) against the fp64 oracle.

fp32 output: norm-wise relative error <= 1e-4, as for sd_group_norm. bf16 output: every element
within half a bf16 ulp of the fp64 value plus the fp32 arithmetic (|d| <= 4e-3 |ref| + 1e-5)."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import unet_latent_attention_b200 as sdk
from conftest import rel_err

pytestmark = pytest.mark.gpu

REL = 1e-4
BF16_REL, BF16_ABS = 4e-3, 1e-5

GN_CASES = [(w.wid, label, s) for w in si.WORKLOADS.values() for label, s in w.group_norm]


def _run(x, gamma, beta, groups, eps, dev, bf16, inplace=False):
    xd = torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    out = xd if inplace else None
    y = sdk.sd_group_norm_silu(xd, torch.from_numpy(gamma).to(dev), torch.from_numpy(beta).to(dev), groups, eps,
                               out=out, out_dtype=torch.bfloat16 if bf16 else torch.float32)
    sdk.sd_device_status()
    assert y.dtype == (torch.bfloat16 if bf16 else torch.float32)
    return y.float().cpu().numpy()


def _check(y, ref, bf16):
    if bf16:
        err = np.abs(y.astype(np.float64) - ref)
        assert (err <= BF16_REL * np.abs(ref) + BF16_ABS).all(), float((err - BF16_REL * np.abs(ref)).max())
    else:
        assert rel_err(y, ref) <= REL


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
@pytest.mark.parametrize("wid,label,shape", GN_CASES, ids=[f"w{w}-{l}" for w, l, _ in GN_CASES])
def test_workload_shapes(cuda, wid, label, shape, bf16):
    x, gamma, beta = si.group_norm_inputs(wid, shape, sub=7)
    y = _run(x, gamma, beta, shape.groups, shape.eps, cuda, bf16)
    _check(y, oracle.group_norm_silu(x, gamma, beta, shape.groups, shape.eps), bf16)


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
@pytest.mark.parametrize("shape,groups", [((1, 32, 7, 9), 32), ((3, 8, 5, 4), 1), ((1, 64, 128, 128), 2),
                                          ((2, 320, 1, 1), 32), ((1, 4, 257, 3), 2)])
def test_streaming_and_odd_shapes(cuda, shape, groups, bf16):
    x = si.normal(shape, 800 + sum(shape))
    C = shape[1]
    gamma = (1 + 0.1 * si.normal((C,), 801)).astype(np.float32)
    beta = (0.1 * si.normal((C,), 802)).astype(np.float32)
    y = _run(x, gamma, beta, groups, 1e-5, cuda, bf16)
    _check(y, oracle.group_norm_silu(x, gamma, beta, groups, 1e-5), bf16)


def test_in_place_fp32(cuda):
    shape = si.GNShape(2, 320, 64, 64)
    x, gamma, beta = si.group_norm_inputs(2, shape, sub=9)
    y = _run(x, gamma, beta, 32, 1e-5, cuda, bf16=False, inplace=True)
    _check(y, oracle.group_norm_silu(x, gamma, beta, 32, 1e-5), False)


def test_bf16_output_may_not_overlap_x(cuda):
    x = torch.randn(2, 64, 8, 8, device=cuda)
    y = x.view(torch.bfloat16).reshape(-1)[:x.numel()].view(x.shape)  # x's first bytes as bf16
    with pytest.raises(sdk.SDError):
        sdk.sd_group_norm_silu(x, torch.ones(64, device=cuda), torch.zeros(64, device=cuda), 32, 1e-5, out=y)


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
def test_sdxl_top_level_groups(cuda, bf16):
    shape = si.GNShape(2, 320, 128, 128)
    x, gamma, beta = si.group_norm_inputs(4, shape, sub=21)
    y = _run(x, gamma, beta, 32, 1e-5, cuda, bf16)
    _check(y, oracle.group_norm_silu(x, gamma, beta, 32, 1e-5), bf16)
