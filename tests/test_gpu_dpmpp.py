"""GPU parity of sd_cfg_dpmpp_2m_step (guidance + DPM-Solver++(2M)) against the fp64 oracle:
norm-wise relative error <= 2e-6 per step on x' and on the data prediction, <= 1e-5 after a
20-step sampling run on Karras sigmas."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import unet_latent_attention_b200 as sdk
from conftest import rel_err

pytestmark = pytest.mark.gpu

REL_STEP, REL_LOOP = 2e-6, 1e-5
W = 7.5


def _t(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


def _inputs(shape, seed):
    return [si.normal(shape, seed + i) for i in range(4)]  # x, eps_u, eps_c, d_prev


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("alphas", [(0.01, 0.02, 0.05), (0.3, 0.35, 0.45), (0.8, 0.9, 0.97)])
@pytest.mark.parametrize("shape", [(8, 4, 96, 96), (1, 4, 64, 64), (3, 5, 7, 11)])
def test_step(cuda, order, alphas, shape):
    x, eu, ec, dp = _inputs(shape, 1100 + sum(shape))
    a_p, a_t, a_n = alphas
    xo, d = sdk.sd_cfg_dpmpp_2m_step(_t(x, cuda), _t(eu, cuda), _t(ec, cuda), _t(dp, cuda) if order == 2 else None,
                                     W, a_p, a_t, a_n, order)
    sdk.sd_device_status()
    rx, rd = oracle.cfg_dpmpp_2m_step(x, eu, ec, dp, W, a_p, a_t, a_n, order)
    assert rel_err(xo.cpu().numpy(), rx) <= REL_STEP
    assert rel_err(d.cpu().numpy(), rd) <= REL_STEP


def test_final_step_returns_the_data_prediction(cuda):
    x, eu, ec, _ = _inputs((2, 4, 32, 32), 1200)
    xo, d = sdk.sd_cfg_dpmpp_2m_step(_t(x, cuda), _t(eu, cuda), _t(ec, cuda), None, W, 0.9, 0.95, 1.0, 1)
    sdk.sd_device_status()
    np.testing.assert_array_equal(xo.cpu().numpy(), d.cpu().numpy())
    assert rel_err(xo.cpu().numpy(), oracle.data_prediction(x, oracle.cfg(eu, ec, W), 0.95)) <= REL_STEP


def test_in_place_and_unaligned(cuda):
    x, eu, ec, dp = _inputs((100003,), 1300)
    xd, dd = _t(x, cuda), _t(dp, cuda)
    out = sdk.sd_cfg_dpmpp_2m_step(xd, _t(eu, cuda), _t(ec, cuda), dd, W, 0.2, 0.3, 0.4, 2, out=xd, d_out=dd)
    sdk.sd_device_status()
    rx, rd = oracle.cfg_dpmpp_2m_step(x, eu, ec, dp, W, 0.2, 0.3, 0.4, 2)
    assert out[0].data_ptr() == xd.data_ptr() and out[1].data_ptr() == dd.data_ptr()
    assert rel_err(xd.cpu().numpy(), rx) <= REL_STEP and rel_err(dd.cpu().numpy(), rd) <= REL_STEP
    # 4-byte offset views: not 16-byte aligned, the scalar path
    base = [torch.from_numpy(np.concatenate([[0.0], a]).astype(np.float32)).to(cuda) for a in (x, eu, ec, dp)]
    views = [b[1:] for b in base]
    xo, d = sdk.sd_cfg_dpmpp_2m_step(*views[:3], views[3], W, 0.2, 0.3, 0.4, 2)
    sdk.sd_device_status()
    assert rel_err(xo.cpu().numpy(), rx) <= REL_STEP and rel_err(d.cpu().numpy(), rd) <= REL_STEP


def test_twenty_step_sampling_run(cuda):
    # batched-serving latent [8, 4, 96, 96], Karras sigmas of the SD schedule, in place
    shape = si.WORKLOADS[5].latent
    sched = sdk.dpmpp_2m_schedule(20)
    x0 = si.normal(shape, 1400)
    eps = [(si.normal(shape, 1500 + 2 * i), si.normal(shape, 1501 + 2 * i)) for i in range(20)]
    xd, dd = _t(x0, cuda), torch.zeros(shape, device=cuda)
    for (a_p, a_t, a_n, order), (eu, ec) in zip(sched, eps):
        sdk.sd_cfg_dpmpp_2m_step(xd, _t(eu, cuda), _t(ec, cuda), dd, W, a_p, a_t, a_n, order, out=xd, d_out=dd)
    sdk.sd_device_status()
    ref = oracle.cfg_dpmpp_2m_loop(x0, eps, W, oracle.dpmpp_2m_schedule(20))
    assert rel_err(xd.cpu().numpy(), ref) <= REL_LOOP


# ---- third order

@pytest.mark.parametrize("alphas", [(0.01, 0.02, 0.035, 0.05), (0.3, 0.35, 0.4, 0.45), (0.8, 0.88, 0.93, 0.97)])
@pytest.mark.parametrize("shape", [(8, 4, 96, 96), (3, 5, 7, 11)])
def test_third_order_step(cuda, alphas, shape):
    x, eu, ec, d1 = _inputs(shape, 1600 + sum(shape))
    d2 = si.normal(shape, 1700 + sum(shape))
    a2, a1, a_t, a_n = alphas
    xo, d = sdk.sd_cfg_dpmpp_3m_step(_t(x, cuda), _t(eu, cuda), _t(ec, cuda), _t(d1, cuda), _t(d2, cuda), W, a2, a1,
                                     a_t, a_n)
    sdk.sd_device_status()
    rx, rd = oracle.cfg_dpmpp_3m_step(x, eu, ec, d1, d2, W, a2, a1, a_t, a_n)
    assert rel_err(xo.cpu().numpy(), rx) <= REL_STEP
    assert rel_err(d.cpu().numpy(), rd) <= REL_STEP


def test_third_order_twenty_step_run(cuda):
    # serving latent, Karras sigmas, orders 1, 2, 3, ..., 3, 1; history rotated through three buffers
    shape = si.WORKLOADS[5].latent
    sched = sdk.dpmpp_3m_schedule(20)
    x0 = si.normal(shape, 1800)
    eps = [(si.normal(shape, 1900 + 2 * i), si.normal(shape, 1901 + 2 * i)) for i in range(20)]
    xd = _t(x0, cuda)
    bufs = [torch.zeros(shape, device=cuda) for _ in range(3)]
    for i, ((a2, a1, a_t, a_n, order), (eu, ec)) in enumerate(zip(sched, eps)):
        d_out, d1, d2 = bufs[i % 3], bufs[(i - 1) % 3], bufs[(i - 2) % 3]
        if order == 3:
            sdk.sd_cfg_dpmpp_3m_step(xd, _t(eu, cuda), _t(ec, cuda), d1, d2, W, a2, a1, a_t, a_n, out=xd, d_out=d_out)
        else:
            sdk.sd_cfg_dpmpp_2m_step(xd, _t(eu, cuda), _t(ec, cuda), d1, W, a1, a_t, a_n, order, out=xd, d_out=d_out)
    sdk.sd_device_status()
    ref = oracle.cfg_dpmpp_3m_loop(x0, eps, W, oracle.dpmpp_3m_schedule(20))
    assert rel_err(xd.cpu().numpy(), ref) <= REL_LOOP


def test_third_order_in_place_over_the_oldest_history(cuda):
    # d_out may overwrite d_prev2 (the history rotates through two buffers), x_out may be x
    x, eu, ec, d1 = _inputs((70001,), 2000)
    d2 = si.normal((70001,), 2010)
    xd, d1d, d2d = _t(x, cuda), _t(d1, cuda), _t(d2, cuda)
    sdk.sd_cfg_dpmpp_3m_step(xd, _t(eu, cuda), _t(ec, cuda), d1d, d2d, W, 0.2, 0.25, 0.3, 0.4, out=xd, d_out=d2d)
    sdk.sd_device_status()
    rx, rd = oracle.cfg_dpmpp_3m_step(x, eu, ec, d1, d2, W, 0.2, 0.25, 0.3, 0.4)
    assert rel_err(xd.cpu().numpy(), rx) <= REL_STEP and rel_err(d2d.cpu().numpy(), rd) <= REL_STEP
