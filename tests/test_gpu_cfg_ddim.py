"""GPU parity of sd_cfg_ddim_step against the fp64 oracle: norm-wise relative error <= 1e-6 per
step, and over the 20-step guided DDIM loop of the serving workload."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import unet_latent_attention_b200 as sdk
from conftest import rel_err

pytestmark = pytest.mark.gpu

REL = 1e-6


def _t(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_single_step_each_schedule_point(cuda, wid):
    shape = si.WORKLOADS[wid].latent
    x, eu, ec = si.latent_inputs(wid, shape)
    for t, a_t, a_p in sdk.ddim_schedule(20)[:: 4 if wid != 5 else 1]:
        out = sdk.sd_cfg_ddim_step(_t(x, cuda), _t(eu, cuda), _t(ec, cuda), 7.5, a_t, a_p).cpu().numpy()
        ref = oracle.cfg_ddim_step(x, eu, ec, 7.5, a_t, a_p)
        assert rel_err(out, ref) <= REL, (t, rel_err(out, ref))


def test_twenty_step_loop_in_place(cuda):
    w = si.WORKLOADS[5]
    x, _, _ = si.latent_inputs(5, w.latent)
    sched = sdk.ddim_schedule(20)
    pairs = [si.latent_inputs(5, w.latent, step=i)[1:] for i in range(20)]
    xd = _t(x, cuda)
    for (t, a_t, a_p), (eu, ec) in zip(sched, pairs):
        sdk.sd_cfg_ddim_step(xd, _t(eu, cuda), _t(ec, cuda), w.guidance, a_t, a_p, out=xd)
    ref = oracle.cfg_ddim_loop(x, pairs, w.guidance, oracle.ddim_schedule(20))
    assert rel_err(xd.cpu().numpy(), ref) <= REL


@pytest.mark.parametrize("n,offset", [(1, 0), (3, 0), (4097, 0), (1000, 1), (77, 3)])
def test_ragged_and_unaligned(cuda, n, offset):
    x, eu, ec = (si.normal((n + offset,), 800 + i) for i in range(3))
    xd, ud, cd = (_t(a, cuda)[offset:] for a in (x, eu, ec))
    out = torch.empty(n + offset, device=cuda)[offset:]
    sdk.sd_cfg_ddim_step(xd, ud, cd, 3.0, 0.3, 0.6, out=out)
    ref = oracle.cfg_ddim_step(x[offset:], eu[offset:], ec[offset:], 3.0, 0.3, 0.6)
    assert rel_err(out.cpu().numpy(), ref) <= REL


def test_noise_pred_halves_are_uncond_then_cond(cuda):
    x, eu, ec = si.latent_inputs(1, (2, 4, 8, 8))
    noise_pred = _t(np.concatenate([eu, ec]), cuda)
    out = sdk.sd_cfg_ddim_step_from_noise_pred(_t(x, cuda), noise_pred, 7.5, 0.2, 0.4).cpu().numpy()
    assert rel_err(out, oracle.cfg_ddim_step(x, eu, ec, 7.5, 0.2, 0.4)) <= REL
