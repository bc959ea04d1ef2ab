"""Failure path on the GPU without a fault: the test hook makes one attention launch (the general
kernel, and the short-key-sequence kernel) skip its first V tile, so the kernel's bounded mbarrier wait expires (after about a second). The kernel
must drain its own copies and MMAs, free tensor memory, return, and report SD_ERR_TIMEOUT through
sd_device_status; the context stays usable and the next launch is correct. Runs in a child
process with a timeout so that a regression cannot hold the test session."""
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

CHILD = textwrap.dedent(r"""
    import sys
    sys.path.insert(0, {root!r})
    import numpy as np, torch
    import oracle, synth_inputs as si
    import unet_latent_attention_b200 as sdk
    dev = torch.device("cuda:0")
    q = si.to_bf16_exact(si.normal((1, 1, 128, 64), 11)).to(dev)
    k = si.to_bf16_exact(si.normal((1, 1, {lk}, 64), 12)).to(dev)
    v = si.to_bf16_exact(si.normal((1, 1, {lk}, 64), 13)).to(dev)
    sdk.sd_device_status()
    sdk.sd_debug_set_fault(1)
    sdk.sd_attention(q, k, v)
    sdk.sd_debug_set_fault(0)
    try:
        sdk.sd_device_status(reset=True)
        print("NO_TIMEOUT_REPORTED"); sys.exit(3)
    except sdk.SDError as e:
        assert e.status == 5, e
    sdk.sd_device_status()          # cleared by the reset
    o = sdk.sd_attention(q, k, v)   # the context is still usable
    sdk.sd_device_status()
    d = np.abs(o.float().cpu().numpy() - oracle.attention(q.cpu(), k.cpu(), v.cpu()))
    assert d.max() <= 2e-2, d.max()
    print("FAULT_PATH_OK")
""")


@pytest.mark.parametrize("lk", [256, 77], ids=["general-kernel", "short-key-kernel"])
def test_bounded_wait_reports_timeout(cuda, lk):
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=root, lk=lk)], capture_output=True, text=True,
                       timeout=90)
    assert r.returncode == 0 and "FAULT_PATH_OK" in r.stdout, (r.stdout[-2000:], r.stderr[-2000:])
