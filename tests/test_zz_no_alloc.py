"""sd_attention_noalloc: the entry point for callers that cannot allocate device memory.

Some callers may not let a library call cudaMalloc: code being captured into a CUDA graph, a
framework that owns every byte of device memory through its own allocator, or a latency-bound
loop that cannot absorb the synchronisation cudaMalloc and cudaFree imply. For them the library
offers sd_attention_noalloc, whose scratch is a fixed file-scope device array. These tests call it
through the C ABI on a shape that splits query-tile items between CTAs (so the scratch is really
used):

* two calls in a row on different inputs, each against the oracle and bit for bit against the
  allocating sd_attention entry point on the same inputs (a hand-off that read a stale slot of the
  previous call would differ);
* in a fresh child process where sd_attention never ran, a call on a splitting shape leaves the
  device's free memory unchanged (sd_attention's workspace for this shape would take about 7 MB).

The file name sorts last so that a run stopping at the first failure has run every other test.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)

from conftest import max_abs_mean_abs  # noqa: E402

import oracle  # noqa: E402
import synth_inputs as si  # noqa: E402
import unet_latent_attention_b200 as sdk  # noqa: E402

pytestmark = pytest.mark.gpu

# 160 items of 256 query rows on 148 SMs: items are split between neighbouring CTAs
B, H, LQ, LK, DH = 2, 80, 256, 640, 40
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _inputs(seed, dev):
    return tuple(si.to_bf16_exact(si.normal((B, H, L, DH), seed + i)).to(dev) for i, L in enumerate((LQ, LK, LK)))


def _call(fn_name, q, k, v, out):
    L = sdk.lib()
    stream = torch.cuda.current_stream(q.device).cuda_stream
    st = getattr(L, fn_name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, LQ, LK, DH,
                             ctypes.c_float(1.0 / np.sqrt(DH)), stream)
    assert st == 0, (fn_name, L.sd_last_error())


def test_noalloc_matches_the_oracle_and_the_allocating_entry_point_twice(cuda):
    for call, seed in enumerate((9501, 9601)):
        q, k, v = _inputs(seed, cuda)
        out = torch.full_like(q, float("nan"))
        _call("sd_attention_noalloc", q, k, v, out)
        sdk.sd_device_status()
        ref = torch.full_like(q, float("nan"))
        _call("sd_attention", q, k, v, ref)
        sdk.sd_device_status()
        assert torch.equal(out, ref), call
        o = out.float().cpu().numpy()
        assert np.isfinite(o).all(), call
        mx, mn = max_abs_mean_abs(o, oracle.attention(q.cpu(), k.cpu(), v.cpu()))
        assert mx <= MAX_ABS and mn <= MEAN_ABS, (call, mx, mn)


def _child():
    """Runs in a fresh process: sd_attention never runs here, so its workspace never exists."""
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    q, k, v = _inputs(9701, dev)
    out = torch.empty_like(q)
    # load the library's module and this head dim's kernel with a shape that does not split items
    small = torch.zeros(1, 1, 128, DH, dtype=torch.bfloat16, device=dev)
    sdk.sd_attention_noalloc(small, small, small)
    sdk.sd_device_status()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    _call("sd_attention_noalloc", q, k, v, out)
    sdk.sd_device_status()
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info(dev)[0]
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
    mx, mn = max_abs_mean_abs(out.float().cpu().numpy(), oracle.attention(q.cpu(), k.cpu(), v.cpu()))
    assert mx <= MAX_ABS and mn <= MEAN_ABS, (mx, mn)
    print("child ok", free0 - free1)


def test_noalloc_allocates_nothing_in_a_fresh_process(cuda):
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "child"], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "child ok 0" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


if __name__ == "__main__" and sys.argv[1:] == ["child"]:
    _child()
