"""sd_attention_noalloc: the entry point for callers that cannot allocate device memory.

Some callers may not let a library call cudaMalloc: code being captured into a CUDA graph, a
framework that owns every byte of device memory through its own allocator, or a latency-bound
loop that cannot absorb the synchronisation cudaMalloc and cudaFree imply. For them the library
offers sd_attention_noalloc, whose scratch is a fixed file-scope device array. This test calls it
through the C ABI on a shape that splits query-tile items between CTAs (so the scratch is really
used) and checks two calls in a row against the allocating sd_attention entry point.

The file name sorts last so that a run stopping at the first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth_inputs as si
import unet_latent_attention_b200 as sdk
from conftest import max_abs_mean_abs

pytestmark = pytest.mark.gpu


def test_noalloc_matches_allocating_entry_point_twice(cuda):
    B, H, Lq, Lk, dh = 2, 80, 256, 640, 40  # 160 items of 256 query rows: more items than SMs
    q = si.to_bf16_exact(si.normal((B, H, Lq, dh), 9501)).to(cuda)
    k = si.to_bf16_exact(si.normal((B, H, Lk, dh), 9502)).to(cuda)
    v = si.to_bf16_exact(si.normal((B, H, Lk, dh), 9503)).to(cuda)
    L = sdk.lib()
    stream = torch.cuda.current_stream(cuda).cuda_stream
    scale = 1.0 / np.sqrt(dh)

    ref = torch.empty_like(q)
    st = L.sd_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), ref.data_ptr(), B, H, Lq, Lk, dh, ctypes.c_float(scale),
                        stream)
    assert st == 0, L.sd_last_error()
    sdk.sd_device_status()
    ref = ref.float().cpu().numpy()

    for call in range(2):
        out = torch.full_like(q, float("nan"))
        st = L.sd_attention_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, H, Lq, Lk, dh,
                                    ctypes.c_float(scale), stream)
        assert st == 0, (call, L.sd_last_error())
        sdk.sd_device_status()
        o = out.float().cpu().numpy()
        assert np.isfinite(o).all(), call
        mx, mn = max_abs_mean_abs(o, ref)
        assert mx <= 2e-2 and mn <= 2e-3, (call, mx, mn)
