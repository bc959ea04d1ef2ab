"""Host-side checks that need no GPU: the library builds and loads, exports every function that
include/sd_kernels.h declares, validates arguments before touching the device, and the binding
refuses CPU tensors instead of falling back."""
import ctypes

import pytest
import torch

import unet_latent_attention_b200 as sdk
from unet_latent_attention_b200 import build as sdbuild


@pytest.fixture(scope="module")
def L():
    sdbuild.build()
    return sdk.lib()


def test_exports_every_header_function(L):
    names = sdk.header_functions()
    assert {"sd_group_norm", "sd_attention", "sd_cfg_ddim_step", "sd_device_status"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, name in sdk.STATUS_NAMES.items():
        assert L.sd_status_string(code).decode() == name
    assert L.sd_version() >= 100


def _err(L):
    return L.sd_last_error().decode()


def test_attention_argument_errors(L):
    P = 1 << 12  # a 16-byte-aligned dummy address; nothing is launched on these paths
    assert L.sd_attention(P, P, P, P, 1, 1, 8, 8, 50, 1.0, None) == 2 and "head dim" in _err(L)
    assert L.sd_attention(P, P, P, P, -1, 1, 8, 8, 40, 1.0, None) == 1
    assert L.sd_attention(P, P, P, P, 1, 1, 8, 8, 40, float("nan"), None) == 1
    assert L.sd_attention(P, P, P, P, 1, 1, 8, 8, 40, -0.5, None) == 2 and "negative scale" in _err(L)
    assert L.sd_attention(P + 2, P, P, P, 1, 1, 8, 8, 40, 1.0, None) == 3
    assert L.sd_attention(P, P, P, P + 64, 1, 1, 8, 8, 40, 1.0, None) == 1 and "overlap" in _err(L)
    assert L.sd_attention(0, 0, 0, 0, 0, 8, 8, 8, 40, 1.0, None) == 0  # empty: no launch
    assert L.sd_attention(0, 0, 0, 0, 1, 1, 4, 0, 40, 1.0, None) == 1  # Lq >= 1 needs a key
    assert L.sd_attention(P, P, P, P, 1 << 31, 1, 8, 8, 40, 1.0, None) == 2


def test_attention_f16_argument_errors(L):
    P = 1 << 12
    assert L.sd_attention_f16(P, P, P, P, 1, 1, 8, 8, 50, 1.0, None) == 2  # head dim
    assert L.sd_attention_f16(P + 2, P, P, P, 1, 1, 8, 8, 40, 1.0, None) == 3  # misaligned
    assert L.sd_attention_f16(P, P, P, P + 64, 1, 1, 8, 8, 40, 1.0, None) == 1  # o overlaps q
    assert L.sd_attention_f16(0, 0, 0, 0, 0, 1, 8, 8, 40, 1.0, None) == 0


def test_attention_layout_argument_errors(L):
    P = 1 << 12
    assert L.sd_attention_layout(P, P + 4096, P + 8192, P + 12288, 1, 1, 8, 8, 40, 1.0, 2, 0, None) == 1  # dtype
    assert L.sd_attention_layout(P, P + 4096, P + 8192, P + 12288, 1, 1, 8, 8, 40, 1.0, 0, 2, None) == 1  # layout
    assert L.sd_attention_layout(P, P, P, P, 1, 1, 8, 8, 48, 1.0, 0, 1, None) == 2  # head dim
    assert L.sd_attention_layout(0, 0, 0, 0, 0, 1, 8, 8, 40, 1.0, 1, 1, None) == 0


def test_group_norm_argument_errors(L):
    P = 1 << 12
    assert L.sd_group_norm(P, P, P, P, 1, 30, 4, 4, 32, 1e-5, None) == 1  # 32 does not divide 30
    assert L.sd_group_norm(P, P, P, P, 1, 32, 4, 4, 32, 0.0, None) == 1   # eps must be > 0
    assert L.sd_group_norm(P, P, P, P + 8, 1, 32, 4, 4, 32, 1e-5, None) == 1  # partial overlap
    assert L.sd_group_norm(0, 0, 0, 0, 0, 32, 4, 4, 32, 1e-5, None) == 0


def test_group_norm_silu_argument_errors(L):
    P = 1 << 12
    assert L.sd_group_norm_silu(P, P, P, P + (1 << 20), 1, 32, 4, 4, 32, 1e-5, 2, None) == 1  # out_bf16 not 0/1
    assert L.sd_group_norm_silu(P, P, P, P, 1, 32, 4, 4, 32, 1e-5, 1, None) == 1  # bf16 output in place
    assert L.sd_group_norm_silu(P, P, P, P + 8, 1, 32, 4, 4, 32, 1e-5, 0, None) == 1  # partial overlap
    assert L.sd_group_norm_silu(P, P, P, P, 1, 30, 4, 4, 32, 1e-5, 0, None) == 1  # 32 does not divide 30
    assert L.sd_group_norm_silu(0, 0, 0, 0, 0, 32, 4, 4, 32, 1e-5, 1, None) == 0


def test_cfg_ddim_argument_errors(L):
    P = 1 << 12
    assert L.sd_cfg_ddim_step(P, P + 4096, P + 8192, P, 16, 7.5, 0.0, 0.5, None) == 1  # alpha_t = 0
    assert L.sd_cfg_ddim_step(P, P + 4096, P + 8192, P, 16, 7.5, 0.5, 1.5, None) == 1  # alpha_prev > 1
    assert L.sd_cfg_ddim_step(P, P + 4096, P + 8192, P + 4, 16, 7.5, 0.5, 0.6, None) == 1  # partial alias
    assert L.sd_cfg_ddim_step(P, P + 4096, P + 8192, P + 4096, 16, 7.5, 0.5, 0.6, None) == 1
    assert L.sd_cfg_ddim_step(0, 0, 0, 0, 0, 7.5, 0.5, 0.6, None) == 0


def test_dpmpp_argument_errors(L):
    P, n = 1 << 12, 16
    Q = [P + i * 4096 for i in range(6)]  # x, eu, ec, d_prev, x_out, d_out: disjoint
    f = L.sd_cfg_dpmpp_2m_step
    assert f(*Q, n, 7.5, 0.2, 0.3, 0.4, 3, None) == 1  # order must be 1 or 2
    assert f(*Q, n, 7.5, 0.2, 1.0, 1.0, 1, None) == 1  # alpha_t = 1: sigma_t = 0
    assert f(*Q, n, 7.5, 0.2, 0.3, 1.0, 2, None) == 1 and "first order" in _err(L)  # last step is order 1
    assert f(*Q, n, 7.5, 0.3, 0.3, 0.4, 2, None) == 1  # alpha_prev = alpha_t
    assert f(Q[0], Q[1], Q[2], 0, Q[4], Q[5], n, 7.5, 0.2, 0.3, 0.4, 2, None) == 1  # order 2 without history
    assert f(Q[0], Q[1], Q[2], Q[3], Q[4], Q[0], n, 7.5, 0.2, 0.3, 0.4, 2, None) == 1  # d_out overlaps x
    assert f(Q[0], Q[1], Q[2], Q[3], Q[3] + 4, Q[5], n, 7.5, 0.2, 0.3, 0.4, 2, None) == 1  # x_out over d_prev
    assert f(0, 0, 0, 0, 0, 0, 0, 7.5, 0.2, 0.3, 0.4, 1, None) == 0  # empty


def test_dpmpp_3m_argument_errors(L):
    P, n = 1 << 12, 16
    Q = [P + i * 4096 for i in range(7)]  # x, eu, ec, d_prev, d_prev2, x_out, d_out: disjoint
    f = L.sd_cfg_dpmpp_3m_step
    assert f(*Q, n, 7.5, 0.1, 0.2, 0.3, 1.0, None) == 1 and "first order" in _err(L)  # to sigma = 0
    assert f(*Q, n, 7.5, 0.2, 0.2, 0.3, 0.4, None) == 1  # equal noise levels
    assert f(Q[0], Q[1], Q[2], 0, Q[4], Q[5], Q[6], n, 7.5, 0.1, 0.2, 0.3, 0.4, None) == 1  # null history
    assert f(Q[0], Q[1], Q[2], Q[3], Q[4], Q[5], Q[3] + 4, n, 7.5, 0.1, 0.2, 0.3, 0.4, None) == 1  # partial alias
    assert f(Q[0], Q[1], Q[2], Q[3], Q[4], Q[5], Q[4], 0, 7.5, 0.1, 0.2, 0.3, 0.4, None) == 0  # d_out == d_prev2


def test_dpmpp_schedule_matches_the_oracle():
    import oracle
    ours, ref = sdk.dpmpp_2m_schedule(20), oracle.dpmpp_2m_schedule(20)
    assert [o for *_, o in ours] == [o for *_, o in ref]
    for a, b in zip(ours, ref):
        assert max(abs(x - y) for x, y in zip(a[:3], b[:3])) < 1e-13
    ours, ref = sdk.dpmpp_3m_schedule(20), oracle.dpmpp_3m_schedule(20)
    assert [o for *_, o in ours] == [o for *_, o in ref]
    for a, b in zip(ours, ref):
        assert max(abs(x - y) for x, y in zip(a[:4], b[:4])) < 1e-13


def test_binding_refuses_cpu_tensors(L):
    q = torch.zeros(1, 1, 8, 40, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        sdk.sd_attention(q, q, q)
    x = torch.zeros(1, 32, 4, 4)
    with pytest.raises(ValueError, match="CUDA"):
        sdk.sd_group_norm(x, torch.ones(32), torch.zeros(32))
    with pytest.raises(ValueError, match="CUDA"):
        sdk.sd_cfg_ddim_step(x, x, x, 7.5, 0.5, 0.6)


def test_schedule_tables_match_the_oracle():
    import oracle
    ours = sdk.ddim_schedule(20)
    ref = oracle.ddim_schedule(20)
    assert [t for t, _, _ in ours] == [t for t, _, _ in ref]
    for (_, a, p), (_, ra, rp) in zip(ours, ref):
        assert abs(a - ra) < 1e-13 and abs(p - rp) < 1e-13


def _ranges(L, items, nkv, grid, dh):
    import ctypes
    L.sd_debug_attention_ranges.argtypes = [ctypes.c_int64] * 4 + [ctypes.POINTER(ctypes.c_int64)]
    L.sd_debug_attention_ranges.restype = ctypes.c_int
    out = (ctypes.c_int64 * (grid + 1))()
    assert L.sd_debug_attention_ranges(items, nkv, grid, dh, out) == 0
    return list(out)


def _cost(a, b, nkv, m):
    segs = (b - 1) // nkv - a // nkv + 1
    return (b - a) + m[0] * (segs - 1) + (m[1] if a % nkv else 0) + (m[2] if b % nkv else 0)


@pytest.mark.parametrize("items,nkv,grid,dh", [(256, 32, 148, 40), (320, 32, 148, 64), (576, 72, 148, 40),
                                                (160, 5, 148, 40), (240, 5, 148, 80), (256, 1, 148, 40),
                                                (149, 3, 148, 160), (1000, 17, 132, 40)])
def test_persistent_grid_ranges(L, items, nkv, grid, dh):
    # host logic of the attention schedule: contiguous cover of all units, no range strictly inside
    # one item (an item spans at most two consecutive CTAs), empty ranges only at the end, and a
    # largest modelled cost no worse than equal unit counts
    u = _ranges(L, items, nkv, grid, dh)
    U = items * nkv
    assert u[0] == 0 and u[-1] == U and all(a <= b for a, b in zip(u, u[1:]))
    for a, b in zip(u, u[1:]):
        if b > a:
            assert not (a % nkv and b % nkv and a // nkv == (b - 1) // nkv), (a, b)
    nonempty = [b > a for a, b in zip(u, u[1:])]
    assert nonempty == sorted(nonempty, reverse=True)
    if nkv == 1:
        assert u == [U * c // grid for c in range(grid + 1)]
    else:
        m = (1.3, 0.5, 1.4) if dh == 64 else (1.0, 0.6, 0.9)
        worst = max(_cost(a, b, nkv, m) for a, b in zip(u, u[1:]) if b > a)
        even = max(_cost(U * c // grid, U * (c + 1) // grid, nkv, m) for c in range(grid))
        assert worst <= even + 1e-9


def test_persistent_grid_ranges_rejects_bad_arguments(L):
    import ctypes
    out = (ctypes.c_int64 * 300)()
    L.sd_debug_attention_ranges.argtypes = [ctypes.c_int64] * 4 + [ctypes.POINTER(ctypes.c_int64)]
    assert L.sd_debug_attention_ranges(10, 4, 20, 40, out) == 1  # grid > items
    assert L.sd_debug_attention_ranges(1000, 4, 257, 40, out) == 1  # grid > 256


def test_binding_argument_checks_on_the_host():
    # checks the bindings make before any device work (CPU tensors suffice to reach them)
    q16 = torch.zeros(1, 1, 8, 40, dtype=torch.float16)
    with pytest.raises(ValueError, match="all bf16 or all fp16"):
        sdk.sd_attention(q16, q16.to(torch.bfloat16), q16)
    with pytest.raises(ValueError, match="layout"):
        sdk.sd_attention(q16, q16, q16, layout="lbhd")
    with pytest.raises(ValueError, match="fp32"):
        sdk.sd_group_norm_silu(torch.zeros(1, 32, 4, 4, dtype=torch.float64), torch.ones(32), torch.zeros(32))
    x = torch.zeros(16)
    with pytest.raises(ValueError, match="order 2 needs d_prev"):
        sdk.sd_cfg_dpmpp_2m_step(x, x, x, None, 7.5, 0.2, 0.3, 0.4, 2)
    with pytest.raises(ValueError, match="one shape"):
        sdk.sd_cfg_dpmpp_3m_step(x, x, x, x, torch.zeros(8), 7.5, 0.1, 0.2, 0.3, 0.4)
    with pytest.raises(ValueError, match="CUDA"):
        sdk.sd_cfg_dpmpp_2m_step(x, x, x, None, 7.5, 0.2, 0.3, 0.4, 1)


def test_noalloc_binding_checks_type_and_shapes_on_the_host():
    # an fp16 tensor or mismatched k/v must never reach the bf16 kernel
    q = torch.zeros(1, 2, 8, 40, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="bf16"):
        sdk.sd_attention_noalloc(q.to(torch.float16), q.to(torch.float16), q.to(torch.float16))
    with pytest.raises(ValueError, match="bf16"):
        sdk.sd_attention_noalloc(q, q, q.to(torch.float16))
    with pytest.raises(ValueError, match="matching q"):
        sdk.sd_attention_noalloc(q, torch.zeros(1, 2, 9, 40, dtype=torch.bfloat16), q)
    with pytest.raises(ValueError, match="matching q"):
        sdk.sd_attention_noalloc(q, torch.zeros(1, 3, 8, 40, dtype=torch.bfloat16),
                                 torch.zeros(1, 3, 8, 40, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="4-D"):
        sdk.sd_attention_noalloc(q[0], q, q)
    with pytest.raises(ValueError, match="out"):
        sdk.sd_attention_noalloc(q, q, q, out=torch.zeros(1, 2, 8, 40, dtype=torch.float32))
    with pytest.raises(ValueError, match="CUDA"):
        sdk.sd_attention_noalloc(q, q, q)
