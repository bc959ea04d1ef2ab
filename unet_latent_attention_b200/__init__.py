"""Python binding of the sm_100a latent-diffusion hot-path library (``libsdk.so``).

Argument marshalling only: every step runs in the CUDA kernels behind the C ABI declared in
``include/sd_kernels.h``. PyTorch supplies device memory and the current CUDA stream. There is no
CPU fallback: if the library is missing or the tensors are not on a CUDA device, the calls raise.

    sd_group_norm(x, gamma, beta, groups=32, eps=1e-5, out=None)
    sd_group_norm_silu(x, gamma, beta, groups=32, eps=1e-5, out=None, out_dtype=None)
    sd_attention(q, k, v, scale=None, out=None)          (bf16 or fp16)
    sd_cfg_ddim_step(x, eps_u, eps_c, w, alpha_t, alpha_prev, out=None)
    sd_cfg_ddim_step_from_noise_pred(x, noise_pred, w, alpha_t, alpha_prev, out=None)
    sd_cfg_dpmpp_2m_step(x, eps_u, eps_c, d_prev, w, alpha_prev, alpha_t, alpha_next, order, out=None, d_out=None)
"""
from __future__ import annotations

import ctypes
import math
import os
import re

from .schedule import (ddim_schedule, dpmpp_2m_schedule, dpmpp_3m_schedule, karras_alpha_bars,  # noqa: F401
                       scaled_linear_alphas_cumprod)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdk.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "sd_kernels.h")

SD_OK = 0
STATUS_NAMES = {0: "SD_OK", 1: "SD_ERR_INVALID_ARG", 2: "SD_ERR_UNSUPPORTED", 3: "SD_ERR_MISALIGNED",
                4: "SD_ERR_CUDA", 5: "SD_ERR_TIMEOUT"}


class SDError(RuntimeError):
    """A non-zero sd_status from the library."""

    def __init__(self, func: str, status: int, detail: str):
        self.status = status
        super().__init__(f"{func}: {STATUS_NAMES.get(status, status)}: {detail}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsdk.so once (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m unet_latent_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i64, f32, f64, vp, c_int = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        L.sd_group_norm.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, f32, vp]
        L.sd_group_norm_silu.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, f32, c_int, vp]
        L.sd_attention.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, f32, vp]
        L.sd_attention_noalloc.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, f32, vp]
        L.sd_attention_f16.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, f32, vp]
        L.sd_attention_layout.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, f32, c_int, c_int, vp]
        L.sd_cfg_ddim_step.argtypes = [vp, vp, vp, vp, i64, f32, f64, f64, vp]
        L.sd_cfg_dpmpp_2m_step.argtypes = [vp, vp, vp, vp, vp, vp, i64, f32, f64, f64, f64, c_int, vp]
        L.sd_cfg_dpmpp_3m_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, f32, f64, f64, f64, f64, vp]
        L.sd_device_status.argtypes = [vp, c_int]
        L.sd_debug_set_fault.argtypes = [c_int]
        L.sd_debug_set_fault.restype = None
        for f in ("sd_group_norm", "sd_group_norm_silu", "sd_attention", "sd_attention_noalloc", "sd_attention_f16",
                  "sd_attention_layout",
                  "sd_cfg_ddim_step",
                  "sd_cfg_dpmpp_2m_step", "sd_cfg_dpmpp_3m_step", "sd_device_status"):
            getattr(L, f).restype = c_int
        L.sd_status_string.argtypes = [c_int]
        L.sd_status_string.restype = ctypes.c_char_p
        L.sd_last_error.argtypes = []
        L.sd_last_error.restype = ctypes.c_char_p
        L.sd_version.restype = c_int
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions that include/sd_kernels.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sd_[a-z_0-9]+)\s*\(", text)))


def _check(func: str, status: int) -> None:
    if status != SD_OK:
        raise SDError(func, status, lib().sd_last_error().decode(errors="replace"))


def _stream(t) -> int:
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


def _require_cuda(*ts) -> None:
    for t in ts:
        if not t.is_cuda:
            raise ValueError("sd kernels run on CUDA tensors only (no CPU fallback)")
        if not t.is_contiguous():
            raise ValueError("sd kernels take contiguous tensors")


def sd_group_norm(x, gamma, beta, groups: int = 32, eps: float = 1e-5, out=None):
    """GroupNorm of fp32 NCHW ``x`` with per-channel ``gamma``/``beta``; ``out`` may be ``x``."""
    import torch
    if x.dtype != torch.float32 or gamma.dtype != torch.float32 or beta.dtype != torch.float32:
        raise ValueError("sd_group_norm takes fp32 tensors")
    if x.dim() != 4:
        raise ValueError("x must be [B, C, H, W]")
    if out is None:
        out = torch.empty_like(x)
    _require_cuda(x, gamma, beta, out)
    B, C, H, W = x.shape
    if gamma.numel() != C or beta.numel() != C or out.shape != x.shape:
        raise ValueError("gamma/beta must have C elements and out the shape of x")
    _check("sd_group_norm", lib().sd_group_norm(x.data_ptr(), gamma.data_ptr(), beta.data_ptr(), out.data_ptr(),
                                                B, C, H, W, groups, eps, _stream(x)))
    return out


def sd_group_norm_silu(x, gamma, beta, groups: int = 32, eps: float = 1e-5, out=None, out_dtype=None):
    """SiLU(GroupNorm(x)) of fp32 NCHW ``x`` in one launch; the output is fp32 (``out`` may be ``x``)
    or bf16 (``out_dtype=torch.bfloat16``)."""
    import torch
    if x.dtype != torch.float32 or gamma.dtype != torch.float32 or beta.dtype != torch.float32:
        raise ValueError("sd_group_norm_silu takes fp32 x, gamma, beta")
    if x.dim() != 4:
        raise ValueError("x must be [B, C, H, W]")
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype or torch.float32, device=x.device)
    if out.dtype not in (torch.float32, torch.bfloat16) or out.shape != x.shape:
        raise ValueError("out must be fp32 or bf16 with the shape of x")
    _require_cuda(x, gamma, beta, out)
    B, C, H, W = x.shape
    if gamma.numel() != C or beta.numel() != C:
        raise ValueError("gamma/beta must have C elements")
    _check("sd_group_norm_silu", lib().sd_group_norm_silu(x.data_ptr(), gamma.data_ptr(), beta.data_ptr(),
                                                          out.data_ptr(), B, C, H, W, groups, eps,
                                                          1 if out.dtype == torch.bfloat16 else 0, _stream(x)))
    return out


def sd_attention(q, k, v, scale: float | None = None, out=None, layout: str = "bhld"):
    """softmax(q k^T * scale) v for q [B,h,Lq,dh], k/v [B,h,Lk,dh] (layout "bhld") or q [B,Lq,h,dh],
    k/v [B,Lk,h,dh] (layout "blhd"), all bf16 or all fp16 (the output has the type and layout of q);
    scale defaults to 1/sqrt(dh)."""
    import torch
    if q.dtype not in (torch.bfloat16, torch.float16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("sd_attention takes q, k, v all bf16 or all fp16")
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D")
    if layout not in ("bhld", "blhd"):
        raise ValueError("layout must be 'bhld' or 'blhd'")
    if layout == "blhd":
        B, Lq, Hh, dh = q.shape
        Lk = k.shape[1]
        if k.shape != (B, Lk, Hh, dh) or v.shape != k.shape:
            raise ValueError("k and v must be [B, Lk, heads, dh] matching q")
    else:
        B, Hh, Lq, dh = q.shape
        Lk = k.shape[2]
        if k.shape[:2] != (B, Hh) or v.shape != k.shape or k.shape[3] != dh:
            raise ValueError("k and v must be [B, heads, Lk, dh] matching q")
    if out is None:
        out = torch.empty_like(q)
    _require_cuda(q, k, v, out)
    if out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must have the shape and type of q")
    if scale is None:
        scale = 1.0 / math.sqrt(dh)
    f16, blhd = q.dtype == torch.float16, layout == "blhd"
    if not f16 and not blhd:
        st = lib().sd_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hh, Lq, Lk, dh, scale,
                                _stream(q))
    else:
        st = lib().sd_attention_layout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hh, Lq, Lk, dh,
                                       scale, int(f16), int(blhd), _stream(q))
    _check("sd_attention", st)
    return out


def sd_attention_noalloc(q, k, v, scale: float | None = None, out=None):
    """sd_attention (bf16, [B, heads, L, dh]) without any device allocation by the library: its
    split-item scratch is a fixed 16 MiB device array instead of a cudaMalloc'd workspace.

    For callers that cannot let a library call cudaMalloc: inside CUDA-graph capture, under a
    framework that owns all device memory, or in loops that cannot absorb cudaMalloc's implicit
    synchronisation. Pass ``out`` to avoid the allocation of the output tensor as well. Calls that
    overlap on the GPU race on the shared scratch.
    """
    import torch
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise ValueError("sd_attention_noalloc takes bf16 q, k, v")
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, heads, L, dh]")
    B, Hh, Lq, dh = q.shape
    Lk = k.shape[2]
    if k.shape != (B, Hh, Lk, dh) or v.shape != k.shape:
        raise ValueError("k and v must be [B, heads, Lk, dh] matching q")
    if out is None:
        out = torch.empty_like(q)
    if out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must have the shape and type of q")
    _require_cuda(q, k, v, out)
    if scale is None:
        scale = 1.0 / math.sqrt(dh)
    _check("sd_attention_noalloc", lib().sd_attention_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                              out.data_ptr(), B, Hh, Lq, Lk, dh, scale,
                                                              _stream(q)))
    return out


def sd_cfg_ddim_step(x, eps_u, eps_c, w: float, alpha_t: float, alpha_prev: float, out=None):
    """x' = DDIM(eta=0) step of fp32 latent x with guided noise eps_u + w (eps_c - eps_u); out may be x."""
    import torch
    for t in (x, eps_u, eps_c):
        if t.dtype != torch.float32:
            raise ValueError("sd_cfg_ddim_step takes fp32 tensors")
    if eps_u.shape != x.shape or eps_c.shape != x.shape:
        raise ValueError("eps_u and eps_c must have the shape of x")
    if out is None:
        out = torch.empty_like(x)
    _require_cuda(x, eps_u, eps_c, out)
    _check("sd_cfg_ddim_step", lib().sd_cfg_ddim_step(x.data_ptr(), eps_u.data_ptr(), eps_c.data_ptr(),
                                                      out.data_ptr(), x.numel(), w, alpha_t, alpha_prev,
                                                      _stream(x)))
    return out


def sd_cfg_ddim_step_from_noise_pred(x, noise_pred, w: float, alpha_t: float, alpha_prev: float, out=None):
    """Same step taking the UNet output for the batch [uncond, cond] (uncond half first)."""
    eps_u, eps_c = noise_pred.chunk(2, dim=0)
    return sd_cfg_ddim_step(x, eps_u, eps_c, w, alpha_t, alpha_prev, out=out)


def sd_cfg_dpmpp_2m_step(x, eps_u, eps_c, d_prev, w: float, alpha_prev: float, alpha_t: float, alpha_next: float,
                         order: int, out=None, d_out=None):
    """Guided DPM-Solver++(2M) step; returns (x_next, d) where d is this step's data prediction (the
    history for the next step). ``d_prev`` is the previous step's d (unused, may be None, for order 1);
    ``out`` may be ``x`` and ``d_out`` may be ``d_prev``."""
    import torch
    for t in (x, eps_u, eps_c) + ((d_prev,) if d_prev is not None else ()):
        if t.dtype != torch.float32 or t.shape != x.shape:
            raise ValueError("sd_cfg_dpmpp_2m_step takes fp32 tensors of one shape")
    if order == 2 and d_prev is None:
        raise ValueError("order 2 needs d_prev")
    out = torch.empty_like(x) if out is None else out
    d_out = torch.empty_like(x) if d_out is None else d_out
    _require_cuda(x, eps_u, eps_c, out, d_out, *((d_prev,) if d_prev is not None else ()))
    _check("sd_cfg_dpmpp_2m_step", lib().sd_cfg_dpmpp_2m_step(
        x.data_ptr(), eps_u.data_ptr(), eps_c.data_ptr(), d_prev.data_ptr() if d_prev is not None else None,
        out.data_ptr(), d_out.data_ptr(), x.numel(), w, alpha_prev, alpha_t, alpha_next, int(order), _stream(x)))
    return out, d_out


def sd_cfg_dpmpp_3m_step(x, eps_u, eps_c, d_prev, d_prev2, w: float, alpha_prev2: float, alpha_prev: float,
                         alpha_t: float, alpha_next: float, out=None, d_out=None):
    """Guided third-order multistep DPM-Solver++ step; returns (x_next, d). ``out`` may be ``x``;
    ``d_out`` may be ``d_prev`` or ``d_prev2``."""
    import torch
    for t in (x, eps_u, eps_c, d_prev, d_prev2):
        if t.dtype != torch.float32 or t.shape != x.shape:
            raise ValueError("sd_cfg_dpmpp_3m_step takes fp32 tensors of one shape")
    out = torch.empty_like(x) if out is None else out
    d_out = torch.empty_like(x) if d_out is None else d_out
    _require_cuda(x, eps_u, eps_c, d_prev, d_prev2, out, d_out)
    _check("sd_cfg_dpmpp_3m_step", lib().sd_cfg_dpmpp_3m_step(
        x.data_ptr(), eps_u.data_ptr(), eps_c.data_ptr(), d_prev.data_ptr(), d_prev2.data_ptr(), out.data_ptr(),
        d_out.data_ptr(), x.numel(), w, alpha_prev2, alpha_prev, alpha_t, alpha_next, _stream(x)))
    return out, d_out


def sd_device_status(stream=None, reset: bool = True) -> int:
    """Synchronise and read the device status word; raises SDError on a recorded device failure."""
    s = stream.cuda_stream if stream is not None else 0
    st = lib().sd_device_status(s, 1 if reset else 0)
    _check("sd_device_status", st)
    return st


def sd_debug_set_fault(flags: int) -> None:
    """Test hook: bit 0 makes attention launches skip their first V tile (the bounded wait expires)."""
    lib().sd_debug_set_fault(int(flags))
