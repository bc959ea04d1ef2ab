"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and the benchmark.

This module holds no arithmetic of the attention, GroupNorm or guidance/DDIM methods: it only
draws reproducible N(0, 1) numbers and names the workload shapes. Both sides of every parity
check (the CPU oracle under ``oracle/`` and the CUDA library) receive the same arrays from here.

Generator: the splitmix64 sequence (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014) used counter-style, output k of stream ``seed`` being
mix(seed + (k + 1) * 0x9E3779B97F4A7C15); pairs of outputs become two normals through the
Box-Muller transform (Box and Muller, 1958). Stream seeds follow ``1000 * workload + tensor id``.
"""
from __future__ import annotations

import dataclasses
import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of the splitmix64 stream whose initial state is ``seed``."""
    k = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + k * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def normal(shape, seed: int, dtype=np.float32) -> np.ndarray:
    """N(0, 1) samples of ``shape`` from stream ``seed`` (Box-Muller over splitmix64 pairs)."""
    n = int(np.prod(shape, dtype=np.int64))
    out = np.empty(n, dtype=np.float64)
    npairs = (n + 1) // 2
    two_pi = 2.0 * np.pi
    for p0 in range(0, npairs, _CHUNK):
        p1 = min(npairs, p0 + _CHUNK)
        bits = splitmix64(seed, 2 * p0, 2 * (p1 - p0))
        mant = (bits >> np.uint64(11)).astype(np.float64)
        u1 = (mant[0::2] + 1.0) * (2.0 ** -53)  # (0, 1]
        u2 = mant[1::2] * (2.0 ** -53)          # [0, 1)
        r = np.sqrt(-2.0 * np.log(u1))
        z = np.empty(2 * (p1 - p0), dtype=np.float64)
        z[0::2] = r * np.cos(two_pi * u2)
        z[1::2] = r * np.sin(two_pi * u2)
        lo = 2 * p0
        hi = min(n, 2 * p1)
        out[lo:hi] = z[: hi - lo]
    return out.reshape(shape).astype(dtype)


def to_bf16_exact(a: np.ndarray):
    """Round an fp32 array to bf16 (round-to-nearest-even) and return a torch bf16 tensor (CPU)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def to_f16_exact(a: np.ndarray):
    """Round an fp32 array to IEEE fp16 (round-to-nearest-even) and return a torch fp16 tensor (CPU)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.float16)


# ---------------------------------------------------------------------------------------------
# Workloads: Stable Diffusion UNet shapes. Attention tensors are [B, heads, L, dh]; GroupNorm
# tensors are NCHW fp32; guidance/DDIM tensors are latents [n_img, 4, h, w] fp32.
# ---------------------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class AttnShape:
    B: int
    heads: int
    Lq: int
    Lk: int
    dh: int

    @property
    def flops(self) -> int:
        # two contractions of Lq x Lk x dh multiply-adds each (true dh, no padding)
        return 4 * self.B * self.heads * self.Lq * self.Lk * self.dh


@dataclasses.dataclass(frozen=True)
class GNShape:
    B: int
    C: int
    H: int
    W: int
    groups: int = 32
    eps: float = 1e-5

    @property
    def bytes(self) -> int:
        return 8 * self.B * self.C * self.H * self.W  # fp32 read once + written once


@dataclasses.dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    attention: tuple  # of (label, AttnShape)
    group_norm: tuple  # of (label, GNShape)
    latent: tuple  # [n_img, 4, h, w] of the guided latent update
    ddim_steps: int = 1
    guidance: float = 7.5


WORKLOADS = {
    1: Workload(1, "SD1.5 16x16-latent toy block",
                (("self", AttnShape(2, 8, 256, 256, 40)), ("cross", AttnShape(2, 8, 256, 77, 40))),
                (("gn", GNShape(2, 320, 16, 16)),), (1, 4, 16, 16)),
    2: Workload(2, "SD1.5 512x512 top level",
                (("self", AttnShape(2, 8, 4096, 4096, 40)), ("cross", AttnShape(2, 8, 4096, 77, 40))),
                (("gn", GNShape(2, 320, 64, 64)),), (1, 4, 64, 64)),
    3: Workload(3, "SD1.5 inner levels",
                (("self_l1", AttnShape(2, 8, 1024, 1024, 80)), ("cross_l1", AttnShape(2, 8, 1024, 77, 80)),
                 ("self_l2", AttnShape(2, 8, 256, 256, 160)), ("cross_l2", AttnShape(2, 8, 256, 77, 160))),
                (("gn_l1", GNShape(2, 640, 32, 32)), ("gn_l2", GNShape(2, 1280, 16, 16))), (1, 4, 32, 32)),
    4: Workload(4, "SDXL 1024x1024 levels",
                (("self_l1", AttnShape(2, 10, 4096, 4096, 64)), ("cross_l1", AttnShape(2, 10, 4096, 77, 64)),
                 ("self_l2", AttnShape(2, 20, 1024, 1024, 64)), ("cross_l2", AttnShape(2, 20, 1024, 77, 64))),
                (("gn", GNShape(2, 640, 64, 64)),), (1, 4, 128, 128)),
    5: Workload(5, "Batched serving SD1.5 768x768",
                (("self", AttnShape(16, 8, 9216, 9216, 40)), ("cross", AttnShape(16, 8, 9216, 77, 40))),
                (), (8, 4, 96, 96), ddim_steps=20),
}

# tensor ids inside a workload's seed space (seed = 1000 * wid + id)
_TID = {"q": 1, "k": 2, "v": 3, "gn_x": 11, "gn_gamma": 12, "gn_beta": 13,
        "lat_x": 21, "eps_u": 22, "eps_c": 23}


def seed_of(wid: int, tensor: str, sub: int = 0) -> int:
    """Stream seed of a named tensor; ``sub`` separates several tensors of one kind (levels, steps)."""
    return 1000 * wid + _TID[tensor] + (sub << 32)


def attention_qkv(wid: int, shape: AttnShape, sub: int = 0, q_scale: float = 1.0):
    """bf16 Q, K, V (torch CPU tensors) drawn N(0, 1) then rounded to bf16; Q optionally scaled."""
    q = normal((shape.B, shape.heads, shape.Lq, shape.dh), seed_of(wid, "q", sub)) * np.float32(q_scale)
    k = normal((shape.B, shape.heads, shape.Lk, shape.dh), seed_of(wid, "k", sub))
    v = normal((shape.B, shape.heads, shape.Lk, shape.dh), seed_of(wid, "v", sub))
    return to_bf16_exact(q), to_bf16_exact(k), to_bf16_exact(v)


def group_norm_inputs(wid: int, shape: GNShape, sub: int = 0):
    """fp32 x ~ N(0,1) [B,C,H,W]; gamma = 1 + 0.1 N(0,1); beta = 0.1 N(0,1) (numpy arrays)."""
    x = normal((shape.B, shape.C, shape.H, shape.W), seed_of(wid, "gn_x", sub))
    gamma = (1.0 + 0.1 * normal((shape.C,), seed_of(wid, "gn_gamma", sub), np.float64)).astype(np.float32)
    beta = (0.1 * normal((shape.C,), seed_of(wid, "gn_beta", sub), np.float64)).astype(np.float32)
    return x, gamma, beta


def latent_inputs(wid: int, latent_shape, step: int = 0):
    """fp32 latent x and the two noise predictions (uncond, cond) of one step, all N(0, 1)."""
    x = normal(latent_shape, seed_of(wid, "lat_x"))
    eu = normal(latent_shape, seed_of(wid, "eps_u", step))
    ec = normal(latent_shape, seed_of(wid, "eps_c", step))
    return x, eu, ec
