"""Oracle: scaled dot-product attention, fp64 (test infrastructure only).

What it computes: for every batch b, head h and query row i,
    s_ij = scale * sum_d Q[b,h,i,d] K[b,h,j,d]
    p_ij = exp(s_ij - max_j s_ij) / sum_j exp(s_ij - max_j s_ij)
    O[b,h,i,:] = sum_j p_ij V[b,h,j,:]
This is the plain softmax(Q K^T * scale) V that the flash-attention kernel of
"从零实现扩散模型推理引擎：Rust + wgpu 的 GPU 加速图像生成架构" §3.2 reaches by tiles: its online
recurrence (running max m, running sum l, rescaled output) equals this definition in exact
arithmetic, so the oracle is the definition itself. Cross-attention (§3.2: Q from the latent map,
K/V from the 77-token text context) is the same function with Lk = 77. No mask, no dropout.

Inputs are converted to fp64 exactly (bf16 and fp32 values are representable in fp64).
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor (possibly bf16): go through fp32, which is exact
        a = a.detach().to("cpu").float().numpy()
    return np.asarray(a, dtype=np.float64)


def softmax_weights(q, k, scale: float) -> np.ndarray:
    """Attention weights P[..., i, j] = softmax_j(scale * q_i . k_j) for q [..., Lq, dh], k [..., Lk, dh]."""
    q = _f64(q)
    k = _f64(k)
    s = scale * np.matmul(q, np.swapaxes(k, -1, -2))  # [..., Lq, Lk]
    s = s - s.max(axis=-1, keepdims=True)  # max subtraction: exp never overflows
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def attention(q, k, v, scale: float | None = None, row_block: int = 1024) -> np.ndarray:
    """softmax(Q K^T * scale) V for Q [B,h,Lq,dh], K/V [B,h,Lk,dh]; returns fp64 [B,h,Lq,dh].

    ``scale`` defaults to 1/sqrt(dh) with the true head dim. Rows are processed in blocks of
    ``row_block`` only to bound memory; the result does not depend on the blocking.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, H, Lq, dh = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dh)
    out = np.empty((B, H, Lq, v.shape[-1]), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, Lq, row_block):
                r1 = min(Lq, r0 + row_block)
                p = softmax_weights(q[b, h, r0:r1], k[b, h], scale)
                out[b, h, r0:r1] = p @ v[b, h]
    return out


def attention_rows(q, k, v, rows, scale: float | None = None) -> np.ndarray:
    """Oracle output for selected rows only: ``rows`` is an int array [n, 3] of (b, h, i).

    Returns fp64 [n, dh]. Used to check full-size launches at sampled outputs.
    """
    rows = np.asarray(rows, dtype=np.int64)
    dh = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(dh)
    out = np.empty((rows.shape[0], v.shape[-1]), dtype=np.float64)
    # group by (b, h) so each head's K and V are converted once
    keys = rows[:, 0] * q.shape[1] + rows[:, 1]
    for key in np.unique(keys):
        sel = np.nonzero(keys == key)[0]
        b, h = int(rows[sel[0], 0]), int(rows[sel[0], 1])
        kb = _f64(k[b, h])
        vb = _f64(v[b, h])
        qb = _f64(q[b, h][rows[sel, 2]])
        out[sel] = softmax_weights(qb, kb, scale) @ vb
    return out
