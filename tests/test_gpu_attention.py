"""GPU parity of sd_attention against the fp64 oracle on seeded inputs.

Gates (bf16 in, fp32 accumulate), both on every comparison:
  * the stated tolerance: max-abs error <= 2e-2 and mean-abs error <= 2e-3;
  * an internal bar: mean-abs error <= 1% of the RMS of the oracle's output over the compared
    values. At Lk = 4096 |O| is about 0.026 and the stated 2e-3 is ~8% of it; dropping one key tile
    moves O by ~13x the internal bar (tests/test_oracle_attention.py pins that on the CPU).
Sizes span several 128x128 tiles with ragged tails; full workload sizes are checked on sampled
rows that the oracle computes one by one. Achieved errors are logged (SD_PARITY_LOG)."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth_inputs as si
import unet_latent_attention_b200 as sdk
from conftest import max_abs_mean_abs, record_parity

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
INTERNAL_MEAN_FRAC = 0.01  # internal bar: mean-abs error <= 1% of the output's RMS


def _run(q, k, v, dev, scale=None):
    o = sdk.sd_attention(q.to(dev), k.to(dev), v.to(dev), scale=scale)
    sdk.sd_device_status()
    return o.float().cpu().numpy()


def _check(o, ref, max_abs=MAX_ABS, mean_abs=MEAN_ABS, name=None):
    mx, mn = max_abs_mean_abs(o, ref)
    rms = float(np.sqrt(np.mean(np.square(np.asarray(ref, np.float64))))) if np.size(ref) else 0.0
    assert np.isfinite(o).all()
    record_parity(name or os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], max_abs=mx, mean_abs=mn,
                  rms_ref=rms)
    assert mx <= max_abs and mn <= mean_abs, (mx, mn)
    assert mn <= INTERNAL_MEAN_FRAC * rms, ("internal bar", mn, rms)
    return mx, mn


def _qkv(B, H, Lq, Lk, dh, seed, q_scale=1.0):
    q = si.to_bf16_exact(si.normal((B, H, Lq, dh), seed) * np.float32(q_scale))
    k = si.to_bf16_exact(si.normal((B, H, Lk, dh), seed + 1))
    v = si.to_bf16_exact(si.normal((B, H, Lk, dh), seed + 2))
    return q, k, v


@pytest.mark.parametrize("dh", [40, 64, 80, 160])
@pytest.mark.parametrize("Lq,Lk", [(1, 1), (7, 77), (129, 255), (300, 77), (513, 640), (256, 1)])
def test_small_shapes(cuda, dh, Lq, Lk):
    q, k, v = _qkv(2, 3, Lq, Lk, dh, 7000 + dh + Lq + Lk)
    o = _run(q, k, v, cuda)
    _check(o, oracle.attention(q, k, v))


@pytest.mark.parametrize("dh", [40, 64, 80, 160])
def test_single_key_returns_v(cuda, dh):
    q, k, v = _qkv(1, 2, 200, 1, dh, 100 + dh)
    o = _run(q, k, v, cuda)
    np.testing.assert_array_equal(o, np.broadcast_to(v.float().numpy(), o.shape))


@pytest.mark.parametrize("dh", [40, 64, 80, 160])
def test_zero_query_gives_mean_of_v(cuda, dh):
    _, k, v = _qkv(1, 2, 1, 300, dh, 200 + dh)
    q = torch.zeros(1, 2, 130, dh, dtype=torch.bfloat16)
    o = _run(q, k, v, cuda)
    ref = np.broadcast_to(v.double().numpy().mean(axis=2, keepdims=True), o.shape)
    _check(o, ref, 4e-3, 1e-3)


@pytest.mark.parametrize("dh", [40, 64])
def test_peaky_scores_exercise_rescaling(cuda, dh):
    # Q x 4 makes the running max jump across key tiles, so the lazy O correction runs
    q, k, v = _qkv(2, 2, 384, 1000, dh, 300 + dh, q_scale=4.0)
    o = _run(q, k, v, cuda)
    _check(o, oracle.attention(q, k, v))


def test_custom_scale(cuda):
    q, k, v = _qkv(1, 2, 200, 300, 64, 400)
    o = _run(q, k, v, cuda, scale=0.05)
    _check(o, oracle.attention(q, k, v, scale=0.05))


def _sampled_rows(shape, n, seed):
    rng = np.random.default_rng(seed)
    rows = np.stack([rng.integers(0, shape.B, n), rng.integers(0, shape.heads, n), rng.integers(0, shape.Lq, n)], 1)
    # always include the first and last rows of the first and last heads (tile edges, ragged tail)
    edge = np.array([[0, 0, 0], [shape.B - 1, shape.heads - 1, shape.Lq - 1], [0, 0, 127], [0, 0, 128]])
    return np.concatenate([edge[edge[:, 2] < shape.Lq], rows])


CASES = [(w.wid, label, s) for w in si.WORKLOADS.values() for label, s in w.attention]


@pytest.mark.parametrize("wid,label,shape", CASES, ids=[f"w{w}-{l}" for w, l, _ in CASES])
def test_workload_shapes(cuda, wid, label, shape):
    q, k, v = si.attention_qkv(wid, shape, sub=CASES.index((wid, label, shape)))
    o = _run(q, k, v, cuda)
    if shape.B * shape.heads * shape.Lq * shape.Lk <= (1 << 26):
        ref = oracle.attention(q, k, v)
        _check(o, ref)
    else:
        rows = _sampled_rows(shape, 96, wid)
        ref = oracle.attention_rows(q, k, v, rows)
        _check(o[rows[:, 0], rows[:, 1], rows[:, 2]], ref)


@pytest.mark.parametrize("dh,heads,Lq,Lk", [(40, 80, 256, 640), (64, 80, 256, 1000), (80, 80, 256, 700),
                                            (160, 120, 128, 300), (40, 96, 300, 129)])
def test_split_items_persistent_schedule(cuda, dh, heads, Lq, Lk):
    # more query-tile items than SMs: the persistent grid splits items between neighbouring CTAs
    # and merges the two partial results; compared in full with the oracle
    q, k, v = _qkv(2, heads, Lq, Lk, dh, 9000 + dh + Lk)
    o = _run(q, k, v, cuda)
    _check(o, oracle.attention(q, k, v))


@pytest.mark.parametrize("dh,heads,Lq,Lk", [(40, 80, 256, 640), (64, 80, 256, 1000), (80, 80, 256, 700),
                                            (160, 120, 128, 300)])
def test_split_items_either_piece_may_merge(cuda, dh, heads, Lq, Lk):
    # test hook bit 1 holds the tail pieces back, so the head pieces publish and the tail pieces
    # merge: the output must be bit-identical to the usual order (one fixed merge order)
    q, k, v = _qkv(2, heads, Lq, Lk, dh, 9200 + dh + Lk)
    qd, kd, vd = q.to(cuda), k.to(cuda), v.to(cuda)
    usual = sdk.sd_attention(qd, kd, vd)
    sdk.sd_device_status()
    try:
        sdk.sd_debug_set_fault(2)
        reversed_ = sdk.sd_attention(qd, kd, vd)
        sdk.sd_device_status()
    finally:
        sdk.sd_debug_set_fault(0)
    assert torch.equal(usual, reversed_)
    _check(reversed_.float().cpu().numpy(), oracle.attention(q, k, v))


def test_split_items_after_other_head_dims(cuda):
    # every head dim's launches share one hand-off workspace; each must leave the counters at zero
    # and find them at zero whatever configuration ran before it (the slots of one configuration
    # must never lie where another expects its counters)
    for dh, heads, Lq, Lk in [(64, 80, 256, 1000), (40, 80, 256, 640), (80, 80, 256, 700), (160, 120, 128, 300),
                              (40, 96, 300, 129), (64, 80, 256, 1000)]:
        q, k, v = _qkv(2, heads, Lq, Lk, dh, 9400 + dh + Lk)
        o = _run(q, k, v, cuda)
        _check(o, oracle.attention(q, k, v))


@pytest.mark.parametrize("dh,B,heads,Lq,Lk", [(40, 1, 1, 2048, 4096), (64, 1, 2, 700, 3000), (80, 1, 1, 256, 2000)])
def test_fewer_items_than_sms(cuda, dh, B, heads, Lq, Lk):
    # a few long items: the grid shrinks to one CTA per item (no split), each streaming many K/V
    # tiles with a ragged last one
    q, k, v = _qkv(B, heads, Lq, Lk, dh, 9500 + dh + Lq + Lk)
    o = _run(q, k, v, cuda)
    _check(o, oracle.attention(q, k, v))


def test_repeated_launches_reuse_the_hand_off_flags(cuda):
    # the split hand-off flags must return to zero after every launch (graph replays rely on it)
    q, k, v = _qkv(2, 80, 256, 640, 40, 9100)
    ref = oracle.attention(q, k, v)
    qd, kd, vd = q.to(cuda), k.to(cuda), v.to(cuda)
    for _ in range(3):
        o = sdk.sd_attention(qd, kd, vd)
        sdk.sd_device_status()
        _check(o.float().cpu().numpy(), ref)


@pytest.mark.parametrize("dh", [40, 64, 80, 160])
@pytest.mark.parametrize("B,heads,Lq,Lk", [(2, 300, 100, 77), (1, 7, 1000, 80), (2, 4, 200, 81), (3, 5, 1, 77),
                                           (2, 37, 129, 50)])
def test_short_key_sequences(cuda, dh, B, heads, Lq, Lk):
    # Lk <= 80 takes the resident-K/V kernel: CTA ranges that cross several heads (K/V buffers
    # reused), the 80-key boundary, a single query row, ragged query tiles; Lk = 81 takes the
    # general kernel's 96-key tile
    q, k, v = _qkv(B, heads, Lq, Lk, dh, 9300 + dh + Lq + Lk)
    o = _run(q, k, v, cuda)
    _check(o, oracle.attention(q, k, v))


LONG_TEXT = [si.AttnShape(2, 8, 4096, 256, 40), si.AttnShape(2, 8, 4096, 512, 40),
             si.AttnShape(2, 10, 1024, 256, 64), si.AttnShape(2, 10, 1024, 512, 64)]


@pytest.mark.parametrize("shape", LONG_TEXT, ids=[f"Lk{s.Lk}-dh{s.dh}" for s in LONG_TEXT])
def test_long_text_cross_attention(cuda, shape):
    # text contexts of 256 and 512 tokens (longer-text encoders): the key sequence spans 2-4 key
    # tiles of the online softmax; sampled rows against the oracle
    q, k, v = si.attention_qkv(6, shape, sub=shape.Lk + shape.dh)
    o = _run(q, k, v, cuda)
    rows = _sampled_rows(shape, 96, shape.Lk)
    _check(o[rows[:, 0], rows[:, 1], rows[:, 2]], oracle.attention_rows(q, k, v, rows))


# ---- fp16 tensors (sd_attention_f16), same gate as bf16

def _qkv16(B, H, Lq, Lk, dh, seed):
    return (si.to_f16_exact(si.normal((B, H, Lq, dh), seed)), si.to_f16_exact(si.normal((B, H, Lk, dh), seed + 1)),
            si.to_f16_exact(si.normal((B, H, Lk, dh), seed + 2)))


@pytest.mark.parametrize("dh", [40, 64, 80, 160])
@pytest.mark.parametrize("Lq,Lk", [(7, 77), (129, 255), (513, 640)])
def test_fp16_small_shapes(cuda, dh, Lq, Lk):
    q, k, v = _qkv16(2, 3, Lq, Lk, dh, 12000 + dh + Lq + Lk)
    o = sdk.sd_attention(q.to(cuda), k.to(cuda), v.to(cuda))
    sdk.sd_device_status()
    assert o.dtype == torch.float16
    _check(o.float().cpu().numpy(), oracle.attention(q, k, v))


def test_fp16_single_key_returns_v(cuda):
    q, k, v = _qkv16(1, 2, 200, 1, 40, 12100)
    o = sdk.sd_attention(q.to(cuda), k.to(cuda), v.to(cuda))
    sdk.sd_device_status()
    np.testing.assert_array_equal(o.float().cpu().numpy(), np.broadcast_to(v.float().numpy(), o.shape))


@pytest.mark.parametrize("dh,heads,Lq,Lk", [(40, 8, 4096, 4096), (64, 10, 1024, 1024), (40, 8, 4096, 77)])
def test_fp16_sd_shapes(cuda, dh, heads, Lq, Lk):
    # SD1.5 / SDXL self- and cross-attention shapes, sampled rows (split items included)
    shape = si.AttnShape(2, heads, Lq, Lk, dh)
    q, k, v = _qkv16(2, heads, Lq, Lk, dh, 12200 + dh + Lk)
    o = sdk.sd_attention(q.to(cuda), k.to(cuda), v.to(cuda))
    sdk.sd_device_status()
    rows = _sampled_rows(shape, 96, 12300 + dh)
    _check(o.float().cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]], oracle.attention_rows(q, k, v, rows))


def test_mixed_types_are_refused(cuda):
    q = torch.zeros(1, 1, 8, 40, dtype=torch.float16, device=cuda)
    with pytest.raises(ValueError):
        sdk.sd_attention(q, q.to(torch.bfloat16), q)


# ---- [B, L, heads, dh] layout (sd_attention_layout, layout 1), bf16 and fp16

@pytest.mark.parametrize("f16", [False, True], ids=["bf16", "fp16"])
@pytest.mark.parametrize("dh,heads,Lq,Lk", [(40, 3, 300, 77), (64, 5, 513, 640), (80, 2, 129, 255), (160, 3, 200, 300),
                                            (40, 80, 256, 640)])
def test_blhd_layout(cuda, f16, dh, heads, Lq, Lk):
    rnd = si.to_f16_exact if f16 else si.to_bf16_exact
    seed = 13000 + dh + heads + Lk
    q = rnd(si.normal((2, Lq, heads, dh), seed))
    k = rnd(si.normal((2, Lk, heads, dh), seed + 1))
    v = rnd(si.normal((2, Lk, heads, dh), seed + 2))
    o = sdk.sd_attention(q.to(cuda), k.to(cuda), v.to(cuda), layout="blhd")
    sdk.sd_device_status()
    assert o.shape == q.shape and o.dtype == q.dtype
    ref = oracle.attention(q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3))
    _check(o.float().cpu().numpy().transpose(0, 2, 1, 3), ref)
