"""fp64 oracle for the rotary-embedding + QK-norm prologue of attention.

TEST INFRASTRUCTURE, like the rest of this package: only ``tests/``,
``__graft_entry__.smoke()`` and the benchmark's CPU legs may use it.

What it computes (apidog guide "Train your own ChatGPT", section 1 "GPT model",
architecture features; and the nanochat overview's list of architecture choices):
the model rotates queries and keys with rotary embeddings (RoPE, no learned
position embedding) and normalises them (QK norm, an RMSNorm without learnable
parameters) before attention.  The pages name both steps but print no formula;
this module takes the plainest reading, written out here:

* RoPE (RoFormer): the head vector x in R^D is split into halves x1 = x[:D/2],
  x2 = x[D/2:]; pair i = (x1[i], x2[i]) is rotated by the angle pos * theta_i,
  theta_i = base^(-2i/D):  y1 = x1 cos - x2 sin,  y2 = x1 sin + x2 cos.
* QK norm: y / sqrt(mean(y^2) + eps) over the head dimension.

A rotation keeps the vector's length, so the two steps commute; the order is not
a reading.  The position of a token is its index in its sequence (training and
prefill: cache_len[b] + t; decode: cache_len[b] - 1, the new token's slot).
The model's activations are bf16, so the rotated, normalised q and k that attention
reads are bf16 values: the compositions below round them (to nearest, ties to even)
before the attention step.

Functions take bf16 bit patterns (uint16) or float64 and return float64.
"""
from __future__ import annotations

import numpy as np

from .swa_oracle import oracle_bwd, oracle_decode, oracle_fwd, oracle_prefill


def _f64(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if x.dtype != np.float64:
        raise TypeError("inputs must be bf16 bits (uint16) or float64")
    return x


def round_bf16(x):
    """x (float64) rounded to the nearest bf16 value, ties to even.  The float64 -> float32 step
    rounds to odd (truncate, then set the last bit when inexact), so the final rounding to bf16's
    8 significant bits is the correct one (no double rounding)."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    over = np.abs(f.astype(np.float64)) > np.abs(x)
    f = np.where(over, np.nextafter(f, np.float32(0)), f).astype(np.float32)   # truncated toward zero
    inexact = (f.astype(np.float64) != x).astype(np.uint64)
    b = np.ascontiguousarray(f).view(np.uint32).astype(np.uint64) | inexact
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def rope_angles(pos, D: int, base: float = 10000.0):
    """Angles pos * theta_i, theta_i = base^(-2i/D), i < D/2: shape pos.shape + (D/2,)."""
    i = np.arange(D // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / D)
    return np.asarray(pos, dtype=np.float64)[..., None] * theta


def oracle_rope_qknorm(x, pos, eps: float, base: float = 10000.0):
    """RoPE then RMS normalisation of every head vector.

    x [..., H, D]; pos broadcastable to x.shape[:-2] (one position per token).
    Returns float64 of x's shape."""
    x = _f64(x)
    D = x.shape[-1]
    d = D // 2
    ang = rope_angles(pos, D, base)[..., None, :]          # [..., 1, D/2], shared by the heads
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :d], x[..., d:]
    y = np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)
    return y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)


def oracle_rope_qknorm_bwd(x, pos, dy, eps: float, base: float = 10000.0):
    """Vector-Jacobian product of oracle_rope_qknorm with respect to x (fp64 autograd on the
    forward written with torch CPU ops, the same steps as oracle_rope_qknorm)."""
    import torch

    x = torch.tensor(_f64(x), dtype=torch.float64, requires_grad=True)
    D = x.shape[-1]
    d = D // 2
    ang = torch.tensor(rope_angles(pos, D, base), dtype=torch.float64)[..., None, :]
    c, s = torch.cos(ang), torch.sin(ang)
    x1, x2 = x[..., :d], x[..., d:]
    y = torch.cat([x1 * c - x2 * s, x1 * s + x2 * c], dim=-1)
    y = y / torch.sqrt(torch.mean(y * y, dim=-1, keepdim=True) + eps)
    y.backward(torch.tensor(_f64(dy), dtype=torch.float64))
    return x.grad.numpy()


def oracle_fwd_rope(q, k, v, W: int, eps: float, base: float = 10000.0, scale: float | None = None):
    """Training forward with the prologue: attention of rope_qknorm(q), rope_qknorm(k) (token t of
    every sequence at position t, rounded to bf16) and v.  Returns (o, lse) float64."""
    T = np.asarray(q).shape[1]
    pos = np.arange(T)[None, :]
    qr = round_bf16(oracle_rope_qknorm(q, pos, eps, base))
    kr = round_bf16(oracle_rope_qknorm(k, pos, eps, base))
    return oracle_fwd(qr, kr, _f64(v), W, scale)


def oracle_bwd_rope(q, k, v, do, W: int, eps: float, base: float = 10000.0, scale: float | None = None):
    """Training backward with the prologue: the attention backward at the rotated, normalised
    (bf16-rounded) q and k, then each of dq, dk taken back through rotate-and-normalise at the raw
    q, k (the rounding to bf16 passes gradients through unchanged, as a cast does in training).
    Returns (dq, dk, dv) float64, dq and dk with respect to the raw q and k."""
    T = np.asarray(q).shape[1]
    pos = np.arange(T)[None, :]
    qr = round_bf16(oracle_rope_qknorm(q, pos, eps, base))
    kr = round_bf16(oracle_rope_qknorm(k, pos, eps, base))
    dqr, dkr, dv = oracle_bwd(qr, kr, _f64(v), _f64(do), W, scale)
    return oracle_rope_qknorm_bwd(q, pos, dqr, eps, base), oracle_rope_qknorm_bwd(k, pos, dkr, eps, base), dv


def oracle_prefill_rope(q, k_new, v_new, k_cache, v_cache, cache_len, W: int, eps: float,
                        base: float = 10000.0, scale: float | None = None):
    """Chunked prefill with the prologue: the chunk's token t of sequence b sits at position
    cache_len[b] + t; its query and key are rotated and normalised there, the key is appended to
    the cache in that form, and attention follows as in oracle_prefill.
    Returns (o, lse, k_cache_after, v_cache_after) float64."""
    Tn = np.asarray(q).shape[1]
    pos = np.asarray(cache_len, dtype=np.int64)[:, None] + np.arange(Tn)[None, :]
    qr = round_bf16(oracle_rope_qknorm(q, pos, eps, base))
    kr = round_bf16(oracle_rope_qknorm(k_new, pos, eps, base))
    return oracle_prefill(qr, kr, _f64(v_new), _f64(k_cache), _f64(v_cache), cache_len, W, scale)


def oracle_decode_rope(q, k_new, v_new, k_cache, v_cache, cache_len, W: int, eps: float,
                       base: float = 10000.0, scale: float | None = None):
    """Decode with the prologue: the new token of sequence b sits in slot cache_len[b] - 1 (its
    position); its key, rotated and normalised there, and its value are written into that slot,
    and its rotated, normalised query attends as in oracle_decode.
    q [B,H,D]; k_new, v_new [B,Hk,D]; caches [B,cap,Hk,D].
    Returns (o, lse, k_cache_after, v_cache_after) float64."""
    cl = np.asarray(cache_len, dtype=np.int64)
    pos = cl - 1
    qr = round_bf16(oracle_rope_qknorm(np.asarray(q)[:, None], pos[:, None], eps, base)[:, 0])
    kr = round_bf16(oracle_rope_qknorm(np.asarray(k_new)[:, None], pos[:, None], eps, base)[:, 0])
    kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
    vn = _f64(v_new)
    for b in range(len(cl)):
        kc[b, pos[b]] = kr[b]
        vc[b, pos[b]] = vn[b]
    o, lse = oracle_decode(qr, kc, vc, cl, W, scale)
    return o, lse, kc, vc
