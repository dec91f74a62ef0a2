"""FP8 (e4m3) attention forward, written out in fp64 (test infrastructure).

Reading (the pages name FP8 only for linear layers, "--fp8" on H100 and Blackwell in the apidog
guide's mixed-precision section; nothing fixes an FP8 attention, so this is the plainest reading
that the rest supports): q, k, v are stored as OCP FP8 E4M3 values (1 sign bit, 4 exponent bits
with bias 7, 3 mantissa bits, subnormals, no infinities, largest finite value 448) with one fp32
descale factor per (sequence, head), so the real operand is e4m3 value * descale, as in FA3's
q_descale / k_descale / v_descale.  Attention is then the plain definition on those real values
(the band, scale and outputs of oracle_fwd).  The kernel's own rounding of P to e4m3 before the
P.V product is its approximation, bounded by the stated tolerance, not part of the definition.

round_e4m3 is written from the format definition (round to nearest, ties to even, saturating at
+-448 as the "satfinite" conversions do); quantize_e4m3 picks the per-(b, head) descale from the
amax so that the largest magnitude maps to 448.
"""
from __future__ import annotations

import numpy as np

from .swa_oracle import oracle_fwd

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUBNORMAL_STEP = 2.0 ** -9


def _rne(x):
    """Round to the nearest integer, ties to even (fp64)."""
    return np.rint(x)   # numpy's rint rounds half to even


def round_e4m3(x):
    """Nearest E4M3 value of each element (fp64 in, fp64 out); NaN stays NaN; |x| > 448 saturates."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore", invalid="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)                                  # below 2^-6 the spacing stays 2^-9 (subnormals)
    quantum = np.where(a >= E4M3_MIN_NORMAL, 2.0 ** (e - 3), E4M3_SUBNORMAL_STEP)
    y = _rne(a / quantum) * quantum                        # a carry into the next binade is exact
    y = np.minimum(y, E4M3_MAX)
    return np.where(np.isnan(x), np.nan, np.copysign(y, x))


def quantize_e4m3(x, head_axis: int = 2):
    """x [B, T, H, D] (fp64 or bf16 bits as uint16) -> (e4m3 values fp64, descale [B, H] fp64) with
    descale = amax / 448 per (b, h) (1 where a head is all zeros); the real value is e4m3 * descale."""
    from .rope_oracle import _f64

    x = _f64(x)
    amax = np.max(np.abs(x), axis=(1, 3))                  # [B, H]
    descale = np.where(amax > 0, amax / E4M3_MAX, 1.0)
    q = round_e4m3(x / descale[:, None, :, None])
    return q, descale


def oracle_fwd_fp8(q8, k8, v8, dq, dk, dv, W: int, scale: float | None = None):
    """FP8 forward: q8 [B, T, H, D], k8 / v8 [B, T, Hk, D] e4m3 values (fp64 arrays), descales
    dq [B, H], dk / dv [B, Hk].  Returns (o, lse) in fp64: the plain definition on the real
    operands e4m3 * descale (oracle_fwd).  scale defaults to 1/sqrt(D)."""
    q = np.asarray(q8, np.float64) * np.asarray(dq, np.float64)[:, None, :, None]
    k = np.asarray(k8, np.float64) * np.asarray(dk, np.float64)[:, None, :, None]
    v = np.asarray(v8, np.float64) * np.asarray(dv, np.float64)[:, None, :, None]
    return oracle_fwd(q, k, v, W, scale)
