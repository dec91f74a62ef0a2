"""Pins of the FP8 (e4m3) attention oracle (oracle/fp8_oracle.py), on the CPU.

round_e4m3 is checked against torch's float8_e4m3fn conversion (an independent implementation of
the OCP E4M3 format) on a dense set of values, on every midpoint between neighbouring
representable values (ties to even) and on all 256 bit patterns; quantize_e4m3 against its
definition; oracle_fwd_fp8 against PyTorch fp64 scaled_dot_product_attention with an explicit band
mask on the dequantised operands (another route to the same definition), and against the
invariance that moving a factor between an operand and its descale leaves the result unchanged
(a dropped or misplaced descale fails both).
"""
import math

import numpy as np
import pytest
import torch

from causal_sliding_window_b200 import inputs
from oracle import oracle_fwd_fp8, quantize_e4m3, round_e4m3


def torch_e4m3(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def all_e4m3_values():
    b = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return np.unique(b[np.isfinite(b)])


def test_round_e4m3_matches_torch_on_a_dense_set():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-448, 448, 200000), rng.normal(0, 1, 200000),
                        rng.uniform(-2 ** -5, 2 ** -5, 100000), np.linspace(-448, 448, 100001)]).astype(np.float32)
    np.testing.assert_array_equal(round_e4m3(x.astype(np.float64)), torch_e4m3(x))


def test_every_representable_value_is_fixed_and_midpoints_round_to_even():
    v = all_e4m3_values()
    assert v.size == 253 and v.max() == 448.0                 # 0 once, +-0 merged; NaN patterns dropped
    np.testing.assert_array_equal(round_e4m3(v), v)
    pos = v[v >= 0]
    mid = (pos[:-1] + pos[1:]) / 2                             # exact midpoints (fp64 holds them)
    np.testing.assert_array_equal(round_e4m3(mid), torch_e4m3(mid.astype(np.float32)))
    # the tie goes to the neighbour with an even mantissa (last bit 0)
    bits = torch.tensor(round_e4m3(mid).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.all(bits % 2 == 0)


def test_saturation_and_special_values():
    got = round_e4m3(np.array([449.0, 464.0, 1e9, -1e9, 0.0, -0.0, np.nan, 2 ** -10, 3 * 2 ** -11]))
    assert list(got[:4]) == [448.0, 448.0, 448.0, -448.0]
    assert got[4] == 0 and got[5] == 0 and math.copysign(1, got[5]) == -1
    assert np.isnan(got[6])
    assert got[7] == 0.0                                       # 2^-10 ties to 0 (even)
    assert got[8] == 2 ** -9                                   # 1.5 * 2^-10 rounds up to the smallest subnormal


def test_quantize_e4m3_scales_each_head_to_the_format_range():
    x = inputs.attention_inputs(2, 64, 3, 64, seed=1, with_do=False)["q"]
    q8, ds = quantize_e4m3(x)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert ds.shape == (2, 3)
    np.testing.assert_allclose(np.max(np.abs(q8), axis=(1, 3)), 448.0)
    np.testing.assert_array_equal(round_e4m3(q8), q8)          # the values are e4m3 values
    rel = np.abs(q8 * ds[:, None, :, None] - xf) / np.maximum(np.abs(xf), 1e-30)
    big = np.abs(xf) >= ds[:, None, :, None] * 2 ** -6          # normal range: relative error <= 2^-4
    assert np.all(rel[big] <= 2 ** -4 + 1e-12)


def _sdpa_band(q, k, v, W, scale):
    B, T, H, D = q.shape
    Hk = k.shape[2]
    qt = torch.tensor(q).permute(0, 2, 1, 3)
    kt = torch.tensor(k).permute(0, 2, 1, 3).repeat_interleave(H // Hk, dim=1)
    vt = torch.tensor(v).permute(0, 2, 1, 3).repeat_interleave(H // Hk, dim=1)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (j <= i) & (j > i - W)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("B,T,H,Hk,D,W", [(2, 96, 4, 2, 64, 33), (1, 70, 2, 2, 128, 10 ** 9)])
def test_oracle_fwd_fp8_is_the_definition_on_the_dequantised_operands(B, T, H, Hk, D, W):
    x = inputs.attention_inputs(B, T, H, D, seed=T + W % 97, with_do=False)
    q8, dq = quantize_e4m3(x["q"])
    k8, dk = quantize_e4m3(np.ascontiguousarray(x["k"][:, :, :Hk]))
    v8, dv = quantize_e4m3(np.ascontiguousarray(x["v"][:, :, :Hk]))
    o, lse = oracle_fwd_fp8(q8, k8, v8, dq, dk, dv, W)
    s = 1.0 / math.sqrt(D)
    ref = _sdpa_band(q8 * dq[:, None, :, None], k8 * dk[:, None, :, None], v8 * dv[:, None, :, None], W, s)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    # a factor moved between the operands and their descales changes nothing
    o2, lse2 = oracle_fwd_fp8(q8 / 2, k8, v8 * 4, dq * 2, dk, dv / 4, W)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)
