"""Pins of the rotary-embedding + QK-norm oracle to facts that do not come from the oracle.

The reading written out in oracle/rope_oracle.py (RoFormer rotation of the pairs
(x[i], x[i + D/2]) by pos * base^(-2i/D), then x / sqrt(mean(x^2) + eps)) is checked against:
complex multiplication by e^(i pos theta) (a different route to the same rotation), the plain
RMS normalisation at position 0, the unit RMS of the output, the relative-position property
of the rotated dot product, the 2-D rotation matrix at D = 2, central finite differences of
the forward for the backward, and consistency of the prefill / decode compositions with the
training forward.
"""
import numpy as np
import pytest

from causal_sliding_window_b200 import inputs
from oracle import (oracle_decode_rope, oracle_fwd_rope, oracle_prefill_rope, oracle_rope_qknorm,
                    oracle_rope_qknorm_bwd, round_bf16)


def _rng(seed):
    return np.random.default_rng(seed)


def complex_reference(x, pos, eps, base=10000.0):
    """Pairs (x[i], x[i + D/2]) as complex numbers, each multiplied by exp(1j * pos * theta_i)."""
    D = x.shape[-1]
    d = D // 2
    z = x[..., :d] + 1j * x[..., d:]
    theta = np.array([base ** (-(2.0 * i) / D) for i in range(d)])
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None, None] * theta)
    y = np.concatenate([z.real, z.imag], axis=-1)
    return y / np.sqrt((y ** 2).sum(-1, keepdims=True) / D + eps)


@pytest.mark.parametrize("D,base", [(8, 10000.0), (64, 10000.0), (128, 500000.0)])
def test_rotation_matches_complex_multiplication(D, base):
    x = _rng(D).standard_normal((2, 7, 3, D))
    pos = np.array([[0, 1, 2, 50, 511, 2047, 100000]] * 2)
    got = oracle_rope_qknorm(x, pos, 1e-6, base)
    # angles reach 1e5 rad: one ulp of theta moves them by ~1e-11, so 1e-9 bounds the rounding
    assert np.allclose(got, complex_reference(x, pos, 1e-6, base), rtol=0, atol=1e-9)


def test_position_zero_is_plain_rms_norm():
    x = _rng(1).standard_normal((1, 1, 4, 16)) * 3.0
    eps = 0.25   # large enough that dropping it would show
    got = oracle_rope_qknorm(x, np.zeros((1, 1), dtype=np.int64), eps)
    ms = (x ** 2).mean(-1, keepdims=True)
    assert np.allclose(got, x / np.sqrt(ms + eps), rtol=0, atol=1e-14)


def test_output_has_unit_rms_without_eps():
    x = _rng(2).standard_normal((3, 9, 2, 32)) * 5.0
    y = oracle_rope_qknorm(x, np.arange(9)[None, :] * 37, 0.0)
    assert np.allclose((y ** 2).mean(-1), 1.0, rtol=0, atol=1e-12)


def test_dot_product_depends_only_on_relative_position():
    rng = _rng(3)
    q, k = rng.standard_normal((1, 1, 1, 64)), rng.standard_normal((1, 1, 1, 64))
    for m, n, s in ((5, 2, 100), (0, 9, 1234), (40, 40, 7)):
        a = (oracle_rope_qknorm(q, [[m]], 0.0) * oracle_rope_qknorm(k, [[n]], 0.0)).sum()
        b = (oracle_rope_qknorm(q, [[m + s]], 0.0) * oracle_rope_qknorm(k, [[n + s]], 0.0)).sum()
        assert abs(a - b) < 1e-10


def test_head_dim_two_is_a_plane_rotation_by_pos_radians():
    x = np.array([[[[0.6, -1.7]]]])
    for pos in (0, 1, 3, 10):
        R = np.array([[np.cos(pos), -np.sin(pos)], [np.sin(pos), np.cos(pos)]])
        r = R @ x[0, 0, 0]
        want = r / np.sqrt((r ** 2).mean())
        assert np.allclose(oracle_rope_qknorm(x, [[pos]], 0.0)[0, 0, 0], want, rtol=0, atol=1e-14)


def test_backward_matches_central_differences():
    rng = _rng(4)
    x = rng.standard_normal((1, 3, 2, 8))
    dy = rng.standard_normal(x.shape)
    pos = np.array([[0, 5, 300]])
    eps = 0.1
    got = oracle_rope_qknorm_bwd(x, pos, dy, eps)
    h = 1e-6
    num = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        num[idx] = ((oracle_rope_qknorm(xp, pos, eps) - oracle_rope_qknorm(xm, pos, eps)) * dy).sum() / (2 * h)
    assert np.allclose(got, num, rtol=0, atol=1e-7)


def test_bf16_inputs_are_read_as_their_values():
    x = inputs.normal_bf16(5, "q", (1, 4, 2, 16))
    pos = np.arange(4)[None, :]
    assert np.array_equal(oracle_rope_qknorm(x, pos, 1e-6), oracle_rope_qknorm(inputs.bf16_bits_to_f64(x), pos, 1e-6))


def test_prefill_from_empty_cache_is_the_training_forward():
    B, T, H, Hk, D, W, eps = 2, 37, 4, 2, 16, 11, 1e-6
    x = inputs.attention_inputs(B, T, H, D, seed=8)
    k, v = (np.ascontiguousarray(x[n][:, :, :Hk]) for n in ("k", "v"))
    o_ref, lse_ref = oracle_fwd_rope(x["q"], k, v, W, eps)
    kc = np.zeros((B, 64, Hk, D), np.uint16)
    o, lse, kc2, _ = oracle_prefill_rope(x["q"], k, v, kc, kc.copy(), np.zeros(B, np.int64), W, eps)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-12) and np.allclose(lse, lse_ref, rtol=0, atol=1e-12)
    pos = np.arange(T)[None, :]
    assert np.array_equal(kc2[:, :T], round_bf16(oracle_rope_qknorm(k, pos, eps)))


def test_decode_is_the_last_row_of_a_one_token_prefill():
    B, cap, H, Hk, D, W, eps = 3, 40, 4, 1, 16, 9, 1e-5
    rng = _rng(9)
    lens = np.array([1, 12, 40])
    kc = rng.standard_normal((B, cap, Hk, D))
    vc = rng.standard_normal((B, cap, Hk, D))
    q = rng.standard_normal((B, H, D))
    kn, vn = rng.standard_normal((B, Hk, D)), rng.standard_normal((B, Hk, D))
    o, lse, kc_d, vc_d = oracle_decode_rope(q, kn, vn, kc, vc, lens, W, eps)
    op, lp, kc_p, vc_p = oracle_prefill_rope(q[:, None], kn[:, None], vn[:, None], kc, vc, lens - 1, W, eps)
    assert np.allclose(o, op[:, 0], rtol=0, atol=1e-12) and np.allclose(lse, lp[..., 0], rtol=0, atol=1e-12)
    for b in range(B):
        n = lens[b]
        assert np.array_equal(kc_d[b, :n], kc_p[b, :n]) and np.array_equal(vc_d[b, :n], vc_p[b, :n])


def test_bf16_rounding_is_to_nearest_even():
    # exact bf16 values stay; halfway cases go to the even neighbour; others to the nearest
    ulp1 = 2.0 ** -7                      # bf16 spacing in [1, 2)
    cases = {1.0: 1.0, 1.0 + ulp1: 1.0 + ulp1, 1.0 + ulp1 / 2: 1.0, 1.0 + 1.5 * ulp1: 1.0 + 2 * ulp1,
             1.0 + 0.49 * ulp1: 1.0, 1.0 + 0.51 * ulp1: 1.0 + ulp1, -3.0 - 0.51 * 2 * ulp1: -3.0 - 2 * ulp1,
             0.0: 0.0}
    for x, want in cases.items():
        assert round_bf16(np.array([x]))[0] == want, x
    x = np.random.default_rng(12).standard_normal(10000) * 7.0
    r = round_bf16(x)
    spacing = 2.0 ** (np.floor(np.log2(np.abs(r))) - 7)
    assert np.all(np.abs(x - r) <= spacing / 2 * (1 + 1e-9))


def test_training_backward_with_the_prologue_matches_autograd():
    """The composed backward equals torch fp64 autograd through rotate-and-normalise, a bf16
    rounding that passes gradients straight through, and masked softmax attention."""
    import torch

    from oracle import oracle_bwd_rope
    from tests.test_oracle_pins import f64

    B, T, H, Hk, D, W, eps = 1, 33, 2, 1, 16, 9, 1e-6
    x = inputs.attention_inputs(B, T, H, D, seed=21)
    k, v = (np.ascontiguousarray(x[n][:, :, :Hk]) for n in ("k", "v"))
    dq, dk, dv = oracle_bwd_rope(x["q"], k, v, x["do"], W, eps)

    tq = torch.tensor(f64(x["q"]), requires_grad=True)
    tk = torch.tensor(f64(k), requires_grad=True)
    tv = torch.tensor(f64(v), requires_grad=True)
    th = torch.tensor([10000.0 ** (-2.0 * i / D) for i in range(D // 2)], dtype=torch.float64)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * th        # [T, D/2]
    c, s_ = torch.cos(ang)[None, :, None, :], torch.sin(ang)[None, :, None, :]

    def prologue(t):
        a, b = t[..., :D // 2], t[..., D // 2:]
        r = torch.cat([a * c - b * s_, a * s_ + b * c], dim=-1)
        y = r / torch.sqrt((r * r).mean(-1, keepdim=True) + eps)
        yr = torch.tensor(round_bf16(y.detach().numpy()))
        return y + (yr - y).detach()                                  # value rounded, gradient straight through

    qr, kr = prologue(tq), prologue(tk)
    kr = kr.repeat_interleave(H // Hk, dim=2)
    vr = tv.repeat_interleave(H // Hk, dim=2)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (j <= i) & (j > i - W)
    sc = torch.einsum("bihd,bjhd->bhij", qr, kr) / np.sqrt(D)
    p = torch.softmax(sc.masked_fill(~mask, float("-inf")), dim=-1)
    o = torch.einsum("bhij,bjhd->bihd", p, vr)
    o.backward(torch.tensor(f64(x["do"])))
    for got, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.allclose(got, ref.numpy(), rtol=0, atol=1e-9)
