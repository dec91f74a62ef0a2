"""Pins for the fp64 oracle, checked against things other than the oracle itself.

Each test ties the oracle to something the definition or mathematics fixes:
a library routine (PyTorch's scaled_dot_product_attention and autograd, fp64,
with an explicit band mask), central finite differences, closed forms
(W = 1, identical keys, one-hot values), and invariants (W >= T equals full
causal, per-row score shifts move lse only, decode equals the last forward
row). test_oracle_mutants.py then plants plausible mistakes in a copy of the
oracle and shows these pins catch them.
"""
import numpy as np
import pytest
import torch

from causal_sliding_window_b200 import inputs
from oracle import (oracle_bwd, oracle_decode, oracle_dkv_rows, oracle_dq_rows, oracle_fwd, oracle_prefill,
                    oracle_fwd_rows)


def band_mask(T, W):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= i) & (j > i - W)


def torch_reference(q, k, v, W, scale, do=None):
    """PyTorch fp64 SDPA with an explicit boolean band mask; q is [B,T,H,D], k, v [B,T,Hk,D] float64
    numpy.  With Hk < H each K/V head is repeated for its H/Hk consecutive query heads inside
    autograd, so the K/V gradients come out summed over each group."""
    tq, tk, tv = (torch.tensor(x).permute(0, 2, 1, 3).contiguous().requires_grad_(do is not None)
                  for x in (q, k, v))
    G = q.shape[2] // k.shape[2]
    ek, ev = (t.repeat_interleave(G, dim=1) for t in (tk, tv))
    mask = torch.tensor(band_mask(q.shape[1], W))
    o = torch.nn.functional.scaled_dot_product_attention(tq, ek, ev, attn_mask=mask, scale=scale)
    scores = (tq @ ek.transpose(-1, -2)) * scale
    lse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
    out = {"o": o.detach().permute(0, 2, 1, 3).numpy(), "lse": lse.detach().numpy()}
    if do is not None:
        o.backward(torch.tensor(do).permute(0, 2, 1, 3))
        out["dq"] = tq.grad.permute(0, 2, 1, 3).numpy()
        out["dk"] = tk.grad.permute(0, 2, 1, 3).numpy()
        out["dv"] = tv.grad.permute(0, 2, 1, 3).numpy()
    return out


def f64(bits):
    return inputs.bf16_bits_to_f64(bits)


CASES = [
    # (B, T, H, D, W)
    (1, 128, 2, 64, 128),   # tiny workload, full causal
    (1, 128, 2, 64, 32),    # tiny workload, short window
    (2, 37, 3, 16, 5),      # ragged, odd heads
    (1, 50, 1, 8, 1),       # W = 1
    (1, 20, 2, 8, 10 ** 9), # W far beyond T
]


@pytest.mark.parametrize("B,T,H,D,W", CASES)
def test_forward_matches_torch_sdpa(B, T, H, D, W):
    x = inputs.attention_inputs(B, T, H, D, seed=7 + T + W % 97, with_do=False)
    o, lse = oracle_fwd(x["q"], x["k"], x["v"], W)
    ref = torch_reference(f64(x["q"]), f64(x["k"]), f64(x["v"]), W, x["scale"])
    np.testing.assert_allclose(o, ref["o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref["lse"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("B,T,H,D,W", CASES)
def test_backward_matches_torch_autograd(B, T, H, D, W):
    x = inputs.attention_inputs(B, T, H, D, seed=11 + T + W % 89)
    dq, dk, dv = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    ref = torch_reference(f64(x["q"]), f64(x["k"]), f64(x["v"]), W, x["scale"], do=f64(x["do"]))
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(got, ref[name], rtol=0, atol=1e-11, err_msg=name)


def test_backward_central_finite_differences():
    """L = sum(dO * O); central differences with h = 1e-6 in fp64, T=16, D=8, W=5."""
    rng = np.random.default_rng(3)
    B, T, H, D, W = 1, 16, 1, 8, 5
    q, k, v, do = (rng.standard_normal((B, T, H, D)) for _ in range(4))
    dq, dk, dv = oracle_bwd(q, k, v, do, W)

    def loss(q_, k_, v_):
        o, _ = oracle_fwd(q_, k_, v_, W)
        return float(np.sum(o * do))

    h = 1e-6
    for name, grad, idx in (("q", dq, 0), ("k", dk, 1), ("v", dv, 2)):
        num = np.zeros_like(grad)
        for flat in range(grad.size):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[idx].reshape(-1)[flat] += h
            args_m[idx].reshape(-1)[flat] -= h
            num.reshape(-1)[flat] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.linalg.norm(num - grad) / np.linalg.norm(grad)
        assert err < 1e-7, (name, err)


def test_one_hot_values_expose_softmax_rows():
    """V = identity (D = T) makes O_i the probability row P_i: band support, sums to 1, ratios exp."""
    rng = np.random.default_rng(5)
    T, W = 24, 7
    q = rng.standard_normal((1, T, 1, T))
    k = rng.standard_normal((1, T, 1, T))
    v = np.eye(T).reshape(1, T, 1, T)
    scale = 0.3
    o, lse = oracle_fwd(q, k, v, W, scale=scale)
    P = o[0, :, 0, :]
    mask = band_mask(T, W)
    assert np.all(P[~mask] == 0.0)
    assert np.all(P[mask] > 0.0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    S = (q[0, :, 0, :] @ k[0, :, 0, :].T) * scale
    for i in range(T):
        j = np.nonzero(mask[i])[0]
        # P_ij / P_ik = exp(S_ij - S_ik); and lse_i = ln sum exp S_ij.
        np.testing.assert_allclose(np.log(P[i, j]) - np.log(P[i, j[0]]), S[i, j] - S[i, j[0]], atol=1e-12)
        np.testing.assert_allclose(lse[0, 0, i], np.log(np.sum(np.exp(S[i, j]))), atol=1e-12)


def test_window_at_least_T_is_full_causal():
    x = inputs.attention_inputs(2, 40, 2, 16, seed=21, with_do=True)
    outs = [oracle_fwd(x["q"], x["k"], x["v"], W) for W in (40, 41, 10 ** 9)]
    for o, lse in outs[1:]:
        assert np.array_equal(o, outs[0][0]) and np.array_equal(lse, outs[0][1])
    grads = [oracle_bwd(x["q"], x["k"], x["v"], x["do"], W) for W in (40, 10 ** 9)]
    for a, b in zip(*grads):
        assert np.array_equal(a, b)
    tq, tk, tv = (torch.tensor(f64(x[n])).permute(0, 2, 1, 3) for n in ("q", "k", "v"))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=x["scale"])
    np.testing.assert_allclose(outs[0][0], ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)


def test_identical_keys_give_window_mean():
    rng = np.random.default_rng(8)
    B, T, H, D, W = 1, 30, 2, 8, 6
    q = rng.standard_normal((B, T, H, D))
    kvec = rng.standard_normal((1, 1, H, D))
    k = np.broadcast_to(kvec, (B, T, H, D)).copy()
    v = rng.standard_normal((B, T, H, D))
    scale = 0.25
    o, lse = oracle_fwd(q, k, v, W, scale=scale)
    for i in range(T):
        lo = max(0, i - W + 1)
        n = i - lo + 1
        np.testing.assert_allclose(o[0, i], v[0, lo:i + 1].mean(axis=0), atol=1e-12)
        for h in range(H):
            expect = scale * np.dot(q[0, i, h], kvec[0, 0, h]) + np.log(n)
            assert abs(lse[0, h, i] - expect) < 1e-12


def test_window_one_closed_form():
    rng = np.random.default_rng(9)
    B, T, H, D = 2, 12, 2, 8
    q, k, v, do = (rng.standard_normal((B, T, H, D)) for _ in range(4))
    scale = 0.4
    o, lse = oracle_fwd(q, k, v, 1, scale=scale)
    np.testing.assert_allclose(o, v, atol=1e-14)
    np.testing.assert_allclose(lse, scale * np.einsum("bthd,bthd->bht", q, k), atol=1e-12)
    dq, dk, dv = oracle_bwd(q, k, v, do, 1, scale=scale)
    assert np.max(np.abs(dq)) < 1e-14 and np.max(np.abs(dk)) < 1e-14
    np.testing.assert_allclose(dv, do, atol=1e-14)


def test_single_token_sequence():
    rng = np.random.default_rng(10)
    q, k, v, do = (rng.standard_normal((3, 1, 2, 8)) for _ in range(4))
    for W in (1, 5):
        o, lse = oracle_fwd(q, k, v, W, scale=0.5)
        np.testing.assert_allclose(o, v, atol=1e-14)
        np.testing.assert_allclose(lse, 0.5 * np.einsum("bthd,bthd->bht", q, k), atol=1e-12)
        dq, dk, dv = oracle_bwd(q, k, v, do, W, scale=0.5)
        np.testing.assert_allclose(dv, do, atol=1e-14)
        assert np.max(np.abs(dq)) < 1e-14 and np.max(np.abs(dk)) < 1e-14


def test_row_score_shift_moves_lse_only():
    """k_j -> k_j + u for all j shifts row i's scores by s<q_i,u>: O unchanged, lse shifted."""
    rng = np.random.default_rng(12)
    B, T, H, D, W = 1, 25, 1, 8, 9
    q, k, v = (rng.standard_normal((B, T, H, D)) for _ in range(3))
    u = rng.standard_normal((1, 1, H, D))
    scale = 0.35
    o1, l1 = oracle_fwd(q, k, v, W, scale=scale)
    o2, l2 = oracle_fwd(q, k + u, v, W, scale=scale)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    shift = scale * np.einsum("bthd,xyhd->bht", q, u)
    np.testing.assert_allclose(l2 - l1, shift, atol=1e-12)


@pytest.mark.parametrize("W", [1, 3, 16, 10 ** 9])
def test_decode_equals_last_forward_row(W):
    B, cap, H, D = 4, 16, 2, 8
    x = inputs.decode_inputs(B, cap, H, D, seed=30, cache_len=np.array([1, 2, 9, 16]))
    o, lse = oracle_decode(x["q"], x["k_cache"], x["v_cache"], x["cache_len"], W)
    for b in range(B):
        L = int(x["cache_len"][b])
        # Prefix with the decode query placed at position L-1.
        q_seq = np.zeros((1, L, H, D), np.uint16)
        q_seq[0, L - 1] = x["q"][b]
        fo, fl = oracle_fwd(q_seq, x["k_cache"][b:b + 1, :L].copy(), x["v_cache"][b:b + 1, :L].copy(), W)
        np.testing.assert_array_equal(o[b], fo[0, L - 1])
        np.testing.assert_array_equal(lse[b], fl[0, :, L - 1])


def test_decode_matches_torch_sdpa():
    B, cap, H, D, W = 3, 40, 2, 16, 11
    x = inputs.decode_inputs(B, cap, H, D, seed=31, cache_len=np.array([1, 23, 40]))
    o, lse = oracle_decode(x["q"], x["k_cache"], x["v_cache"], x["cache_len"], W)
    for b in range(B):
        L = int(x["cache_len"][b])
        lo = max(0, L - W)
        tq = torch.tensor(f64(x["q"][b]))[:, None, :]                       # [H,1,D]
        tk = torch.tensor(f64(x["k_cache"][b, lo:L])).permute(1, 0, 2)     # [H,n,D]
        tv = torch.tensor(f64(x["v_cache"][b, lo:L])).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=x["scale"])
        np.testing.assert_allclose(o[b], ref[:, 0].numpy(), atol=1e-12)
        ref_lse = torch.logsumexp((tq @ tk.transpose(-1, -2))[:, 0] * x["scale"], dim=-1)
        np.testing.assert_allclose(lse[b], ref_lse.numpy(), atol=1e-12)


def test_selected_rows_agree_with_full_passes():
    x = inputs.attention_inputs(2, 70, 3, 16, seed=40)
    W = 20
    o, lse = oracle_fwd(x["q"], x["k"], x["v"], W)
    dq, dk, dv = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    rows = np.array([[0, 0, 0], [1, 2, 69], [0, 1, 19], [1, 0, 20], [0, 2, 55]])
    ro, rl = oracle_fwd_rows(x["q"], x["k"], x["v"], W, rows)
    rdq = oracle_dq_rows(x["q"], x["k"], x["v"], x["do"], W, rows)
    rdk, rdv = oracle_dkv_rows(x["q"], x["k"], x["v"], x["do"], W, rows)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(ro[r], o[b, i, h], atol=1e-13)
        assert abs(rl[r] - lse[b, h, i]) < 1e-13
        np.testing.assert_allclose(rdq[r], dq[b, i, h], atol=1e-12)
        np.testing.assert_allclose(rdk[r], dk[b, i, h], atol=1e-12)
        np.testing.assert_allclose(rdv[r], dv[b, i, h], atol=1e-12)


def test_input_generator_is_deterministic_and_normal():
    a = inputs.normal_bf16(5, "q", (4, 1000))
    b = inputs.normal_bf16(5, "q", (4, 1000))
    c = inputs.normal_bf16(5, "k", (4, 1000))
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    x = inputs.bf16_bits_to_f64(inputs.normal_bf16(1, "v", (200000,)))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    peaky = inputs.bf16_bits_to_f64(inputs.rms_peaky_bf16(2, "q", (50, 128)))
    rms = np.sqrt(np.mean(peaky ** 2, axis=1))
    np.testing.assert_allclose(rms, 1.5, rtol=5e-3)
    lens = inputs.uniform_int(3, "cache_len", 10000, 1, 2048)
    assert lens.min() >= 1 and lens.max() <= 2048 and abs(lens.mean() - 1024.5) < 30


GQA_CASES = [
    # (B, T, H, Hk, D, W): grouped K/V heads (the GPT config's n_kv_head)
    (1, 40, 4, 2, 16, 9),
    (2, 33, 6, 1, 8, 10 ** 9),   # one K/V head for all query heads
    (1, 70, 8, 4, 16, 25),
]


def gqa_inputs(B, T, H, Hk, D, seed):
    """Attention inputs whose K / V keep only their first Hk heads."""
    x = inputs.attention_inputs(B, T, H, D, seed=seed)
    x["k"] = np.ascontiguousarray(x["k"][:, :, :Hk])
    x["v"] = np.ascontiguousarray(x["v"][:, :, :Hk])
    return x


@pytest.mark.parametrize("B,T,H,Hk,D,W", GQA_CASES)
def test_grouped_kv_heads_match_torch(B, T, H, Hk, D, W):
    x = gqa_inputs(B, T, H, Hk, D, seed=300 + T)
    o, lse = oracle_fwd(x["q"], x["k"], x["v"], W)
    dq, dk, dv = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    ref = torch_reference(f64(x["q"]), f64(x["k"]), f64(x["v"]), W, x["scale"], do=f64(x["do"]))
    assert dk.shape == (B, T, Hk, D) and dv.shape == (B, T, Hk, D)
    for got, name in ((o, "o"), (lse, "lse"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        np.testing.assert_allclose(got, ref[name], rtol=0, atol=1e-11, err_msg=name)


def test_grouped_kv_heads_reduce_to_repeated_heads():
    """Grouped K/V equals multi-head attention on K/V repeated per group; dK/dV of a K/V head is the
    sum of the repeated heads' gradients."""
    B, T, H, Hk, D, W = 1, 48, 6, 2, 16, 13
    x = gqa_inputs(B, T, H, Hk, D, seed=91)
    kr, vr = (np.ascontiguousarray(np.repeat(x[n], H // Hk, axis=2)) for n in ("k", "v"))
    o_g, lse_g = oracle_fwd(x["q"], x["k"], x["v"], W)
    o_m, lse_m = oracle_fwd(x["q"], kr, vr, W)
    np.testing.assert_array_equal(o_g, o_m)
    np.testing.assert_array_equal(lse_g, lse_m)
    dq_g, dk_g, dv_g = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    dq_m, dk_m, dv_m = oracle_bwd(x["q"], kr, vr, x["do"], W)
    np.testing.assert_array_equal(dq_g, dq_m)
    np.testing.assert_allclose(dk_g, dk_m.reshape(B, T, Hk, H // Hk, D).sum(axis=3), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv_g, dv_m.reshape(B, T, Hk, H // Hk, D).sum(axis=3), rtol=0, atol=1e-12)


def test_grouped_kv_rows_and_decode():
    B, T, H, Hk, D, W = 2, 45, 4, 2, 16, 11
    x = gqa_inputs(B, T, H, Hk, D, seed=17)
    o, lse = oracle_fwd(x["q"], x["k"], x["v"], W)
    dq, dk, dv = oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
    rows = np.array([[0, 0, 0], [1, 3, 44], [0, 1, 10], [1, 2, 11]])
    o_r, lse_r = oracle_fwd_rows(x["q"], x["k"], x["v"], W, rows)
    np.testing.assert_allclose(o_r, o[rows[:, 0], rows[:, 2], rows[:, 1]], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse_r, lse[rows[:, 0], rows[:, 1], rows[:, 2]], rtol=0, atol=1e-13)
    np.testing.assert_allclose(oracle_dq_rows(x["q"], x["k"], x["v"], x["do"], W, rows),
                               dq[rows[:, 0], rows[:, 2], rows[:, 1]], rtol=0, atol=1e-12)
    krows = np.array([[0, 0, 0], [1, 1, 44], [0, 1, 20], [1, 0, 33]])   # (b, K/V head, key)
    dk_r, dv_r = oracle_dkv_rows(x["q"], x["k"], x["v"], x["do"], W, krows)
    np.testing.assert_allclose(dk_r, dk[krows[:, 0], krows[:, 2], krows[:, 1]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv_r, dv[krows[:, 0], krows[:, 2], krows[:, 1]], rtol=0, atol=1e-12)
    # decode of the last row equals forward row L-1 for every query head of each group
    cache_len = np.array([T, 20])
    q_dec = np.ascontiguousarray(np.stack([x["q"][b, cache_len[b] - 1] for b in range(B)]))
    od, ld_ = oracle_decode(q_dec, x["k"], x["v"], cache_len, W)
    for b in range(B):
        L = int(cache_len[b])
        sub_o, sub_lse = oracle_fwd(x["q"][b:b + 1, :L], x["k"][b:b + 1, :L], x["v"][b:b + 1, :L], W)
        np.testing.assert_allclose(od[b], sub_o[0, L - 1], rtol=0, atol=1e-13)
        np.testing.assert_allclose(ld_[b], sub_lse[0, :, L - 1], rtol=0, atol=1e-13)


def test_grouped_kv_heads_must_divide():
    x = inputs.attention_inputs(1, 8, 3, 8, seed=1)
    with pytest.raises(ValueError):
        oracle_fwd(x["q"], x["k"][:, :, :2].copy(), x["v"][:, :, :2].copy(), 4)


def prefill_inputs(B, Tn, cap, H, Hk, D, seed):
    x = inputs.attention_inputs(B, Tn, H, D, seed=seed)
    c = inputs.decode_inputs(B, cap, Hk, D, seed=seed + 1)
    return (x["q"], np.ascontiguousarray(x["k"][:, :, :Hk]), np.ascontiguousarray(x["v"][:, :, :Hk]),
            c["k_cache"], c["v_cache"])


def test_prefill_on_an_empty_cache_is_the_forward():
    q, kn, vn, kc, vc = prefill_inputs(2, 40, 64, 4, 2, 16, seed=5)
    o, lse, kc2, vc2 = oracle_prefill(q, kn, vn, kc, vc, np.array([0, 0]), 13)
    ro, rl = oracle_fwd(q, kn, vn, 13)
    np.testing.assert_array_equal(o, ro)
    np.testing.assert_array_equal(lse, rl)
    np.testing.assert_array_equal(kc2[:, :40], kn)
    np.testing.assert_array_equal(vc2[:, 40:], vc[:, 40:])


def test_prefill_of_one_token_is_a_decode_step():
    q, kn, vn, kc, vc = prefill_inputs(3, 1, 50, 4, 2, 16, seed=8)
    L = np.array([0, 17, 49])
    o, lse, kc2, vc2 = oracle_prefill(q, kn, vn, kc, vc, L, 9)
    od, ld_ = oracle_decode(np.ascontiguousarray(q[:, 0]), kc2, vc2, L + 1, 9)
    np.testing.assert_allclose(o[:, 0], od, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, 0], ld_, rtol=0, atol=1e-13)


def test_prefill_in_two_chunks_equals_one_chunk():
    """Chunked prefill: chunk A then chunk B over the updated cache gives chunk A+B's outputs."""
    q, kn, vn, kc, vc = prefill_inputs(2, 30, 80, 4, 1, 16, seed=12)
    L = np.array([3, 25])
    o, lse, kc_ab, vc_ab = oracle_prefill(q, kn, vn, kc, vc, L, 17)
    oa, la, kc_a, vc_a = oracle_prefill(q[:, :12], kn[:, :12], vn[:, :12], kc, vc, L, 17)
    ob, lb, kc_b, vc_b = oracle_prefill(q[:, 12:], kn[:, 12:], vn[:, 12:], kc_a, vc_a, L + 12, 17)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(np.concatenate([la, lb], axis=2), lse, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(kc_b, kc_ab)

