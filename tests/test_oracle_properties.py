"""Property-based pins: random small shapes, windows, head groupings, cache lengths and rotary
positions, each checked against a route that does not go through the oracle's own code
(PyTorch fp64 SDPA with an explicit band mask and autograd; complex multiplication for the
rotation; the decode / prefill compositions against the forward rows).  Hypothesis draws the
cases; the number of examples is bounded so the suite stays within seconds.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

from causal_sliding_window_b200 import inputs
from oracle import oracle_bwd, oracle_decode, oracle_fwd, oracle_fwd_rows, oracle_prefill, oracle_rope_qknorm
from tests.test_oracle_pins import f64, torch_reference
from tests.test_rope_oracle_pins import complex_reference

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)


@st.composite
def attention_case(draw):
    Hk = draw(st.sampled_from([1, 2]))
    G = draw(st.sampled_from([1, 2, 3]))
    return dict(B=draw(st.integers(1, 2)), T=draw(st.integers(1, 45)), H=Hk * G, Hk=Hk,
                D=draw(st.sampled_from([4, 8, 16])), W=draw(st.integers(1, 60)), seed=draw(st.integers(0, 10 ** 6)))


@SETTINGS
@given(attention_case())
def test_forward_and_backward_match_sdpa_autograd(c):
    x = inputs.attention_inputs(c["B"], c["T"], c["H"], c["D"], seed=c["seed"])
    k, v = (np.ascontiguousarray(x[n][:, :, :c["Hk"]]) for n in ("k", "v"))
    o, lse = oracle_fwd(x["q"], k, v, c["W"])
    dq, dk, dv = oracle_bwd(x["q"], k, v, x["do"], c["W"])
    ref = torch_reference(f64(x["q"]), f64(k), f64(v), c["W"], x["scale"], do=f64(x["do"]))
    for got, name in ((o, "o"), (lse, "lse"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        np.testing.assert_allclose(got, ref[name], rtol=0, atol=1e-10, err_msg=name)


@SETTINGS
@given(st.integers(1, 3), st.integers(1, 40), st.sampled_from([(2, 1), (2, 2), (4, 2)]), st.integers(1, 50),
       st.integers(0, 10 ** 6))
def test_decode_is_the_last_forward_row(B, cap, heads, W, seed):
    H, Hk = heads
    D = 8
    lens = inputs.uniform_int(seed, "cache_len", B, 1, cap)
    x = inputs.decode_inputs(B, cap, H, D, seed=seed, cache_len=lens)
    kc, vc = (np.ascontiguousarray(x[n][:, :, :Hk]) for n in ("k_cache", "v_cache"))
    o, lse = oracle_decode(x["q"], kc, vc, lens, W)
    for b in range(B):
        L = int(lens[b])
        q_full = np.zeros((1, L, H, D), np.uint16)
        q_full[0, L - 1] = x["q"][b]
        rows = np.array([(0, h, L - 1) for h in range(H)])
        ro, rl = oracle_fwd_rows(q_full, kc[b:b + 1, :L], vc[b:b + 1, :L], W, rows)
        np.testing.assert_allclose(o[b], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], rl, rtol=0, atol=1e-12)


@SETTINGS
@given(st.integers(1, 2), st.integers(1, 20), st.integers(1, 30), st.integers(1, 40), st.integers(0, 10 ** 6))
def test_prefill_of_a_whole_sequence_split_in_two_chunks(B, Tn1, Tn2, W, seed):
    """Appending two chunks one after the other gives the forward over the concatenation."""
    H, Hk, D = 2, 1, 8
    T = Tn1 + Tn2
    x = inputs.attention_inputs(B, T, H, D, seed=seed, with_do=False)
    k, v = (np.ascontiguousarray(x[n][:, :, :Hk]) for n in ("k", "v"))
    cap = T + 3
    kc = np.zeros((B, cap, Hk, D), np.uint16)
    vc = np.zeros_like(kc)
    o1, l1, kc, vc = oracle_prefill(x["q"][:, :Tn1], k[:, :Tn1], v[:, :Tn1], kc, vc, np.zeros(B, np.int64), W)
    assert kc.dtype == np.uint16   # the caches come back in their input form (bf16 bits)
    o2, l2, _, _ = oracle_prefill(x["q"][:, Tn1:], k[:, Tn1:], v[:, Tn1:], kc, vc, np.full(B, Tn1), W)
    o, lse = oracle_fwd(x["q"], k, v, W)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([l1, l2], axis=2), lse, rtol=0, atol=1e-12)


@SETTINGS
@given(st.sampled_from([2, 4, 8, 32, 128]), st.lists(st.integers(0, 70000), min_size=1, max_size=4),
       st.floats(0.0, 1.0), st.sampled_from([10000.0, 500000.0]), st.integers(0, 10 ** 6))
def test_rotation_matches_complex_multiplication(D, positions, eps, base, seed):
    x = np.random.default_rng(seed).standard_normal((1, len(positions), 2, D))
    pos = np.array([positions])
    np.testing.assert_allclose(oracle_rope_qknorm(x, pos, eps, base), complex_reference(x, pos, eps, base),
                               rtol=0, atol=1e-9)
