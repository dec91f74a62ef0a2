"""Planted mistakes in a copy of the oracle must be caught by the pins.

Each mutant is the oracle's C source with one plausible error (an off-by-one
window edge, a dropped scale, a flipped sign, a transposed operand, a wrong
logarithm base, a missing normalisation). It is compiled to a temporary
library on the CPU and swapped in for the real one; the pin checks of
test_oracle_pins.py must then fail. The unmodified source must pass them.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle.swa_oracle as so
from causal_sliding_window_b200 import inputs
from tests.test_oracle_pins import f64, torch_reference

SRC = os.path.join(os.path.dirname(so.__file__), "swa_oracle.c")

MUTANTS = {
    "window_edge_off_by_one": ("long lo = i - W + 1;", "long lo = i - W;"),
    "dq_scale_dropped": ("dq[at4(T, H, D, b, i, h, d)] += scale * ds *", "dq[at4(T, H, D, b, i, h, d)] += ds *"),
    "delta_sign_flipped": ("double ds = pij * (dp - delta);", "double ds = pij * (dp + delta);"),
    "dk_uses_k_not_q": ("dk[at4(T, Hk, D, b, j, hk, d)] += scale * ds * ld(q,",
                        "dk[at4(T, Hk, D, b, j, hk, d)] += scale * ds * ld(k,"),
    "dv_uses_key_row_of_dO": ("dv[at4(T, Hk, D, b, j, hk, d)] += pij * ld(dout, in_bf16, at4(T, H, D, b, i, h, d));",
                              "dv[at4(T, Hk, D, b, j, hk, d)] += pij * ld(dout, in_bf16, at4(T, H, D, b, j, h, d));"),
    "kv_head_map_modulo": ("long hk = h / (H / Hk);", "long hk = h % Hk;"),
    "kv_group_sums_one_head": ("for (long h = hk * G; h < (hk + 1) * G; ++h) {\n                for (long i = 0;",
                               "for (long h = hk * G; h < hk * G + 1; ++h) {\n                for (long i = 0;"),
    "lse_log2": ("*lse_i = m + log(l);", "*lse_i = m + log2(l);"),
    "softmax_not_normalised": ("for (long c = 0; c < n; ++c) p[c] /= l;", ""),
    "decode_window_short_by_one": ("long lo = L - W;", "long lo = L - W + 1;"),
    "decode_scale_dropped": ("s[j - lo] = acc * scale;", "s[j - lo] = acc;"),
}


def _compile(source: str, path: str):
    csrc = path + ".c"
    with open(csrc, "w") as f:
        f.write(source)
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", path, csrc, "-lm"])


def _pins_pass() -> bool:
    """A compact run of the library-routine pins (forward, backward, decode)."""
    for (B, T, H, D, W) in ((1, 40, 2, 16, 9), (1, 24, 1, 8, 10 ** 9)):
        x = inputs.attention_inputs(B, T, H, D, seed=T + 3)
        o, lse = so.oracle_fwd(x["q"], x["k"], x["v"], W)
        dq, dk, dv = so.oracle_bwd(x["q"], x["k"], x["v"], x["do"], W)
        ref = torch_reference(f64(x["q"]), f64(x["k"]), f64(x["v"]), W, x["scale"], do=f64(x["do"]))
        for got, name in ((o, "o"), (lse, "lse"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
            if not np.allclose(got, ref[name], rtol=0, atol=1e-10):
                return False
    # grouped K/V heads: 4 query heads on 2 K/V heads
    x = inputs.attention_inputs(1, 30, 4, 8, seed=61)
    k2, v2 = (np.ascontiguousarray(x[n][:, :, :2]) for n in ("k", "v"))
    o, lse = so.oracle_fwd(x["q"], k2, v2, 7)
    dq, dk, dv = so.oracle_bwd(x["q"], k2, v2, x["do"], 7)
    ref = torch_reference(f64(x["q"]), f64(k2), f64(v2), 7, x["scale"], do=f64(x["do"]))
    for got, name in ((o, "o"), (lse, "lse"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        if not np.allclose(got, ref[name], rtol=0, atol=1e-10):
            return False
    import torch

    x = inputs.decode_inputs(3, 30, 2, 16, seed=4, cache_len=np.array([1, 17, 30]))
    W = 12
    o, lse = so.oracle_decode(x["q"], x["k_cache"], x["v_cache"], x["cache_len"], W)
    for b in range(3):
        L = int(x["cache_len"][b])
        lo = max(0, L - W)
        tq = torch.tensor(f64(x["q"][b]))[:, None, :]
        tk = torch.tensor(f64(x["k_cache"][b, lo:L])).permute(1, 0, 2)
        tv = torch.tensor(f64(x["v_cache"][b, lo:L])).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=x["scale"])[:, 0].numpy()
        if not np.allclose(o[b], ref, rtol=0, atol=1e-10):
            return False
    return True


@pytest.fixture()
def swap_lib():
    saved = so._lib
    yield
    so._lib = saved


def _load_variant(source: str, tmp: str):
    path = os.path.join(tmp, "variant.so")
    _compile(source, path)
    import ctypes

    saved = so._lib
    so._lib = None
    real = so.build_oracle
    try:
        so.build_oracle = lambda force=False: path  # load the variant through the same argtypes setup
        so._load()
    finally:
        so.build_oracle = real
    return saved


def test_unmodified_source_passes(swap_lib):
    with tempfile.TemporaryDirectory() as tmp:
        _load_variant(open(SRC).read(), tmp)
        assert _pins_pass()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, swap_lib):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation anchor missing: {name}"
    with tempfile.TemporaryDirectory() as tmp:
        _load_variant(src.replace(old, new), tmp)
        assert not _pins_pass(), f"pins did not catch mutant {name}"
