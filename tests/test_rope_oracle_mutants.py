"""Planted mistakes in a copy of the rotary-embedding + QK-norm oracle must fail its pins.

Each mutant is oracle/rope_oracle.py with one plausible error (flipped rotation, interleaved
instead of half-split pairs, a wrong frequency exponent, a dropped eps, an off-by-one position
in decode or prefill).  The copy is loaded as a module of its own; the compact pin checks below
(the same facts as test_rope_oracle_pins.py) must then fail.  The unmodified source passes.
"""
import os
import types

import numpy as np
import pytest

import oracle
from oracle import round_bf16
from tests.test_rope_oracle_pins import complex_reference

SRC = os.path.join(os.path.dirname(oracle.__file__), "rope_oracle.py")

MUTANTS = {
    "rotation_reversed": ("np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)",
                          "np.concatenate([x1 * c + x2 * s, -x1 * s + x2 * c], axis=-1)"),
    "pairs_interleaved": ("x1, x2 = x[..., :d], x[..., d:]\n    y = np.concatenate",
                          "x1, x2 = x[..., 0::2], x[..., 1::2]\n    y = np.concatenate"),
    "theta_exponent_halved": ("theta = base ** (-2.0 * i / D)", "theta = base ** (-i / D)"),
    "eps_dropped": ("np.mean(y * y, axis=-1, keepdims=True) + eps)", "np.mean(y * y, axis=-1, keepdims=True))"),
    "decode_position_is_length": ("    pos = cl - 1\n", "    pos = cl\n"),
    "prefill_positions_from_zero": ("pos = np.asarray(cache_len, dtype=np.int64)[:, None] + np.arange(Tn)[None, :]",
                                    "pos = 0 * np.asarray(cache_len, dtype=np.int64)[:, None] + np.arange(Tn)[None, :]"),
}


def _load(source: str):
    mod = types.ModuleType("rope_oracle_copy")
    exec(compile(source.replace("from .swa_oracle import", "from oracle.swa_oracle import"), SRC, "exec"),
         mod.__dict__)
    return mod


def _pins_pass(m) -> bool:
    try:
        return _pins_hold(m)
    except (IndexError, ValueError):   # an oracle that fails on valid input fails its pins
        return False


def _pins_hold(m) -> bool:
    rng = np.random.default_rng(11)
    x = rng.standard_normal((1, 5, 2, 16))
    pos = np.array([[0, 1, 7, 300, 2047]])
    if not np.allclose(m.oracle_rope_qknorm(x, pos, 1e-6), complex_reference(x, pos, 1e-6), rtol=0, atol=1e-9):
        return False
    x0 = rng.standard_normal((1, 1, 1, 16))
    want = x0 / np.sqrt((x0 ** 2).mean(-1, keepdims=True) + 0.25)
    if not np.allclose(m.oracle_rope_qknorm(x0, [[0]], 0.25), want, rtol=0, atol=1e-14):
        return False
    B, cap, H, Hk, D, W, eps = 2, 20, 2, 1, 8, 6, 1e-5
    lens = np.array([3, 20])
    kc, vc = rng.standard_normal((B, cap, Hk, D)), rng.standard_normal((B, cap, Hk, D))
    q, kn, vn = rng.standard_normal((B, H, D)), rng.standard_normal((B, Hk, D)), rng.standard_normal((B, Hk, D))
    o, lse, _, _ = m.oracle_decode_rope(q, kn, vn, kc, vc, lens, W, eps)
    op, lp, _, _ = m.oracle_prefill_rope(q[:, None], kn[:, None], vn[:, None], kc, vc, lens - 1, W, eps)
    if not (np.allclose(o, op[:, 0], rtol=0, atol=1e-12) and np.allclose(lse, lp[..., 0], rtol=0, atol=1e-12)):
        return False
    # the appended key sits at its position: rotate-and-normalise of k_new at cache_len - 1
    _, _, kc_after, _ = m.oracle_decode_rope(q, kn, vn, kc, vc, lens, W, eps)
    for b in range(B):
        want = round_bf16(complex_reference(kn[b][None, None], [[lens[b] - 1]], eps)[0, 0])
        if not np.allclose(kc_after[b, lens[b] - 1], want, rtol=0, atol=1e-12):
            return False
    return True


def test_unmodified_oracle_passes():
    assert _pins_pass(_load(open(SRC).read()))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    assert not _pins_pass(_load(src.replace(old, new)))
