"""The C-ABI library loads, exports every entry point its header declares, and
rejects bad arguments with the documented status before launching anything
(these calls never reach the GPU, so they run on a CPU-only machine)."""
import ctypes
import os
import re

import pytest

from causal_sliding_window_b200.build import HEADER, build_library

build_library()
from causal_sliding_window_b200 import ops  # noqa: E402

ERR_INVALID, ERR_UNSUPPORTED, ERR_WORKSPACE = -1, -2, -5
A = 1 << 20          # a fake, 256-byte-aligned device address; never dereferenced on these paths
MIS = A + 8          # misaligned


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(attn_[a-z_0-9]+)\s*\(", text, flags=re.M)))


def test_header_entry_points_are_exported():
    names = declared_functions()
    assert {"attn_fwd", "attn_bwd", "attn_decode", "attn_bwd_workspace_bytes",
            "attn_decode_workspace_bytes", "attn_device_status", "attn_status_string",
            "attn_selftest_wait_timeout", "attn_poll_device_status"} <= set(names)
    lib = ctypes.CDLL(ops.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(ops.EXPORTED) | {n for n in names if hasattr(ops, n)}


def test_library_is_sm100a_only_build():
    from causal_sliding_window_b200 import build

    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags


def fwd(q=A, k=A, v=A, o=A, lse=A, B=1, T=16, H=1, D=128, W=4, scale=0.1):
    return ops._lib.attn_fwd(q, k, v, o, lse, B, T, H, D, W, scale, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), ERR_INVALID), (dict(lse=None), ERR_INVALID), (dict(o=MIS), ERR_INVALID),
    (dict(B=0), ERR_INVALID), (dict(T=0), ERR_INVALID), (dict(H=-1), ERR_INVALID), (dict(W=0), ERR_INVALID),
    (dict(scale=0.0), ERR_INVALID), (dict(scale=float("nan")), ERR_INVALID), (dict(scale=-1.0), ERR_INVALID),
    (dict(D=96), ERR_UNSUPPORTED), (dict(D=256), ERR_UNSUPPORTED),
])
def test_fwd_rejects_bad_arguments(kw, expect):
    assert fwd(**kw) == expect


def bwd(ws_bytes=None, ws=A, B=1, T=16, H=1, D=128, W=4, scale=0.1, dq=A):
    if ws_bytes is None:
        ws_bytes = ops.attn_bwd_workspace_bytes(B, T, H, D) if B > 0 and T > 0 and H > 0 else 0
    return ops._lib.attn_bwd(A, A, A, A, A, A, dq, A, A, ws, ws_bytes, B, T, H, D, W, scale, None)


def test_bwd_rejects_bad_arguments():
    assert bwd(ws=None) == ERR_INVALID
    assert bwd(ws=A + 16) == ERR_INVALID               # workspace must be 256-byte aligned
    assert bwd(dq=MIS) == ERR_INVALID
    assert bwd(W=0) == ERR_INVALID
    assert bwd(D=80) == ERR_UNSUPPORTED
    assert bwd(ws_bytes=ops.attn_bwd_workspace_bytes(1, 16, 1, 128) - 1) == ERR_WORKSPACE


def test_workspace_sizes():
    # lse*log2e and Delta [B*H, Tp] fp32, each 256-byte padded.
    assert ops.attn_bwd_workspace_bytes(32, 2048, 12, 128) == 2 * 32 * 12 * 2048 * 4
    assert ops.attn_bwd_workspace_bytes(1, 130, 1, 64) == 2 * 256 * 4   # Tp = 256
    assert ops.attn_bwd_workspace_bytes(1, 1, 1, 128) == 2 * 512   # 128 floats per row, no 256-byte padding needed
    assert ops.attn_bwd_workspace_bytes(0, 1, 1, 64) == 0
    # ticket counters [B, head groups of 4 heads (D = 128) / 8 heads (D = 64)] + partial (m, l) and o
    # for ceil(cap / 128) chunks of 128 cache slots
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert ops.attn_decode_workspace_bytes(32, 2048, 12, 128) == a256(32 * 3 * 4) + a256(32 * 16 * 12 * 2 * 4) + a256(
        32 * 16 * 12 * 128 * 4)
    assert ops.attn_decode_workspace_bytes(2, 100, 9, 64) == a256(2 * 2 * 4) + a256(2 * 1 * 9 * 2 * 4) + a256(
        2 * 1 * 9 * 64 * 4)
    assert ops.attn_decode_workspace_bytes(1, 0, 1, 64) == 0
    for bad_d in (0, 4, 7, 96):
        assert ops.attn_decode_workspace_bytes(1, 16, 1, bad_d) == 0


def test_grouped_decode_workspace_size():
    """With grouped K/V heads a thread serves up to 4 query heads of one K/V head (a divisor of the
    group where there is one) over runs of 64 cache slots; counters per group of 4 (D = 128) or 8
    (D = 64) (K/V head, query subgroup) pairs, partials per query head and 64-slot run."""
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    # 12 query heads over 4 K/V heads: 3 per thread, 4 pairs -> 1 counter per sequence, 32 runs
    assert ops.attn_decode_gqa_workspace_bytes(32, 2048, 12, 4, 128) == a256(32 * 1 * 4) + a256(
        32 * 32 * 12 * 2 * 4) + a256(32 * 32 * 12 * 128 * 4)
    # MQA, 8 query heads: 4 per thread, 2 subgroups, 8 pairs per CTA at D = 64
    assert ops.attn_decode_gqa_workspace_bytes(2, 100, 8, 1, 64) == a256(2 * 1 * 4) + a256(2 * 2 * 8 * 2 * 4) + a256(
        2 * 2 * 8 * 64 * 4)
    # 40 query heads over 8 K/V heads: groups of 5 -> 4 + 1 (ragged), 16 pairs -> 4 counters
    assert ops.attn_decode_gqa_workspace_bytes(1, 64, 40, 8, 128) == a256(1 * 4 * 4) + a256(1 * 1 * 40 * 2 * 4) + a256(
        1 * 1 * 40 * 128 * 4)
    for B, cap, H, D in ((32, 2048, 12, 128), (2, 100, 9, 64), (3, 1, 1, 128)):
        assert ops.attn_decode_gqa_workspace_bytes(B, cap, H, H, D) == ops.attn_decode_workspace_bytes(B, cap, H, D)
    assert ops.attn_decode_gqa_workspace_bytes(2, 64, 6, 4, 128) == 0      # 4 does not divide 6
    assert ops.attn_decode_gqa_workspace_bytes(2, 64, 6, 0, 128) == 0
    assert ops.attn_decode_gqa_workspace_bytes(2, 64, 6, 3, 96) == 0


def dec(q=A, cl=A, ws=A, ws_bytes=None, B=2, cap=64, H=2, D=128, W=8, scale=0.1, lse=A):
    if ws_bytes is None:
        ws_bytes = ops.attn_decode_workspace_bytes(B, cap, H, D) if B > 0 and cap > 0 and H > 0 else 0
    return ops._lib.attn_decode(q, A, A, cl, A, lse, ws, ws_bytes, B, cap, H, D, W, scale, None)


def test_decode_rejects_bad_arguments():
    assert dec(q=None) == ERR_INVALID
    assert dec(cl=None) == ERR_INVALID
    assert dec(cl=A + 2) == ERR_INVALID
    assert dec(ws=A + 64) == ERR_INVALID
    assert dec(cap=0) == ERR_INVALID
    assert dec(W=0) == ERR_INVALID
    assert dec(D=32) == ERR_UNSUPPORTED
    assert dec(ws_bytes=16) == ERR_WORKSPACE


def test_status_strings_and_selftest_argument_check():
    assert ops.attn_status_string(0) == "ok"
    assert ops.attn_status_string(-4) == "device wait timed out"
    assert ops.attn_status_string(7) == "unknown status"
    assert ops._lib.attn_selftest_wait_timeout(0, None) == ERR_INVALID


def test_product_path_has_no_oracle_or_fallback():
    """The package never imports the oracle, and ops raises if the library is absent."""
    pkg = os.path.dirname(ops.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(root, f)).read()
                assert "oracle" not in src.replace("oracle_", "").lower() or f == "inputs.py", f
    src = open(ops.__file__).read()
    assert "raise ImportError" in src


def test_grouped_kv_heads_argument_checks():
    # Hkv must be >= 1 and divide H (checked before any launch)
    assert ops._lib.attn_fwd_gqa(A, A, A, A, A, 1, 16, 6, 4, 128, 4, 0.1, None) == ERR_INVALID
    assert ops._lib.attn_fwd_gqa(A, A, A, A, A, 1, 16, 6, 0, 128, 4, 0.1, None) == ERR_INVALID
    ws = ops.attn_bwd_workspace_bytes(1, 16, 6, 128)
    assert ops._lib.attn_bwd_gqa(A, A, A, A, A, A, A, A, A, A, ws, 1, 16, 6, 5, 128, 4, 0.1, None) == ERR_INVALID
    dws = ops.attn_decode_workspace_bytes(2, 64, 6, 128)
    assert ops._lib.attn_decode_gqa(A, A, A, A, A, A, A, dws, 2, 64, 6, 4, 128, 8, 0.1, None) == ERR_INVALID
    assert ops._lib.attn_fwd_gqa(A, A, A, A, A, 1, 16, 6, 2, 96, 4, 0.1, None) == ERR_UNSUPPORTED


def test_prefill_argument_checks():
    args = lambda **kw: dict(dict(B=2, Tn=16, cap=64, H=4, Hkv=2, D=128, W=8, scale=0.1), **kw)  # noqa: E731
    call = lambda a, cl=A: ops._lib.attn_prefill(A, A, A, A, A, cl, A, A, a["B"], a["Tn"], a["cap"], a["H"],  # noqa: E731
                                                  a["Hkv"], a["D"], a["W"], a["scale"], None)
    assert call(args(cap=15)) == ERR_INVALID          # cap < Tn
    assert call(args(Hkv=3)) == ERR_INVALID           # Hkv must divide H
    assert call(args(), cl=A + 2) == ERR_INVALID      # cache_len misaligned
    assert call(args(W=0)) == ERR_INVALID
    assert call(args(D=96)) == ERR_UNSUPPORTED
    assert ops.attn_status_string(-6) == "cache capacity exceeded"



def test_rope_argument_checks():
    """Each rotary entry point rejects bad arguments before launching anything."""
    lib = ops._lib
    # tables: pointers, sizes, base
    assert lib.attn_rope_tables(None, A, 16, 128, 10000.0, None) == ERR_INVALID
    assert lib.attn_rope_tables(A, A + 4, 16, 128, 10000.0, None) == ERR_INVALID   # misaligned
    assert lib.attn_rope_tables(A, A, 0, 128, 10000.0, None) == ERR_INVALID
    assert lib.attn_rope_tables(A, A, 16, 127, 10000.0, None) == ERR_INVALID       # odd D
    assert lib.attn_rope_tables(A, A, 16, 128, 1.0, None) == ERR_INVALID           # base must exceed 1
    assert lib.attn_rope_tables(A, A, 16, 128, float("nan"), None) == ERR_INVALID
    # rotate-and-normalise (forward and backward)
    args = dict(pos0=None, cs=A, sn=A, max_pos=64, B=2, T=8, H=3, D=128, eps=1e-6)
    fwd = lambda **kw: (lambda a: lib.attn_rope_qknorm(A, A, a["pos0"], a["cs"], a["sn"], a["max_pos"], a["B"],  # noqa: E731
                                                        a["T"], a["H"], a["D"], a["eps"], None))(dict(args, **kw))
    bwd = lambda **kw: (lambda a: lib.attn_rope_qknorm_bwd(A, A, A, a["pos0"], a["cs"], a["sn"], a["max_pos"],  # noqa: E731
                                                            a["B"], a["T"], a["H"], a["D"], a["eps"], None))(dict(args, **kw))
    for call in (fwd, bwd):
        assert call(cs=None) == ERR_INVALID
        assert call(max_pos=0) == ERR_INVALID
        assert call(eps=-1.0) == ERR_INVALID
        assert call(eps=float("inf")) == ERR_INVALID
        assert call(pos0=A + 2) == ERR_INVALID
        assert call(B=0) == ERR_INVALID
        assert call(D=96) == ERR_UNSUPPORTED
    assert lib.attn_rope_qknorm_bwd(A, None, A, None, A, A, 64, 2, 8, 3, 128, 1e-6, None) == ERR_INVALID
    # prefill with the prologue: workspace size is checked first
    assert ops.attn_prefill_rope_workspace_bytes(2, 77, 4, 128) == (2 * 77 * 4 * 128 * 2 + 255) // 256 * 256
    assert ops.attn_prefill_rope_workspace_bytes(2, 77, 4, 96) == 0
    need = ops.attn_prefill_rope_workspace_bytes(2, 16, 4, 128)
    pre = lambda ws_bytes, ws=A, cs=A, eps=1e-6: lib.attn_prefill_rope(  # noqa: E731
        A, A, A, A, A, A, cs, A, 64, eps, A, A, ws, ws_bytes, 2, 16, 64, 4, 2, 128, 8, 0.1, None)
    assert pre(need - 1) == ERR_WORKSPACE
    assert pre(need, ws=A + 16) == ERR_INVALID      # workspace must be 256-byte aligned
    assert pre(need, cs=None) == ERR_INVALID
    assert pre(need, eps=-0.5) == ERR_INVALID
    # decode with the prologue: grouped workspace size, new token's K / V present
    dneed = ops.attn_decode_gqa_workspace_bytes(2, 64, 4, 2, 128)
    dec_r = lambda ws_bytes, kn=A, Hkv=2: lib.attn_decode_rope(  # noqa: E731
        A, kn, A, A, A, A, A, A, 64, 1e-6, A, A, A, ws_bytes, 2, 64, 4, Hkv, 128, 8, 0.1, None)
    assert dec_r(dneed - 1) == ERR_WORKSPACE
    assert dec_r(dneed, kn=None) == ERR_INVALID
    assert dec_r(dneed, Hkv=3) == ERR_INVALID        # 3 does not divide 4


def test_training_rope_argument_checks():
    lib = ops._lib
    fwd = lambda qr=A, cs=A, eps=1e-6, Hkv=2, D=128: lib.attn_fwd_rope(  # noqa: E731
        A, A, A, qr, A, A, A, cs, A, 64, eps, 2, 16, 4, Hkv, D, 8, 0.1, None)
    assert fwd(qr=None) == ERR_INVALID
    assert fwd(cs=None) == ERR_INVALID
    assert fwd(eps=-1.0) == ERR_INVALID
    assert fwd(Hkv=3) == ERR_INVALID
    assert fwd(D=96) == ERR_UNSUPPORTED
    ws = ops.attn_bwd_workspace_bytes(2, 16, 4, 128)
    bwd = lambda ws_bytes=ws, kr=A, cs=A: lib.attn_bwd_rope(  # noqa: E731
        A, A, A, kr, A, A, A, A, A, A, A, A, ws_bytes, cs, A, 64, 1e-6, 2, 16, 4, 2, 128, 8, 0.1, None)
    assert bwd(kr=None) == ERR_INVALID
    assert bwd(cs=None) == ERR_INVALID
    assert bwd(ws_bytes=ws - 1) == ERR_WORKSPACE


def test_header_is_plain_c(tmp_path):
    """The boundary header compiles as C99, and every entry point it declares can be named from C."""
    import subprocess

    names = declared_functions()
    src = tmp_path / "use_header.c"
    src.write_text('#include "swa_attn.h"\n' + "".join(f"void* p_{n} = (void*)&{n};\n" for n in names))
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-c", "-I", os.path.dirname(HEADER),
                           str(src), "-o", str(tmp_path / "use_header.o")])


def test_fp8_forward_argument_checks():
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert ops.attn_fwd_fp8_workspace_bytes(2, 100, 3, 128) == a256(2 * 3 * 128 * 112)   # T rounded up to 16
    assert ops.attn_fwd_fp8_workspace_bytes(2, 100, 3, 64) == 0
    f = ops._lib.attn_fwd_fp8
    ws = ops.attn_fwd_fp8_workspace_bytes(1, 16, 1, 128)
    assert f(None, A, A, A, A, A, A, A, A, ws, 1, 16, 1, 1, 128, 8, 0.1, None) == ERR_INVALID
    assert f(A, A, A, A, A, A, A, A, A, ws, 1, 16, 1, 1, 64, 8, 0.1, None) == ERR_UNSUPPORTED
    assert f(A, A, A, A, A, A, A, A, A, ws - 16, 1, 16, 1, 1, 128, 8, 0.1, None) == ERR_WORKSPACE
    assert f(A, A, A, A + 2, A, A, A, A, A, ws, 1, 16, 1, 1, 128, 8, 0.1, None) == ERR_INVALID   # descale misaligned
    assert f(A, A, A, A, A, A, A, A, A, ws, 1, 16, 4, 3, 128, 8, 0.1, None) == ERR_INVALID        # 3 does not divide 4
