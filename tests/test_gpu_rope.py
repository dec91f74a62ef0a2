"""GPU parity of the rotary-embedding + QK-norm prologue (through the C ABI) against the
fp64 oracle: the tables, the rotate-and-normalise op and its backward, chunked prefill and
decode with the prologue fused (rotated keys written by the append, the decode query rotated
inside the decode kernel), and the position-range error.

Tolerances: tables 1e-6 absolute (fp32 of double-precision angles); the op's bf16 output within
one bf16 rounding of the fp64 value plus 1e-5 (relative L2 <= 2e-3); its backward relative L2
<= 1e-2 like the attention gradients; attention outputs as test_gpu_parity.py (O relative L2
<= 5e-3 and max-abs <= 2e-2, lse max-abs <= 1e-3).  The oracle rounds the rotated q, k to bf16
before attention, as the kernels do (the model's activations are bf16).
"""
import numpy as np
import pytest
import torch

from causal_sliding_window_b200 import inputs
from oracle import (oracle_decode_rope, oracle_prefill_rope, oracle_rope_qknorm, oracle_rope_qknorm_bwd,
                    rope_angles)
from tests.test_gpu_parity import (LSE_ABS, O_ABS, O_REL, G_REL, Guarded, dev_bf16, host_f64, rel_l2)

pytestmark = pytest.mark.gpu
EPS = 1e-6
NAN_BF16 = 0x7FC0


@pytest.fixture(scope="module")
def ops(cuda_device):
    from causal_sliding_window_b200 import ops as _ops

    _ops.attn_device_status(clear=True)
    return _ops


@pytest.mark.parametrize("D,base", [(128, 10000.0), (64, 10000.0), (128, 500000.0)])
def test_tables_match_the_angles(ops, D, base):
    cos, sin = ops.rope_tables(5000, D, "cuda", base)
    ang = rope_angles(np.arange(5000), D, base)
    assert np.max(np.abs(cos.cpu().numpy() - np.cos(ang))) <= 1e-6
    assert np.max(np.abs(sin.cpu().numpy() - np.sin(ang))) <= 1e-6


def _check_rounded(got, ref):
    """got (bf16 values) within one bf16 rounding of ref plus 1e-5."""
    spacing = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= spacing * 0.5001 + 1e-5)
    assert rel_l2(got, ref) <= 2e-3


@pytest.mark.parametrize("B,T,H,D", [(3, 300, 4, 128), (2, 129, 3, 64)])
def test_rope_qknorm_forward_and_backward(ops, B, T, H, D):
    x = inputs.normal_bf16(D + T, "q", (B, T, H, D))
    dy = inputs.normal_bf16(D + T, "do", (B, T, H, D))
    pos0 = np.array([0, 17, 1000][:B], dtype=np.int32)
    cos, sin = ops.rope_tables(2048, D, "cuda")
    p0 = torch.from_numpy(pos0).cuda()
    y = Guarded((B, T, H, D), torch.bfloat16)
    ops.attn_rope_qknorm(dev_bf16(x), y.t, cos, sin, EPS, pos0=p0)
    dx = Guarded((B, T, H, D), torch.bfloat16)
    ops.attn_rope_qknorm_bwd(dev_bf16(x), dev_bf16(dy), dx.t, cos, sin, EPS, pos0=p0)
    xin = dev_bf16(x)   # in place: y is x
    ops.attn_rope_qknorm(xin, xin, cos, sin, EPS, pos0=p0)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    assert y.guards_intact() and dx.guards_intact()
    pos = pos0[:, None] + np.arange(T)[None, :]
    ref = oracle_rope_qknorm(x, pos, EPS)
    _check_rounded(host_f64(y.t), ref)
    assert torch.equal(xin, y.t)
    assert rel_l2(host_f64(dx.t), oracle_rope_qknorm_bwd(x, pos, dy, EPS)) <= G_REL
    # without pos0 every sequence starts at position 0
    y0 = torch.empty_like(y.t)
    ops.attn_rope_qknorm(dev_bf16(x), y0, cos, sin, EPS)
    torch.cuda.synchronize()
    _check_rounded(host_f64(y0), oracle_rope_qknorm(x, np.arange(T)[None, :], EPS))


def test_positions_outside_the_tables_are_reported_and_not_written(ops):
    B, T, H, D = 2, 40, 2, 128
    x = inputs.normal_bf16(3, "q", (B, T, H, D))
    cos, sin = ops.rope_tables(50, D, "cuda")
    y = torch.full((B, T, H, D), 7.0, dtype=torch.bfloat16, device="cuda")
    ops.attn_rope_qknorm(dev_bf16(x), y, cos, sin, EPS, pos0=torch.tensor([0, 30], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == -7   # ATTN_ERR_POSITION_RANGE
    got = host_f64(y)
    assert np.all(got[1, 20:] == 7.0)          # positions 50.. have no table row
    _check_rounded(got[1, :20], oracle_rope_qknorm(x[1:2, :20], 30 + np.arange(20)[None, :], EPS)[0])
    assert ops.attn_device_status(clear=True) == 0   # the flag was cleared


PREFILL = [
    # (B, Tn, cap, H, Hkv, D, W, cache_len before the chunk)
    (3, 77, 700, 4, 2, 128, 129, (0, 5, 600)),
    (2, 300, 1024, 4, 4, 128, 10 ** 9, (0, 700)),
    (2, 64, 400, 6, 1, 64, 50, (3, 200)),
]


@pytest.mark.parametrize("B,Tn,cap,H,Hkv,D,W,lens", PREFILL)
def test_prefill_with_rope_matches_oracle(ops, B, Tn, cap, H, Hkv, D, W, lens):
    seed = Tn + cap
    q = inputs.normal_bf16(seed, "q", (B, Tn, H, D))
    kn = inputs.normal_bf16(seed, "k", (B, Tn, Hkv, D))
    vn = inputs.normal_bf16(seed, "v", (B, Tn, Hkv, D))
    kc = inputs.normal_bf16(seed, "kcache", (B, cap, Hkv, D))
    vc = inputs.normal_bf16(seed, "vcache", (B, cap, Hkv, D))
    cl = np.array(lens, dtype=np.int32)
    for b, L in enumerate(cl):   # slots after the chunk hold NaN: never read past the chunk
        kc[b, L + Tn:] = vc[b, L + Tn:] = NAN_BF16
    cos, sin = ops.rope_tables(2048, D, "cuda")
    dkc, dvc = dev_bf16(kc), dev_bf16(vc)
    o, lse = ops.prefill_rope(dev_bf16(q), dev_bf16(kn), dev_bf16(vn), dkc, dvc, torch.from_numpy(cl).cuda(),
                              cos, sin, EPS, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    ro, rl, rkc, rvc = oracle_prefill_rope(q, kn, vn, kc, vc, cl, W, EPS)
    go, gl = host_f64(o), host_f64(lse)
    assert np.isfinite(go).all()
    assert rel_l2(go, ro) <= O_REL and np.max(np.abs(go - ro)) <= O_ABS
    assert np.max(np.abs(gl - rl)) <= LSE_ABS
    gk, gv = host_f64(dkc), host_f64(dvc)
    for b, L in enumerate(cl):
        n = L + Tn
        assert np.array_equal(gv[b, :n], rvc[b, :n])                 # values copied bit for bit
        assert np.array_equal(gk[b, :L], rkc[b, :L])                 # earlier keys untouched
        # appended keys: the oracle's rounded value, or one bf16 step away where fp32 and fp64
        # land on different sides of a rounding boundary
        diff = np.abs(gk[b, L:n] - rkc[b, L:n])
        assert np.mean(diff == 0) > 0.99
        assert np.all(diff <= 2.0 ** (np.floor(np.log2(np.maximum(np.abs(rkc[b, L:n]), 1e-30))) - 6))


@pytest.mark.parametrize("H,Hkv,D", [(12, 12, 128), (12, 4, 128), (8, 1, 64)])
def test_decode_with_rope_matches_oracle(ops, H, Hkv, D):
    B, cap, W = 6, 300, 150
    lens = np.array([1, 64, 149, 151, 300, 233], dtype=np.int32)
    x = inputs.decode_inputs(B, cap, H, D, seed=H + Hkv + D + 1, cache_len=lens)
    kc = np.ascontiguousarray(x["k_cache"][:, :, :Hkv])
    vc = np.ascontiguousarray(x["v_cache"][:, :, :Hkv])
    for b, L in enumerate(lens):   # NaN outside the window and in the new token's slot (it is written)
        lo = max(0, int(L) - W)
        kc[b, :lo] = vc[b, :lo] = NAN_BF16
        kc[b, L - 1:] = vc[b, L - 1:] = NAN_BF16
    kn = inputs.normal_bf16(H, "k", (B, Hkv, D))
    vn = inputs.normal_bf16(H, "v", (B, Hkv, D))
    cos, sin = ops.rope_tables(1024, D, "cuda")
    dkc, dvc = dev_bf16(kc), dev_bf16(vc)
    cl = torch.from_numpy(lens).cuda()
    o, lse = ops.decode_rope(dev_bf16(x["q"]), dev_bf16(kn), dev_bf16(vn), dkc, dvc, cl, cos, sin, EPS, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    ro, rl, rkc, _ = oracle_decode_rope(x["q"], kn, vn, kc, vc, lens, W, EPS)
    go, gl = host_f64(o), host_f64(lse)
    assert np.isfinite(go).all()
    assert rel_l2(go, ro) <= O_REL and np.max(np.abs(go - ro)) <= O_ABS
    assert np.max(np.abs(gl - rl)) <= LSE_ABS
    gk, gv = host_f64(dkc), host_f64(dvc)
    for b, L in enumerate(lens):
        assert np.array_equal(gv[b, L - 1], inputs.bf16_bits_to_f64(vn[b]))
        d = np.abs(gk[b, L - 1] - rkc[b, L - 1])
        assert np.all(d <= 2.0 ** (np.floor(np.log2(np.maximum(np.abs(rkc[b, L - 1]), 1e-30))) - 6))
        assert np.isnan(gk[b, L:]).all()       # slots after the new token are not written


@pytest.mark.parametrize("B,T,H,Hkv,D,W", [(2, 300, 4, 2, 128, 129), (1, 257, 2, 2, 64, 10 ** 9),
                                            (2, 1024, 40, 8, 128, 512)])   # every CTA runs several items
def test_training_forward_and_backward_with_rope(ops, B, T, H, Hkv, D, W):
    from oracle import oracle_bwd_rope, oracle_fwd_rope

    x = inputs.attention_inputs(B, T, H, D, seed=T + H)
    k, v = (np.ascontiguousarray(x[n][:, :, :Hkv]) for n in ("k", "v"))
    cos, sin = ops.rope_tables(T, D, "cuda")
    q_d, k_d, v_d, do_d = dev_bf16(x["q"]), dev_bf16(k), dev_bf16(v), dev_bf16(x["do"])
    q_rot, k_rot = torch.empty_like(q_d), torch.empty_like(k_d)
    o = Guarded((B, T, H, D), torch.bfloat16)
    lse = Guarded((B, H, T), torch.float32)
    ops.attn_fwd_rope(q_d, k_d, v_d, q_rot, k_rot, o.t, lse.t, cos, sin, EPS, W)
    dq, dk, dv = Guarded((B, T, H, D), torch.bfloat16), Guarded((B, T, Hkv, D), torch.bfloat16), \
        Guarded((B, T, Hkv, D), torch.bfloat16)
    ws = torch.empty(ops.attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device="cuda")
    ops.attn_bwd_rope(q_d, k_d, q_rot, k_rot, v_d, o.t, lse.t, do_d, dq.t, dk.t, dv.t, ws, cos, sin, EPS, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    assert all(g.guards_intact() for g in (o, lse, dq, dk, dv))
    # the rotated queries the forward kernel wrote (its in-kernel prologue) and the rotated keys
    pos = np.arange(T)[None, :]
    _check_rounded(host_f64(q_rot), oracle_rope_qknorm(x["q"], pos, EPS))
    _check_rounded(host_f64(k_rot), oracle_rope_qknorm(k, pos, EPS))
    ro, rl = oracle_fwd_rope(x["q"], k, v, W, EPS)
    go, gl = host_f64(o.t), host_f64(lse.t)
    assert rel_l2(go, ro) <= O_REL and np.max(np.abs(go - ro)) <= O_ABS
    assert np.max(np.abs(gl - rl)) <= LSE_ABS
    rdq, rdk, rdv = oracle_bwd_rope(x["q"], k, v, x["do"], W, EPS)
    for got, ref in ((dq, rdq), (dk, rdk), (dv, rdv)):
        assert rel_l2(host_f64(got.t), ref) <= G_REL


def test_training_forward_with_rope_reports_positions_outside_the_tables(ops):
    """Tables shorter than the sequence: the forward's in-kernel prologue flags the positions it
    cannot rotate (ATTN_ERR_POSITION_RANGE) and rotates the others."""
    B, T, H, D, W = 1, 300, 2, 128, 64
    x = inputs.attention_inputs(B, T, H, D, seed=77, with_do=False)
    cos, sin = ops.rope_tables(200, D, "cuda")
    q_d, k_d, v_d = dev_bf16(x["q"]), dev_bf16(x["k"]), dev_bf16(x["v"])
    q_rot, k_rot = torch.empty_like(q_d), torch.empty_like(k_d)
    o = torch.empty_like(q_d)
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    ops.attn_fwd_rope(q_d, k_d, v_d, q_rot, k_rot, o, lse, cos, sin, EPS, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == -7   # ATTN_ERR_POSITION_RANGE
    _check_rounded(host_f64(q_rot)[:, :200], oracle_rope_qknorm(x["q"][:, :200], np.arange(200)[None, :], EPS))
    assert ops.attn_device_status(clear=True) == 0
