"""GPU parity of the FP8 (e4m3) forward, attn_fwd_fp8, against the fp64 oracle (oracle_fwd_fp8).

Both sides consume the same e4m3 bytes and descales: the seeded bf16 inputs are scaled per
(sequence, head) so that their largest magnitude maps to 448 and converted with torch's
float8_e4m3fn conversion (a library routine, neither side's arithmetic).  The oracle is the plain
definition on e4m3 value * descale.  Tolerances (stated here, derived from the kernel's one extra
rounding): the kernel rounds each softmax weight P to e4m3 before the P.V product, a relative
error of at most 2^-4 per weight and about 2^-4 / sqrt(3) = 3.6% in root mean square; O, a
weighted average of V rows, inherits that relative error, so O is held to relative L2 <= 6e-2.
lse comes from the fp32 scores of exact e4m3 products and the unrounded weights: max-abs <= 1e-3.
"""
import numpy as np
import pytest
import torch

from causal_sliding_window_b200 import inputs
from oracle import oracle_fwd_fp8

pytestmark = pytest.mark.gpu

O_REL_FP8, LSE_ABS = 6e-2, 1e-3


def to_e4m3(bits, heads):
    """bf16 bits [B, T, Hx, D] -> (e4m3 tensor on the GPU, its values as fp64, descale [B, Hx] fp32)."""
    x = (np.ascontiguousarray(bits[:, :, :heads]).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    amax = np.abs(x).max(axis=(1, 3))
    ds = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
    q8 = torch.tensor(x / ds.astype(np.float64)[:, None, :, None], dtype=torch.float32).to(torch.float8_e4m3fn)
    return q8.cuda(), q8.to(torch.float64).numpy(), torch.tensor(ds).cuda()


def run_fp8(ops, B, T, H, Hkv, W, seed):
    x = inputs.attention_inputs(B, T, H, 128, seed=seed, with_do=False)
    q8, qv, dq = to_e4m3(x["q"], H)
    k8, kv, dk = to_e4m3(x["k"], Hkv)
    v8, vv, dv = to_e4m3(x["v"], Hkv)
    o = torch.full((B, T, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, H, T), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(ops.attn_fwd_fp8_workspace_bytes(B, T, Hkv, 128), dtype=torch.uint8, device="cuda")
    ops.attn_fwd_fp8(q8, k8, v8, dq, dk, dv, o, lse, ws, W)
    torch.cuda.synchronize()
    assert ops.attn_device_status(clear=True) == 0
    ro, rl = oracle_fwd_fp8(qv, kv, vv, dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy(), W)
    go = o.double().cpu().numpy()
    gl = lse.double().cpu().numpy()
    return go, gl, ro, rl


@pytest.mark.parametrize("B,T,H,Hkv,W", [(1, 128, 2, 2, 128), (2, 333, 4, 2, 100), (1, 1000, 3, 3, 10 ** 9),
                                          (2, 1024, 40, 8, 512)])   # the last: every CTA runs several items
def test_fp8_forward_matches_oracle(cuda_device, B, T, H, Hkv, W):
    from causal_sliding_window_b200 import ops

    go, gl, ro, rl = run_fp8(ops, B, T, H, Hkv, W, seed=300 + T + H)
    assert np.isfinite(go).all() and np.isfinite(gl).all()
    rel = float(np.linalg.norm(go - ro) / np.linalg.norm(ro))
    assert rel <= O_REL_FP8, rel
    assert float(np.max(np.abs(gl - rl))) <= LSE_ABS
    # and no (b, h) slice is off on its own
    for b in range(B):
        for h in range(H):
            assert np.linalg.norm(go[b, :, h] - ro[b, :, h]) / np.linalg.norm(ro[b, :, h]) <= O_REL_FP8, (b, h)
