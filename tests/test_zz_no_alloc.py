"""attn_decode_noalloc: single-token decode for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: plugins whose host engine owns
every byte of device memory and forbids allocation outside its own arena, and
latency-bound token loops where an allocation could block on, or synchronise
with, the device. attn_decode_noalloc runs the same decode on a fixed 8 MiB
scratch array inside the library. These tests call it through the C ABI twice
in a row and check each result against the fp64 oracle (the decode tolerances
of the other GPU tests) and bit for bit against attn_decode, which runs the same
kernel on a caller-owned workspace. This file is collected last so that a run
stopping at the first failure has already run every other test; it also passes
alone in a fresh process (its first call does the one-time scratch set-up).
"""
import ctypes

import numpy as np
import pytest
import torch

from causal_sliding_window_b200 import inputs
from oracle import oracle_decode

pytestmark = pytest.mark.gpu

O_REL, O_ABS, LSE_ABS = 5e-3, 2e-2, 1e-3


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _host(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rel(a, b):
    return float(np.linalg.norm((a - b).ravel()) / np.linalg.norm(b.ravel()))


@pytest.mark.parametrize("B,cap,H,D,W", [(32, 2048, 12, 128, 2048), (7, 300, 13, 64, 100)])
def test_noalloc_decode_matches_oracle_and_workspace_decode_twice(cuda_device, B, cap, H, D, W):
    from causal_sliding_window_b200 import ops

    x = inputs.decode_inputs(B, cap, H, D, seed=4242 + H)
    q, kc, vc = _dev(x["q"]), _dev(x["k_cache"]), _dev(x["v_cache"])
    cl = torch.from_numpy(x["cache_len"]).cuda()
    ref_o, ref_l = ops.decode(q, kc, vc, cl, W)          # existing entry point, own workspace
    oo, ol = oracle_decode(x["q"], x["k_cache"], x["v_cache"], x["cache_len"], W)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    scale = 1.0 / np.sqrt(D)
    for _ in range(2):                                    # two calls in a row share the scratch
        o = torch.full((B, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        status = ops._lib.attn_decode_noalloc(
            ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
            ctypes.c_void_p(cl.data_ptr()), ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
            B, cap, H, D, W, ctypes.c_float(scale), stream)
        assert status == 0
        torch.cuda.synchronize()
        assert ops.attn_device_status(clear=True) == 0
        # the oracle, at the decode tolerances of the other GPU tests
        go, gl = _host(o), lse.double().cpu().numpy()
        assert np.isfinite(go).all() and np.isfinite(gl).all()
        assert _rel(go, oo) <= O_REL and np.max(np.abs(go - oo)) <= O_ABS
        assert np.max(np.abs(gl - ol)) <= LSE_ABS
        # the same kernel on a caller-owned workspace: identical bits
        assert torch.equal(o.view(torch.int16), ref_o.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), ref_l.view(torch.int32))


def test_noalloc_decode_rejects_sizes_beyond_its_scratch(cuda_device):
    from causal_sliding_window_b200 import ops

    # 64 sequences x capacity 4096 x 16 heads x 128 needs more than the fixed 8 MiB.
    assert ops.attn_decode_workspace_bytes(64, 4096, 16, 128) > (8 << 20)
    a = ctypes.c_void_p(1 << 20)
    status = ops._lib.attn_decode_noalloc(a, a, a, a, a, a, 64, 4096, 16, 128, 4096, ctypes.c_float(0.1), None)
    assert status == -5            # ATTN_ERR_WORKSPACE
