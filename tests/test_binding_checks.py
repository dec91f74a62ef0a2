"""The Python binding rejects unusable tensors before calling the library (no CPU fallback, no
crash): CPU tensors, wrong dtypes, non-contiguous or mismatched shapes all raise ValueError."""
import pytest
import torch

from causal_sliding_window_b200 import ops


def _bf16(*shape, device="cpu"):
    return torch.zeros(shape, dtype=torch.bfloat16, device=device)


def test_cpu_tensors_are_rejected_not_computed():
    q = _bf16(1, 16, 2, 64)
    with pytest.raises(ValueError):
        ops.forward(q, q, q, 8)
    with pytest.raises(ValueError):
        ops.attn_rope_qknorm(q, q, torch.zeros(16, 32), torch.zeros(16, 32), 1e-6)


def test_wrong_dtype_and_shapes_are_rejected():
    q32 = torch.zeros(1, 16, 2, 64)
    with pytest.raises(ValueError):
        ops.forward(q32, q32, q32, 8)
    q = _bf16(1, 16, 2, 64)
    k = _bf16(1, 16, 3, 64)      # 3 K/V heads do not divide 2 query heads
    with pytest.raises(ValueError):
        ops.attn_fwd(q, k, k, q, torch.zeros(1, 2, 16), 8)
    with pytest.raises(ValueError):
        ops.forward(q.transpose(1, 2), q.transpose(1, 2), q.transpose(1, 2), 8)   # not contiguous


def test_rope_tables_must_match_the_head_dim():
    with pytest.raises(ValueError):
        ops._tables(torch.zeros(16, 31), torch.zeros(16, 31), 64)
    with pytest.raises(ValueError):
        ops._tables(torch.zeros(16, 32, dtype=torch.float64), torch.zeros(16, 32, dtype=torch.float64), 64)
