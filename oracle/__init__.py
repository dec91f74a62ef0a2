"""fp64 CPU oracle for causal sliding-window attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs may import this
package. The CUDA product path never touches it.

The arithmetic lives in ``swa_oracle.c`` (plain C, fp64, OpenMP over
independent (b, h) slices or selected rows); this module compiles it with gcc
on first use and wraps it with ctypes. Every function follows the definition
cited in the C file's header.
"""
from .swa_oracle import (  # noqa: F401
    build_oracle,
    oracle_decode,
    oracle_bwd,
    oracle_dkv_rows,
    oracle_dq_rows,
    oracle_fwd,
    oracle_fwd_rows,
    oracle_prefill,
    oracle_threads,
)
from .fp8_oracle import oracle_fwd_fp8, quantize_e4m3, round_e4m3  # noqa: F401
from .rope_oracle import (  # noqa: F401
    oracle_bwd_rope,
    oracle_decode_rope,
    oracle_fwd_rope,
    oracle_prefill_rope,
    oracle_rope_qknorm,
    oracle_rope_qknorm_bwd,
    rope_angles,
    round_bf16,
)
