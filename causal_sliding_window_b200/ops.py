"""ctypes binding of libswa_b200.so, with the C entry points' names.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI (include/swa_attn.h). PyTorch supplies device
memory and the stream. Importing this module loads the library and raises
if it is missing; there is no fallback path.

Low-level calls (caller provides every buffer, torch tensors on one CUDA device):
  attn_fwd(q, k, v, o, lse, W, scale=None, stream=None)
  attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, W, scale=None, stream=None)
  attn_decode(q, k_cache, v_cache, cache_len, o, lse, workspace, W, scale=None, stream=None)
K and V (and dK, dV, the caches) may have fewer heads than Q (grouped K/V heads, Hkv dividing H);
the calls then go to the C entry points' _gqa forms.
Rotary embedding + QK norm (the attention prologue): attn_rope_tables, attn_rope_qknorm,
attn_rope_qknorm_bwd, attn_prefill_rope, attn_decode_rope; cos / sin tables are float32
[max_pos, D/2] CUDA tensors.
Convenience wrappers that allocate outputs: forward, backward, decode, rope_tables, prefill_rope,
decode_rope.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswa_b200.so")

ATTN_OK = 0
STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported configuration", -3: "kernel launch failed",
          -4: "device wait timed out", -5: "workspace too small", -6: "cache capacity exceeded",
          -7: "token position outside the rotary tables"}

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m causal_sliding_window_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

_p, _i, _f, _sz, _ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_longlong
_lib.attn_fwd.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_fwd.restype = _i
_lib.attn_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i]
_lib.attn_bwd_workspace_bytes.restype = _sz
_lib.attn_bwd.argtypes = [_p] * 10 + [_sz, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_bwd.restype = _i
_lib.attn_decode_workspace_bytes.argtypes = [_i, _i, _i, _i]
_lib.attn_decode_workspace_bytes.restype = _sz
_lib.attn_decode_gqa_workspace_bytes.argtypes = [_i, _i, _i, _i, _i]
_lib.attn_decode_gqa_workspace_bytes.restype = _sz
_lib.attn_decode.argtypes = [_p] * 7 + [_sz, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_decode.restype = _i
_lib.attn_fwd_gqa.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_fwd_gqa.restype = _i
_lib.attn_bwd_gqa.argtypes = [_p] * 10 + [_sz, _i, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_bwd_gqa.restype = _i
_lib.attn_decode_gqa.argtypes = [_p] * 7 + [_sz, _i, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_decode_gqa.restype = _i
_lib.attn_prefill.argtypes = [_p] * 8 + [_i, _i, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_prefill.restype = _i
_lib.attn_fwd_fp8_workspace_bytes.argtypes = [_i, _i, _i, _i]
_lib.attn_fwd_fp8_workspace_bytes.restype = _sz
_lib.attn_fwd_fp8.argtypes = [_p] * 9 + [_sz] + [_i] * 6 + [_f, _p]
_lib.attn_fwd_fp8.restype = _i
_lib.attn_decode_noalloc.argtypes = [_p] * 6 + [_i, _i, _i, _i, _i, _f, _p]
_lib.attn_decode_noalloc.restype = _i
_d = ctypes.c_double
_lib.attn_rope_tables.argtypes = [_p, _p, _i, _i, _d, _p]
_lib.attn_rope_tables.restype = _i
_lib.attn_rope_qknorm.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_rope_qknorm.restype = _i
_lib.attn_rope_qknorm_bwd.argtypes = [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _f, _p]
_lib.attn_rope_qknorm_bwd.restype = _i
_lib.attn_prefill_rope_workspace_bytes.argtypes = [_i, _i, _i, _i]
_lib.attn_prefill_rope_workspace_bytes.restype = _sz
_lib.attn_prefill_rope.argtypes = [_p] * 8 + [_i, _f, _p, _p, _p, _sz] + [_i] * 7 + [_f, _p]
_lib.attn_prefill_rope.restype = _i
_lib.attn_decode_rope.argtypes = [_p] * 8 + [_i, _f, _p, _p, _p, _sz] + [_i] * 6 + [_f, _p]
_lib.attn_decode_rope.restype = _i
_lib.attn_fwd_rope.argtypes = [_p] * 9 + [_i, _f] + [_i] * 6 + [_f, _p]
_lib.attn_fwd_rope.restype = _i
_lib.attn_bwd_rope.argtypes = [_p] * 12 + [_sz, _p, _p, _i, _f] + [_i] * 6 + [_f, _p]
_lib.attn_bwd_rope.restype = _i
_lib.attn_bwd_set_profile_events.argtypes = [_p, _p]
_lib.attn_bwd_set_profile_events.restype = _i
_lib.attn_device_status.argtypes = [_i]
_lib.attn_device_status.restype = _i
_lib.attn_poll_device_status.argtypes = [_p]
_lib.attn_poll_device_status.restype = _i
_lib.attn_selftest_wait_timeout.argtypes = [_ll, _p]
_lib.attn_selftest_wait_timeout.restype = _i
_lib.attn_status_string.argtypes = [_i]
_lib.attn_status_string.restype = ctypes.c_char_p

EXPORTED = ["attn_fwd", "attn_fwd_gqa", "attn_bwd_workspace_bytes", "attn_bwd", "attn_bwd_gqa",
            "attn_decode_workspace_bytes", "attn_decode_gqa_workspace_bytes", "attn_decode", "attn_decode_gqa", "attn_decode_noalloc", "attn_prefill", "attn_bwd_set_profile_events", "attn_device_status", "attn_poll_device_status",
            "attn_selftest_wait_timeout",
            "attn_status_string", "attn_rope_tables", "attn_rope_qknorm", "attn_rope_qknorm_bwd",
            "attn_prefill_rope_workspace_bytes", "attn_prefill_rope", "attn_decode_rope", "attn_fwd_rope",
            "attn_bwd_rope", "attn_fwd_fp8_workspace_bytes", "attn_fwd_fp8"]


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status})")
        self.status = status


def _check(status: int, where: str):
    if status != ATTN_OK:
        raise AttnError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bthd(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("expected contiguous bf16 CUDA tensors of shape [B, T, H, D]")
    shape = ts[0].shape
    if any(t.shape != shape for t in ts):
        raise ValueError("shape mismatch")
    return shape


def _kv_heads(qshape, *kv):
    """K/V tensors share one [B, T, Hkv, D] shape, with B, T, D of q and Hkv dividing q's H."""
    kshape = _bthd(*kv)
    B, T, H, D = qshape
    if kshape[0] != B or kshape[1] != T or kshape[3] != D or kshape[2] < 1 or H % kshape[2] != 0:
        raise ValueError("K/V must be [B, T, Hkv, D] with Hkv dividing the query heads")
    return kshape[2]


def _scale(scale, D):
    return 1.0 / math.sqrt(D) if scale is None else float(scale)


def attn_fwd(q, k, v, o, lse, W: int, scale=None, stream=None):
    B, T, H, D = _bthd(q, o)
    Hkv = _kv_heads((B, T, H, D), k, v)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, T) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, T] tensor")
    if Hkv == H:
        _check(_lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, T, H, D, int(W), _scale(scale, D),
                             _stream(stream)), "attn_fwd")
    else:
        _check(_lib.attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, T, H, Hkv, D, int(W),
                                 _scale(scale, D), _stream(stream)), "attn_fwd_gqa")


def attn_bwd_workspace_bytes(B: int, T: int, H: int, D: int) -> int:
    return int(_lib.attn_bwd_workspace_bytes(B, T, H, D))


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, W: int, scale=None, stream=None):
    B, T, H, D = _bthd(q, o, dout, dq)
    Hkv = _kv_heads((B, T, H, D), k, v, dk, dv)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, T):
        raise ValueError("lse must be float32 [B, H, T]")
    ws_bytes = workspace.numel() * workspace.element_size()
    ptrs = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace))
    if Hkv == H:
        _check(_lib.attn_bwd(*ptrs, ws_bytes, B, T, H, D, int(W), _scale(scale, D), _stream(stream)), "attn_bwd")
    else:
        _check(_lib.attn_bwd_gqa(*ptrs, ws_bytes, B, T, H, Hkv, D, int(W), _scale(scale, D), _stream(stream)),
               "attn_bwd_gqa")


def attn_decode_workspace_bytes(B: int, cap: int, H: int, D: int) -> int:
    return int(_lib.attn_decode_workspace_bytes(B, cap, H, D))


def attn_decode_gqa_workspace_bytes(B: int, cap: int, H: int, Hkv: int, D: int) -> int:
    return int(_lib.attn_decode_gqa_workspace_bytes(B, cap, H, Hkv, D))


def attn_decode(q, k_cache, v_cache, cache_len, o, lse, workspace, W: int, scale=None, stream=None):
    B, cap, Hkv, D = _bthd(k_cache, v_cache)
    H = q.shape[1] if q.dim() == 3 else -1
    if (tuple(q.shape) != (B, H, D) or tuple(o.shape) != (B, H, D) or q.dtype != torch.bfloat16
            or H % Hkv != 0):
        raise ValueError("q and o must be bf16 [B, H, D] with the caches' head count dividing H")
    if cache_len.dtype != torch.int32 or tuple(cache_len.shape) != (B,) or not cache_len.is_cuda:
        raise ValueError("cache_len must be an int32 CUDA tensor of shape [B]")
    ws_bytes = workspace.numel() * workspace.element_size()
    ptrs = (_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_len), _ptr(o), _ptr(lse), _ptr(workspace))
    if Hkv == H:
        _check(_lib.attn_decode(*ptrs, ws_bytes, B, cap, H, D, int(W), _scale(scale, D), _stream(stream)),
               "attn_decode")
    else:
        _check(_lib.attn_decode_gqa(*ptrs, ws_bytes, B, cap, H, Hkv, D, int(W), _scale(scale, D), _stream(stream)),
               "attn_decode_gqa")


def attn_prefill(q, k_new, v_new, k_cache, v_cache, cache_len, o, lse, W: int, scale=None, stream=None):
    """Append a chunk's K / V to the caches and attend its queries (see attn_prefill in the header)."""
    B, Tn, H, D = _bthd(q, o)
    Hkv = _kv_heads((B, Tn, H, D), k_new, v_new)
    Bc, cap, Hc, Dc = _bthd(k_cache, v_cache)
    if (Bc, Hc, Dc) != (B, Hkv, D):
        raise ValueError("caches must be [B, cap, Hkv, D] matching k_new")
    if cache_len.dtype != torch.int32 or tuple(cache_len.shape) != (B,) or not cache_len.is_cuda:
        raise ValueError("cache_len must be an int32 CUDA tensor of shape [B]")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, Tn) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, Tn] tensor")
    _check(_lib.attn_prefill(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(cache_len),
                             _ptr(o), _ptr(lse), B, Tn, cap, H, Hkv, D, int(W), _scale(scale, D), _stream(stream)),
           "attn_prefill")


def prefill(q, k_new, v_new, k_cache, v_cache, cache_len, W: int, scale=None, stream=None):
    """attn_prefill with freshly allocated outputs; returns (o, lse)."""
    B, Tn, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Tn), dtype=torch.float32, device=q.device)
    attn_prefill(q, k_new, v_new, k_cache, v_cache, cache_len, o, lse, W, scale, stream)
    return o, lse


def attn_decode_noalloc(q, k_cache, v_cache, cache_len, o, lse, W: int, scale=None, stream=None):
    """attn_decode on the library's fixed 8 MiB scratch, for callers that cannot allocate.

    Shares one scratch array across calls: do not overlap calls on the GPU.  The first
    call on a device performs a one-time address lookup; make it before stream capture.
    """
    B, cap, H, D = _bthd(k_cache, v_cache)
    if tuple(q.shape) != (B, H, D) or tuple(o.shape) != (B, H, D) or q.dtype != torch.bfloat16:
        raise ValueError("q and o must be bf16 [B, H, D]")
    if cache_len.dtype != torch.int32 or tuple(cache_len.shape) != (B,) or not cache_len.is_cuda:
        raise ValueError("cache_len must be an int32 CUDA tensor of shape [B]")
    _check(_lib.attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_len), _ptr(o), _ptr(lse),
                                    B, cap, H, D, int(W), _scale(scale, D), _stream(stream)), "attn_decode_noalloc")


def attn_bwd_set_profile_events(after_pre=None, after_main=None):
    """Record torch.cuda.Event objects between attn_bwd's launches (None disables)."""
    h = lambda e: None if e is None else ctypes.c_void_p(e.cuda_event)  # noqa: E731
    _check(_lib.attn_bwd_set_profile_events(h(after_pre), h(after_main)), "attn_bwd_set_profile_events")


def attn_device_status(clear: bool = True) -> int:
    return int(_lib.attn_device_status(1 if clear else 0))


def attn_fwd_fp8_workspace_bytes(B: int, T: int, Hkv: int, D: int) -> int:
    return int(_lib.attn_fwd_fp8_workspace_bytes(B, T, Hkv, D))


def attn_fwd_fp8(q, k, v, q_descale, k_descale, v_descale, o, lse, workspace, W: int, scale=None, stream=None):
    """FP8 forward: q [B, T, H, 128], k / v [B, T, Hkv, 128] torch.float8_e4m3fn (or uint8 holding e4m3
    bytes); descales float32 [B, H] / [B, Hkv] / [B, Hkv] (real value = e4m3 value * descale);
    o bf16 [B, T, H, 128] and lse float32 [B, H, T] written; workspace of attn_fwd_fp8_workspace_bytes."""
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    for t in (q, k, v):
        if t.element_size() != 1 or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("q, k, v must be contiguous 1-byte (e4m3) CUDA tensors")
    if tuple(k.shape) != (B, T, Hkv, D) or tuple(v.shape) != (B, T, Hkv, D) or H % Hkv != 0:
        raise ValueError("k and v must be [B, T, Hkv, D] with Hkv dividing H")
    for t, shp in ((q_descale, (B, H)), (k_descale, (B, Hkv)), (v_descale, (B, Hkv))):
        if t.dtype != torch.float32 or tuple(t.shape) != shp or not t.is_contiguous():
            raise ValueError("descales must be contiguous float32 [B, H] (q) and [B, Hkv] (k, v)")
    if o.dtype != torch.bfloat16 or tuple(o.shape) != (B, T, H, D):
        raise ValueError("o must be bf16 [B, T, H, D]")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, T):
        raise ValueError("lse must be float32 [B, H, T]")
    ws = workspace.numel() * workspace.element_size()
    _check(_lib.attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(q_descale), _ptr(k_descale), _ptr(v_descale), _ptr(o),
                             _ptr(lse), _ptr(workspace), ws, B, T, H, Hkv, D, int(W), _scale(scale, D),
                             _stream(stream)), "attn_fwd_fp8")


def attn_poll_device_status(stream=None) -> int:
    """Status recorded by the library's kernels on `stream` since its last poll (read and cleared;
    waits for that stream only)."""
    return int(_lib.attn_poll_device_status(_stream(stream)))


def attn_selftest_wait_timeout(limit_cycles: int, stream=None) -> int:
    return int(_lib.attn_selftest_wait_timeout(int(limit_cycles), _stream(stream)))


def attn_status_string(status: int) -> str:
    return _lib.attn_status_string(int(status)).decode()


# ---------------------------------------------------------------------------
# Convenience wrappers (allocate outputs with torch; compute still in the kernels)
# ---------------------------------------------------------------------------

def forward(q, k, v, W: int, scale=None, stream=None):
    B, T, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    attn_fwd(q, k, v, o, lse, W, scale, stream)
    return o, lse


def backward(q, k, v, o, lse, dout, W: int, scale=None, stream=None, workspace=None):
    B, T, H, D = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        workspace = torch.empty(attn_bwd_workspace_bytes(B, T, H, D), dtype=torch.uint8, device=q.device)
    attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, W, scale, stream)
    return dq, dk, dv


def decode_workspace(B: int, cap: int, H: int, D: int, device, Hkv=None) -> torch.Tensor:
    """Zero-filled decode workspace (the decode call keeps it zeroed between calls); Hkv = number of
    K/V heads of the caches (default H)."""
    n = attn_decode_gqa_workspace_bytes(B, cap, H, H if Hkv is None else Hkv, D)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def decode(q, k_cache, v_cache, cache_len, W: int, scale=None, stream=None, workspace=None):
    B, H, D = q.shape
    cap = k_cache.shape[1]
    o = torch.empty((B, H, D), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = decode_workspace(B, cap, H, D, q.device, Hkv=k_cache.shape[2])
    attn_decode(q, k_cache, v_cache, cache_len, o, lse, workspace, W, scale, stream)
    return o, lse


# ---------------------------------------------------------------------------
# Rotary embedding + QK norm
# ---------------------------------------------------------------------------

def _tables(cos, sin, D):
    if (cos.dtype != torch.float32 or sin.dtype != torch.float32 or not cos.is_cuda or not cos.is_contiguous()
            or not sin.is_contiguous() or cos.dim() != 2 or cos.shape != sin.shape or cos.shape[1] != D // 2):
        raise ValueError("rotary tables must be contiguous float32 CUDA tensors [max_pos, D/2]")
    return cos.shape[0]


def _pos0(pos0, B):
    if pos0 is None:
        return None
    if pos0.dtype != torch.int32 or tuple(pos0.shape) != (B,) or not pos0.is_cuda:
        raise ValueError("pos0 must be an int32 CUDA tensor of shape [B]")
    return pos0


def attn_rope_tables(cos, sin, base: float = 10000.0, stream=None):
    """Fill cos / sin [max_pos, D/2] for th_i = base^(-2i/D)."""
    D = 2 * cos.shape[1]
    max_pos = _tables(cos, sin, D)
    _check(_lib.attn_rope_tables(_ptr(cos), _ptr(sin), max_pos, D, float(base), _stream(stream)), "attn_rope_tables")


def rope_tables(max_pos: int, D: int, device, base: float = 10000.0, stream=None):
    cos = torch.empty((max_pos, D // 2), dtype=torch.float32, device=device)
    sin = torch.empty_like(cos)
    attn_rope_tables(cos, sin, base, stream)
    return cos, sin


def attn_rope_qknorm(x, y, cos, sin, eps: float, pos0=None, stream=None):
    B, T, H, D = _bthd(x, y)
    max_pos = _tables(cos, sin, D)
    _check(_lib.attn_rope_qknorm(_ptr(x), _ptr(y), _ptr(_pos0(pos0, B)), _ptr(cos), _ptr(sin), max_pos, B, T, H, D,
                                 float(eps), _stream(stream)), "attn_rope_qknorm")


def attn_rope_qknorm_bwd(x, dy, dx, cos, sin, eps: float, pos0=None, stream=None):
    B, T, H, D = _bthd(x, dy, dx)
    max_pos = _tables(cos, sin, D)
    _check(_lib.attn_rope_qknorm_bwd(_ptr(x), _ptr(dy), _ptr(dx), _ptr(_pos0(pos0, B)), _ptr(cos), _ptr(sin),
                                     max_pos, B, T, H, D, float(eps), _stream(stream)), "attn_rope_qknorm_bwd")


def attn_prefill_rope_workspace_bytes(B: int, Tn: int, H: int, D: int) -> int:
    return int(_lib.attn_prefill_rope_workspace_bytes(B, Tn, H, D))


def attn_prefill_rope(q, k_new, v_new, k_cache, v_cache, cache_len, cos, sin, eps: float, o, lse, workspace, W: int,
                      scale=None, stream=None):
    B, Tn, H, D = _bthd(q, o)
    Hkv = _kv_heads((B, Tn, H, D), k_new, v_new)
    Bc, cap, Hc, Dc = _bthd(k_cache, v_cache)
    if (Bc, Hc, Dc) != (B, Hkv, D):
        raise ValueError("caches must be [B, cap, Hkv, D] matching k_new")
    if cache_len.dtype != torch.int32 or tuple(cache_len.shape) != (B,) or not cache_len.is_cuda:
        raise ValueError("cache_len must be an int32 CUDA tensor of shape [B]")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, Tn) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, Tn] tensor")
    max_pos = _tables(cos, sin, D)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.attn_prefill_rope(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(cache_len),
                                  _ptr(cos), _ptr(sin), max_pos, float(eps), _ptr(o), _ptr(lse), _ptr(workspace),
                                  ws_bytes, B, Tn, cap, H, Hkv, D, int(W), _scale(scale, D), _stream(stream)),
           "attn_prefill_rope")


def prefill_rope(q, k_new, v_new, k_cache, v_cache, cache_len, cos, sin, eps: float, W: int, scale=None, stream=None):
    """attn_prefill_rope with freshly allocated outputs and workspace; returns (o, lse)."""
    B, Tn, H, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Tn), dtype=torch.float32, device=q.device)
    ws = torch.empty(attn_prefill_rope_workspace_bytes(B, Tn, H, D), dtype=torch.uint8, device=q.device)
    attn_prefill_rope(q, k_new, v_new, k_cache, v_cache, cache_len, cos, sin, eps, o, lse, ws, W, scale, stream)
    return o, lse


def attn_decode_rope(q, k_new, v_new, k_cache, v_cache, cache_len, cos, sin, eps: float, o, lse, workspace, W: int,
                     scale=None, stream=None):
    B, cap, Hkv, D = _bthd(k_cache, v_cache)
    H = q.shape[1] if q.dim() == 3 else -1
    if (tuple(q.shape) != (B, H, D) or tuple(o.shape) != (B, H, D) or q.dtype != torch.bfloat16 or H % Hkv != 0
            or not q.is_contiguous() or not o.is_contiguous()):
        raise ValueError("q and o must be contiguous bf16 [B, H, D] with the caches' head count dividing H")
    for t in (k_new, v_new):
        if tuple(t.shape) != (B, Hkv, D) or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("k_new and v_new must be contiguous bf16 [B, Hkv, D]")
    if cache_len.dtype != torch.int32 or tuple(cache_len.shape) != (B,) or not cache_len.is_cuda:
        raise ValueError("cache_len must be an int32 CUDA tensor of shape [B]")
    max_pos = _tables(cos, sin, D)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.attn_decode_rope(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(cache_len),
                                 _ptr(cos), _ptr(sin), max_pos, float(eps), _ptr(o), _ptr(lse), _ptr(workspace),
                                 ws_bytes, B, cap, H, Hkv, D, int(W), _scale(scale, D), _stream(stream)),
           "attn_decode_rope")


def decode_rope(q, k_new, v_new, k_cache, v_cache, cache_len, cos, sin, eps: float, W: int, scale=None, stream=None,
                workspace=None):
    """attn_decode_rope with freshly allocated outputs (and workspace unless given); returns (o, lse)."""
    B, H, D = q.shape
    cap, Hkv = k_cache.shape[1], k_cache.shape[2]
    o = torch.empty((B, H, D), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = decode_workspace(B, cap, H, D, q.device, Hkv=Hkv)
    attn_decode_rope(q, k_new, v_new, k_cache, v_cache, cache_len, cos, sin, eps, o, lse, workspace, W, scale, stream)
    return o, lse


def attn_fwd_rope(q, k, v, q_rot, k_rot, o, lse, cos, sin, eps: float, W: int, scale=None, stream=None):
    """Training forward with the prologue; q_rot, k_rot receive the rotated, normalised inputs."""
    B, T, H, D = _bthd(q, q_rot, o)
    Hkv = _kv_heads((B, T, H, D), k, k_rot, v)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, T) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, T] tensor")
    max_pos = _tables(cos, sin, D)
    _check(_lib.attn_fwd_rope(_ptr(q), _ptr(k), _ptr(v), _ptr(q_rot), _ptr(k_rot), _ptr(o), _ptr(lse), _ptr(cos),
                              _ptr(sin), max_pos, float(eps), B, T, H, Hkv, D, int(W), _scale(scale, D),
                              _stream(stream)), "attn_fwd_rope")


def attn_bwd_rope(q, k, q_rot, k_rot, v, o, lse, dout, dq, dk, dv, workspace, cos, sin, eps: float, W: int, scale=None,
                  stream=None):
    """Training backward with the prologue: dq, dk, dv with respect to the raw q, k, v."""
    B, T, H, D = _bthd(q, q_rot, o, dout, dq)
    Hkv = _kv_heads((B, T, H, D), k, k_rot, v, dk, dv)
    max_pos = _tables(cos, sin, D)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.attn_bwd_rope(_ptr(q), _ptr(k), _ptr(q_rot), _ptr(k_rot), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                              _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, _ptr(cos), _ptr(sin), max_pos,
                              float(eps), B, T, H, Hkv, D, int(W), _scale(scale, D), _stream(stream)), "attn_bwd_rope")
