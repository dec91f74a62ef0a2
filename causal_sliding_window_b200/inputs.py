"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no attention arithmetic. It only produces the bf16 bit
patterns that both the CUDA path and the fp64 oracle consume, so the two sides
always see identical inputs.

Generator (counter-based, reproducible on any machine):
  * splitmix64 finaliser (Steele, Lea & Flood, "Fast splittable pseudorandom
    number generators", OOPSLA 2014) applied to ``key + (i + 1) * 0x9E3779B97F4A7C15``
    for element counter ``i``; ``key`` mixes the seed with a per-tensor tag.
  * Box-Muller (cosine branch) on two 53-bit uniforms per normal.
  * float64 -> float32 (round to nearest even) -> bf16 (round to nearest even).

Workload shapes follow the nanochat depth family described on the pages
(width = 64 * depth, head dim 128, sequence 2048): depth 12 -> 6 heads,
depth 24 -> 12 heads, depth 26 -> 13 heads.
"""
from __future__ import annotations

import os

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Per-tensor tags, so Q, K, V, dO and the caches drawn from one seed differ.
TAGS = {"q": 1, "k": 2, "v": 3, "do": 4, "kcache": 5, "vcache": 6, "qdec": 7, "cache_len": 8}


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, tag: int) -> np.uint64:
    with np.errstate(over="ignore"):
        z = np.array([(seed * 0x632BE59BD9B4E019 + tag * 0xD1B54A32D192ED03) & 0xFFFFFFFFFFFFFFFF],
                     dtype=np.uint64)
        return _mix(z)[0]


def _u64_stream(seed: int, tag: int, start: int, count: int) -> np.ndarray:
    key = _key(seed, tag)
    with np.errstate(over="ignore"):
        ctr = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix(key + ctr * _GOLDEN)


def normal_f64(seed: int, tag: int, n: int, chunk: int = 1 << 22) -> np.ndarray:
    """n standard normals (float64) from the counter-based stream (seed, tag).

    Chunks are independent (the stream is counter-based), so they are filled
    by a thread pool; the result does not depend on the chunking.
    """
    out = np.empty(n, dtype=np.float64)
    inv = 1.0 / 9007199254740992.0  # 2**-53

    def fill(s: int):
        c = min(chunk, n - s)
        u = _u64_stream(seed, tag, 2 * s, 2 * c)
        u1 = ((u[0::2] >> np.uint64(11)).astype(np.float64) + 0.5) * inv
        u2 = ((u[1::2] >> np.uint64(11)).astype(np.float64) + 0.5) * inv
        out[s:s + c] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)

    starts = range(0, n, chunk)
    if n <= chunk:
        for s in starts:
            fill(s)
    else:
        from concurrent.futures import ThreadPoolExecutor

        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    return out


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 -> float32 (RNE) -> bf16 (RNE); returns uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((f >> np.uint32(16)) & np.uint32(1))
    return ((f + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16(seed: int, tag: str, shape) -> np.ndarray:
    """bf16 bits (uint16 array of ``shape``) drawn i.i.d. N(0, 1)."""
    n = int(np.prod(shape))
    return f64_to_bf16_bits(normal_f64(seed, TAGS[tag], n)).reshape(shape)


def rms_peaky_bf16(seed: int, tag: str, shape, gain: float = 1.5) -> np.ndarray:
    """Rows along the last axis RMS-normalised (no epsilon) then multiplied by ``gain``.

    This is the depth-26 input recipe: the nanochat model applies QK norm before
    attention (apidog guide "Train your own ChatGPT", section 1, architecture
    features), so the kernel sees unit-RMS rows; the gain of 1.5 sharpens the
    softmax.
    """
    n = int(np.prod(shape))
    x = normal_f64(seed, TAGS[tag], n).reshape(-1, shape[-1])
    x = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True)) * gain
    return f64_to_bf16_bits(x).reshape(shape)


def uniform_int(seed: int, tag: str, n: int, lo: int, hi: int) -> np.ndarray:
    """n integers uniform in [lo, hi] (inclusive), int32."""
    u = _u64_stream(seed, TAGS[tag], 0, n)
    span = np.uint64(hi - lo + 1)
    return (lo + (u % span).astype(np.int64)).astype(np.int32)


# ---------------------------------------------------------------------------
# Named workloads. Each returns a dict of bf16-bit numpy arrays plus metadata.
# ---------------------------------------------------------------------------

def attention_inputs(B: int, T: int, H: int, D: int, seed: int, peaky: bool = False,
                     with_do: bool = True) -> dict:
    shape = (B, T, H, D)
    if peaky:
        q = rms_peaky_bf16(seed, "q", shape)
        k = rms_peaky_bf16(seed, "k", shape)
    else:
        q = normal_bf16(seed, "q", shape)
        k = normal_bf16(seed, "k", shape)
    v = normal_bf16(seed, "v", shape)
    out = {"q": q, "k": k, "v": v, "B": B, "T": T, "H": H, "D": D, "scale": 1.0 / np.sqrt(D)}
    if with_do:
        out["do"] = normal_bf16(seed, "do", shape)
    return out


def decode_inputs(B: int, cap: int, H: int, D: int, seed: int, len_lo: int = 1,
                  len_hi: int | None = None, cache_len: np.ndarray | None = None) -> dict:
    if len_hi is None:
        len_hi = cap
    if cache_len is None:
        cache_len = uniform_int(seed, "cache_len", B, len_lo, len_hi)
    return {
        "q": normal_bf16(seed, "qdec", (B, H, D)),
        "k_cache": normal_bf16(seed, "kcache", (B, cap, H, D)),
        "v_cache": normal_bf16(seed, "vcache", (B, cap, H, D)),
        "cache_len": np.asarray(cache_len, dtype=np.int32),
        "B": B, "cap": cap, "H": H, "D": D, "scale": 1.0 / np.sqrt(D),
    }


# The five workloads of the target: (name, B, T, H, D, windows, seed, peaky).
WORKLOADS = {
    "tiny": dict(B=1, T=128, H=2, D=64, windows=(128, 32), seed=0, peaky=False),
    "d12": dict(B=32, T=2048, H=6, D=128, windows=(2048, 1024), seed=12, peaky=False),
    "d24": dict(B=32, T=2048, H=12, D=128, windows=(512, 512, 512, 2048), seed=24, peaky=False),
    "d26": dict(B=32, T=2048, H=13, D=128, windows=(2048, 256), seed=26, peaky=True),
}
DECODE_WORKLOAD = dict(B=32, cap=2048, H=12, D=128, windows=(2048, 1024), seed=1000)
