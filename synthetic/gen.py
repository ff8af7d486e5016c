"""Counter-based seeded generator for the attention workloads.

Every random number comes from SplitMix64 (Steele, Lea and Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014), used as a counter
based generator: output i of a stream is the SplitMix64 finaliser applied to
``key + (i + 1) * GAMMA``. The key of a stream is itself output ``stream`` of
the generator seeded with the base seed. Normal deviates come from the
Box-Muller transform; tensors are drawn in float64, rounded to float32 and then
to bfloat16 with round-to-nearest-even. The bfloat16 values are the canonical
inputs for both the GPU path and the fp64 oracle.

Nothing here computes attention; the module only draws numbers.
"""

from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_Q = 0
STREAM_K = 1
STREAM_V = 2
STREAM_DO = 3
STREAM_OUTLIER = 4
STREAM_SIGN = 5

# Element counters of the three outlier masks (Q, K, V) are offset by this
# much so that the masks are independent draws from one stream.
_OUTLIER_TENSOR_OFFSET = 1 << 40

_CHUNK = 1 << 23


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output finaliser on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, counters: np.ndarray) -> np.ndarray:
    """Outputs number ``counters`` (0-based) of SplitMix64 seeded with ``seed``."""
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (c + np.uint64(1)) * GAMMA)


def _stream_key(seed: int, stream: int) -> int:
    return int(splitmix64(seed, np.array([stream], dtype=np.uint64))[0])


def uniform01(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    """n uniforms in [0, 1) with 53 random bits, from one stream."""
    key = _stream_key(seed, stream)
    out = np.empty(n, dtype=np.float64)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        z = splitmix64(key, np.arange(offset + s, offset + e, dtype=np.uint64))
        out[s:e] = (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return out


def normal(seed: int, stream: int, n: int) -> np.ndarray:
    """n standard normal deviates (float64) by Box-Muller on counter pairs."""
    key = _stream_key(seed, stream)
    npairs = (n + 1) // 2
    out = np.empty(2 * npairs, dtype=np.float64)
    for s in range(0, npairs, _CHUNK):
        e = min(npairs, s + _CHUNK)
        idx = np.arange(s, e, dtype=np.uint64)
        z1 = splitmix64(key, idx * np.uint64(2))
        z2 = splitmix64(key, idx * np.uint64(2) + np.uint64(1))
        u1 = ((z1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)  # (0, 1]
        u2 = (z2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)          # [0, 1)
        r = np.sqrt(-2.0 * np.log(u1))
        t = 2.0 * np.pi * u2
        out[2 * s:2 * e:2] = r * np.cos(t)
        out[2 * s + 1:2 * e:2] = r * np.sin(t)
    return out[:n]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even.

    Inputs here are finite; NaN handling is not needed.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return ((b + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 values (exact)."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bfloat16 value; returns float32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def sign_vector(seed: int, d: int) -> np.ndarray:
    """Random +-1 vector of length d: the sign of the top bit of SplitMix64
    outputs 0..d-1 of stream ``STREAM_SIGN`` under ``seed`` (+1 when the top
    bit is clear). Returned as float64."""
    key = _stream_key(seed, STREAM_SIGN)
    z = splitmix64(key, np.arange(d, dtype=np.uint64))
    return 1.0 - 2.0 * (z >> np.uint64(63)).astype(np.float64)


def attention_inputs(B: int, Hq: int, Hkv: int, N: int, d: int, seed: int,
                     outlier_rate: float = 0.0, outlier_mult: float = 10.0,
                     with_dout: bool = True) -> dict:
    """Seeded bf16 inputs Q [B,Hq,N,d], K and V [B,Hkv,N,d], dO [B,Hq,N,d].

    Returns bf16 bit patterns (uint16). With ``outlier_rate`` > 0, each entry of
    Q, K and V is independently multiplied by ``outlier_mult`` with that
    probability (three independent masks) before rounding to bf16.
    """
    shapes = {"q": (B, Hq, N, d), "k": (B, Hkv, N, d), "v": (B, Hkv, N, d)}
    streams = {"q": STREAM_Q, "k": STREAM_K, "v": STREAM_V}
    out = {}
    for t, (name, shp) in enumerate(shapes.items()):
        n = int(np.prod(shp))
        x = normal(seed, streams[name], n)
        if outlier_rate > 0.0:
            u = uniform01(seed, STREAM_OUTLIER, n, offset=t * _OUTLIER_TENSOR_OFFSET)
            x = np.where(u < outlier_rate, x * outlier_mult, x)
        out[name] = f32_to_bf16_bits(x.astype(np.float32)).reshape(shp)
    if with_dout:
        n = B * Hq * N * d
        out["do"] = f32_to_bf16_bits(normal(seed, STREAM_DO, n).astype(np.float32)).reshape(B, Hq, N, d)
    return out
