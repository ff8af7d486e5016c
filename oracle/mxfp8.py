"""fp64 emulation of an FP8 forward with microscaling (MX) block scales.

TEST INFRASTRUCTURE ONLY: see the package docstring for who may import this.

"FlashAttention-3: Fast and Accurate Attention with Asynchrony and
Low-precision" (abstract) names block quantisation for FP8 without fixing the
block. This module is the reading in which the blocks are the ones B200's
tensor cores scale in hardware: the Open Compute Project "OCP Microscaling
Formats (MX) Specification" v1.0, format MXFP8 (E4M3): blocks of 32
consecutive elements along the contraction dimension of a product share one
power-of-two scale (an E8M0 exponent). Following the specification's
conversion:

* shared exponent e = floor(log2(max |v|)) - 8 (8 = the largest normal
  exponent of E4M3), clamped to the E8M0 range [-127, 127]; a block of zeros
  takes e = -127;
* elements v / 2^e rounded to E4M3 (nearest, ties to even) and clamped to
  +-448, the largest finite E4M3 value (so a block whose largest magnitude has
  a significand above 1.75 loses its top values to the clamp).

A second rule, "fit", takes the smallest exponent that needs no clamp. On the
FP8 workload's input recipe the clamp costs accuracy: with the rotation, the
"fit" rule tracks exact attention about as closely as one exact-amax scale per
64 rows x d, and the specification's rule about 10-20 % less closely
(measured here on seeded inputs; ``tests/test_oracle_mxfp8_pins.py``).

The quotient v / 2^e is exact in float32 for the inputs used here, so the code
is decided in float32 as in the per-block FP8 reading (``oracle/fp8.py``).

Attention (readings, stated here because the sources give none):

* S = Q K^T contracts over d: Q and K rows are quantised in blocks of 32
  columns. Optionally Q and K are first rotated by diag(sigma) H_d as in the
  FP8 path (the 1/d folds into the softmax scale).
* O = P V contracts over the keys: V is quantised in blocks of 32 keys of each
  column, and so is P, per row, tile by tile.
* Keys are visited 128 at a time with a running max m (exact by default, so
  P <= 1; optionally raised only past tau, as the bf16 path defers its
  rescale): P = exp2(c S - m) rounded to float32, then MX-quantised along the
  keys of the tile; the row sum l accumulates the unquantised P; O = acc / l.

Parity pins (``tests/test_oracle_mxfp8_pins.py``): closed-form blocks from the
conversion rule (scale, clamp, zero block, where the two rules differ), the
power-of-two scale and the range of each block's largest code, the element
error bound, exact agreement with ``oracle.attention_forward`` when every
operand is exactly representable and P is left unquantised, the error bound of
P's quantisation otherwise, the blocking axes of Q, K and V (closed forms), the
E8M0 exponent range, a query row's independence of the other rows (P blocked
along the keys of its own row), GQA against repeated KV heads, and seeded
comparisons with per-tensor FP8 and the 64-row-block FP8
emulation on inputs with outliers. ``tests/test_oracle_mxfp8_mutations.py``
plants mistakes in a copy of this module and checks the pins catch them.
"""

from __future__ import annotations

import math

import numpy as np

from .fp8 import E4M3_MAX, e4m3_round, rotate_rows

MX_BLOCK = 32
E4M3_EMAX = 8          # largest normal exponent of E4M3 (448 = 1.75 * 2^8)
E8M0_MIN, E8M0_MAX = -127, 127


def mx_quantize(x, axis: int = -1, block: int = MX_BLOCK, rule: str = "ocp"):
    """MXFP8 (E4M3) quantisation of ``x`` along ``axis`` in blocks of ``block``
    consecutive elements (a ragged last block is padded with zeros for the
    scale). Returns (codes as float32 values on the E4M3 grid, shape of x;
    int exponents e, one per block: x ~ codes * 2^e).

    rule "ocp": the specification's e = floor(log2 amax) - 8, with the codes
    clamped at +-448 (a block whose largest magnitude has a significand above
    1.75 loses its top values to the clamp). rule "fit": the smallest e with
    amax / 2^e <= 448, i.e. one more than "ocp" exactly when the significand
    of amax exceeds 1.75, so nothing is clamped (a software choice the E8M0
    format allows equally)."""
    if rule not in ("ocp", "fit"):
        raise ValueError("rule must be 'ocp' or 'fit'")
    x = np.moveaxis(np.asarray(x, np.float64), axis, -1)
    n = x.shape[-1]
    nb = -(-n // block)
    pad = nb * block - n
    xp = np.concatenate([x, np.zeros(x.shape[:-1] + (pad,))], axis=-1) if pad else x
    xb = xp.reshape(x.shape[:-1] + (nb, block))
    amax = np.max(np.abs(xb), axis=-1)
    m, E = np.frexp(amax)                              # amax = m 2^E, m in [0.5, 1)
    e = E - 1 - E4M3_EMAX                              # floor(log2 amax) - 8
    if rule == "fit":
        e = e + (m > 0.875)                            # significand above 1.75: 448 < amax / 2^e
    e = np.where(amax > 0, e, E8M0_MIN)
    e = np.clip(e, E8M0_MIN, E8M0_MAX).astype(np.int64)
    scaled = (xb * np.ldexp(1.0, -e)[..., None]).astype(np.float32)
    codes = e4m3_round(np.clip(scaled, -E4M3_MAX, E4M3_MAX))
    codes = codes.reshape(xp.shape)[..., :n]
    return np.moveaxis(codes, -1, axis), np.moveaxis(e, -1, axis)


def mx_dequantize(codes, e, axis: int = -1, block: int = MX_BLOCK) -> np.ndarray:
    """codes * 2^e, with each block's exponent broadcast over its elements."""
    codes = np.moveaxis(np.asarray(codes, np.float64), axis, -1)
    e = np.moveaxis(np.asarray(e), axis, -1)
    n = codes.shape[-1]
    scale = np.repeat(np.ldexp(1.0, e), block, axis=-1)[..., :n]
    return np.moveaxis(codes * scale, -1, axis)


def mx_roundtrip(x, axis: int = -1, block: int = MX_BLOCK, rule: str = "ocp") -> np.ndarray:
    """The float64 values an MXFP8 tensor represents after quantising x."""
    c, e = mx_quantize(x, axis, block, rule)
    return mx_dequantize(c, e, axis, block)


def mxfp8_attention_forward(q, k, v, causal: bool, scale: float, sigma=None, tile: int = 128,
                            quantize_p: bool = True, rule: str = "ocp", tau: float = 0.0):
    """Emulate the MXFP8 forward (readings in the module docstring) in
    float64, with the scale rule of ``mx_quantize``. ``quantize_p=False``
    leaves P unquantised (used to pin the score and softmax assembly).
    ``tau`` > 0 lets a row keep its running max until a tile's max exceeds
    it by more than tau (log2 units), as the bf16 path's deferred rescale
    does; P then reaches up to 2^tau, which MX block scales absorb.
    Returns (O, LSE) with LSE in natural log."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    if sigma is not None:
        q = rotate_rows(q, sigma).astype(np.float32).astype(np.float64)
        k = rotate_rows(k, sigma).astype(np.float32).astype(np.float64)
        sfac = scale / d
    else:
        sfac = scale
    qh = mx_roundtrip(q.astype(np.float32), axis=-1, rule=rule)    # blocks of 32 along d
    kh = mx_roundtrip(k.astype(np.float32), axis=-1, rule=rule)
    vh = mx_roundtrip(v.astype(np.float32), axis=-2, rule=rule)    # blocks of 32 keys per column
    c = sfac * math.log2(math.e)
    o = np.empty((B, Hq, N, d))
    lse = np.empty((B, Hq, N))
    rows = np.arange(N)
    for b in range(B):
        for h in range(Hq):
            kvh = h // g
            m = np.full(N, -np.inf)
            l = np.zeros(N)
            acc = np.zeros((N, d))
            for j0 in range(0, N, tile):
                j1 = min(N, j0 + tile)
                s = c * (qh[b, h] @ kh[b, kvh, j0:j1].T)
                if causal:
                    s = np.where(np.arange(j0, j1)[None, :] > rows[:, None], -np.inf, s)
                tmax = np.max(s, axis=1)
                m_new = np.where(tmax > m + tau, np.maximum(m, tmax), m)
                m_use = np.where(np.isneginf(m_new), 0.0, m_new)
                alpha = np.where(np.isneginf(m), 0.0, np.exp2(m - m_use))
                p = np.exp2(s - m_use[:, None]).astype(np.float32).astype(np.float64)
                l = l * alpha + p.sum(axis=1)
                pq = mx_roundtrip(p, axis=-1, rule=rule) if quantize_p else p
                acc = acc * alpha[:, None] + pq @ vh[b, kvh, j0:j1]
                m = m_new
            o[b, h] = acc / l[:, None]
            lse[b, h] = (m + np.log2(l)) * math.log(2.0)
    return o, lse
