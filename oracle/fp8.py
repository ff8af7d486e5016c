"""fp64 emulation of the block-quantised, Hadamard-rotated FP8 forward.

TEST INFRASTRUCTURE ONLY: see the package docstring for who may import this.

"FlashAttention-3: Fast and Accurate Attention with Asynchrony and
Low-precision" (abstract) names two steps for FP8: block quantisation (one
scale per block rather than per tensor) and incoherent processing (rotating Q
and K so that outliers spread before quantisation), and compares against a
baseline FP8 attention. The abstract gives neither the block shape nor the
rotation. Readings used here:

* Block: 64 consecutive rows x all d columns of one (batch, head) matrix; one
  float32 scale per block, s = amax / 448, s = 1 for an all-zero block.
* Rotation: y = x diag(sigma) H_d, with H_d the Sylvester Hadamard matrix and
  sigma a +-1 vector shared by Q and K, so (Q R)(K R)^T = d Q K^T exactly. The
  1/d is folded into the softmax scale (a power of two for d = 64 and 128).
  V is not rotated.
* Format: e4m3 with no infinities (largest finite 448), round to nearest even,
  saturating. The quantised code is decided in float32, the precision the
  kernel uses: y is rounded once to float32, inv = 448 / amax and y * inv are
  single float32 operations, then rounded to e4m3.
* P: within each 128-key tile, P = exp2(c S - m) with a running max m that a
  row raises only when the tile's max exceeds it by more than tau = 0.8
  (log2 units; the same stale max enters the row sum and O, so the result is
  the softmax's), multiplied by w = sV(key block) / max(sV) * 256 and rounded
  to e4m3; the 256 and max(sV) are undone at the end. This folds V's
  per-block scale into P; 2^0.8 * 256 = 445.7 keeps P w below 448.
* Baseline FP8: one amax scale per tensor for each of Q, K and V, no rotation,
  exact softmax with the row's final maximum, and the unnormalised P~ =
  exp(S - m) rounded to e4m3 with no scale factor (the quantity a tiled
  kernel multiplies by V; the division by the row sum comes once at the
  end). Rounding the normalised probabilities instead is kept as an option:
  at large N most of them fall below e4m3's subnormals, which would make the
  baseline look far worse than a real FP8 kernel.

Parity pins: ``e4m3_round`` against torch's float8_e4m3fn conversion for
in-range values; ``hadamard`` by orthogonality and the Sylvester recursion;
``block_quantize`` by the largest element mapping to 448 and a half-quantum
error bound; ``fp8_attention_forward`` against exact attention within the
error bound of e4m3 rounding, and against its own single-tile reading (P
rounded against the row's final maximum) within two half-quanta of P;
``per_tensor_quantize`` and ``naive_fp8_attention_forward`` by closed forms
on inputs already on the e4m3 grid (hand-computed codes of P, both P forms,
per-tensor rather than per-head scales). The ratio of
FP8 errors the abstract reports (2.6x) is parity unpinned: it is reported, not
asserted.
"""

from __future__ import annotations

import math

import numpy as np

E4M3_MAX = 448.0
_E4M3_MIN_NORMAL_EXP = -6   # smallest normal is 2^-6
_E4M3_MANT_BITS = 3


def hadamard(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix H_d (entries +-1, H H^T = d I), d a power of 2."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def rotate_rows(x, sigma) -> np.ndarray:
    """y = x diag(sigma) H_d along the last axis, in float64.

    For bf16 inputs every sum is exact in float64 (8-bit significands, at most
    d = 128 terms), so y does not depend on summation order.
    """
    x = np.asarray(x, np.float64)
    sigma = np.asarray(sigma, np.float64)
    return (x * sigma) @ hadamard(x.shape[-1])


def e4m3_round(x) -> np.ndarray:
    """Round float32 values to the e4m3 grid: nearest, ties to even, saturating
    at +-448. Returns float32 values on the grid."""
    x = np.asarray(x, np.float32).astype(np.float64)
    ax = np.abs(x)
    _, E = np.frexp(ax)                       # ax = m 2^E, m in [0.5, 1)
    e = np.maximum(E - 1, _E4M3_MIN_NORMAL_EXP)
    quantum = np.ldexp(1.0, e - _E4M3_MANT_BITS)
    r = np.round(ax / quantum) * quantum      # np.round: half to even
    r = np.minimum(r, E4M3_MAX)
    return (np.sign(x) * r).astype(np.float32)


def e4m3_encode(vals) -> np.ndarray:
    """Bit codes (uint8) of values already on the e4m3 grid."""
    v = np.asarray(vals, np.float64)
    sign = (np.signbit(v)).astype(np.uint8) << 7
    a = np.abs(v)
    _, E = np.frexp(a)
    e = E - 1
    normal = a >= 2.0 ** _E4M3_MIN_NORMAL_EXP
    exp_field = np.where(normal, e + 7, 0)
    mant = np.where(normal, a / np.ldexp(1.0, e) - 1.0, a / 2.0 ** (_E4M3_MIN_NORMAL_EXP)) * 8.0
    mant = np.where(a == 0, 0, mant)
    exp_field = np.where(a == 0, 0, exp_field)
    return (sign | (exp_field.astype(np.uint8) << 3) | np.rint(mant).astype(np.uint8)).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """Values (float64) of e4m3 codes; 0x7F and 0xFF are NaN."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


def block_quantize(y, block_rows: int = 64):
    """Quantise [..., N, d] to e4m3 with one float32 scale per block of
    ``block_rows`` rows. Returns (values on the e4m3 grid as float32 [..., N, d],
    scales float32 [..., ceil(N / block_rows)])."""
    y32 = np.asarray(y, np.float64).astype(np.float32)
    *lead, N, d = y32.shape
    nb = -(-N // block_rows)
    vals = np.empty_like(y32)
    scales = np.empty((*lead, nb), np.float32)
    for bi in range(nb):
        blk = y32[..., bi * block_rows:(bi + 1) * block_rows, :]
        amax = np.max(np.abs(blk), axis=(-2, -1)).astype(np.float32)
        nz = amax > 0
        safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
        inv = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)
        scales[..., bi] = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
        scaled = (blk * inv[..., None, None]).astype(np.float32)
        vals[..., bi * block_rows:(bi + 1) * block_rows, :] = e4m3_round(scaled)
    return vals, scales


def _expand_rows(scales, N, block_rows):
    return np.repeat(np.asarray(scales, np.float64), block_rows, axis=-1)[..., :N]


FP8_TAU = 0.8


def fp8_attention_forward(q, k, v, causal: bool, scale: float, sigma=None,
                          block_rows: int = 64, tile: int = 128, p_lift: float = 256.0, tau: float = FP8_TAU):
    """Emulate the FP8 forward (readings in the module docstring) in float64.

    Q and K are rotated with ``sigma`` (skipped when None), all three are block
    quantised, scores come from the dequantised operands, and keys are visited
    ``tile`` at a time. Each row keeps a running max that it raises to the
    tile's max only when that exceeds it by more than ``tau`` (log2 units;
    ``tau = 0`` is the exact running max), so P <= 2^tau; P is rounded to
    e4m3 after folding in V's block scale (P w <= 2^tau * p_lift, below 448
    for tau = 0.8, p_lift = 256). Returns (O, LSE).
    """
    if 2.0 ** tau * p_lift > E4M3_MAX:
        raise ValueError("2^tau * p_lift must stay within e4m3's range")
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    if sigma is not None:
        q, k = rotate_rows(q, sigma), rotate_rows(k, sigma)
        sfac = scale / d
    else:
        sfac = scale
    qv, qs = block_quantize(q, block_rows)
    kv_, ks = block_quantize(k, block_rows)
    vv, vs = block_quantize(v, block_rows)
    qh = qv.astype(np.float64) * _expand_rows(qs, N, block_rows)[..., None]
    kh = kv_.astype(np.float64) * _expand_rows(ks, N, block_rows)[..., None]
    c = sfac * math.log2(math.e)
    o = np.empty((B, Hq, N, d))
    lse = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            kvh = h // g
            vref = float(np.max(vs[b, kvh]))
            wkey = _expand_rows(vs[b, kvh], N, block_rows) / vref * p_lift
            m = np.full(N, -np.inf)
            l = np.zeros(N)
            acc = np.zeros((N, d))
            for j0 in range(0, N, tile):
                j1 = min(N, j0 + tile)
                s = c * (qh[b, h] @ kh[b, kvh, j0:j1].T)
                if causal:
                    s = np.where(np.arange(j0, j1)[None, :] > np.arange(N)[:, None], -np.inf, s)
                tmax = np.max(s, axis=1)
                m_new = np.where(tmax > m + tau, np.maximum(m, tmax), m)
                alpha = np.where(np.isneginf(m), 0.0, np.exp2(m - m_new))
                p = np.exp2(s - m_new[:, None])
                l = l * alpha + p.sum(axis=1)
                pq = e4m3_round((p * wkey[None, j0:j1]).astype(np.float32)).astype(np.float64)
                acc = acc * alpha[:, None] + pq @ vv[b, kvh, j0:j1].astype(np.float64)
                m = m_new
            o[b, h] = acc * (vref / p_lift) / l[:, None]
            lse[b, h] = (m + np.log2(l)) * math.log(2.0)
    return o, lse


def per_tensor_quantize(x):
    """One e4m3 scale for the whole tensor: s = amax / 448 (1 when amax = 0),
    codes e4m3(x * (448 / amax)) decided in float32. Returns (values on the
    e4m3 grid as float64, s)."""
    x32 = np.asarray(x, np.float64).astype(np.float32)
    amax = np.max(np.abs(x32)).astype(np.float32)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0)).astype(np.float32)
    inv = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)
    s = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float64)
    return e4m3_round((x32 * inv).astype(np.float32)).astype(np.float64), s


def naive_fp8_attention_forward(q, k, v, causal: bool, scale: float, row_chunk: int = 2048, heads=None,
                                p_form: str = "unnormalised"):
    """Baseline FP8 attention: one amax scale per tensor for each of Q, K and
    V, no rotation, exact softmax with the row's final maximum, and P rounded
    to e4m3 with no extra scale factor. ``p_form`` says which P is rounded:

    * "unnormalised" (the baseline reported): P~ = exp(S - m) in (0, 1], the
      quantity a tiled kernel feeds to its P V product (the division by the
      row sum comes once at the end), so O = (e4m3(P~) V) / sum_j P~.
    * "normalised": the softmax probabilities exp(S - m) / sum_j exp(S - m)
      themselves, O = e4m3(P) V. At large N most of them fall below e4m3's
      subnormal range and round to zero, so this form is far less accurate.

    Returns O. Query rows are formed ``row_chunk`` at a time (each row still
    sees all of its keys). ``heads``, a list of (b, h), limits which heads'
    outputs are computed (the others are NaN); the scales still come from the
    whole tensors."""
    if p_form not in ("unnormalised", "normalised"):
        raise ValueError(p_form)
    qv, qs = per_tensor_quantize(q)
    kv_, ks = per_tensor_quantize(k)
    vv, vs = per_tensor_quantize(v)
    qh, kh = qv * qs, kv_ * ks
    vs = np.broadcast_to(vs, vv.shape[:2] + (1, 1))   # one value per (b, kv head): the tensor's scale
    B, Hq, N, d = qh.shape
    g = Hq // kh.shape[1]
    o = np.full((B, Hq, N, d), np.nan)
    todo = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else list(heads)
    for b, h in todo:
        for r0 in range(0, N, row_chunk):
            r1 = min(N, r0 + row_chunk)
            s = scale * (qh[b, h, r0:r1] @ kh[b, h // g].T)
            if causal:
                s = np.where(np.arange(N)[None, :] > np.arange(r0, r1)[:, None], -np.inf, s)
            e = np.exp(s - np.max(s, axis=1, keepdims=True))
            l = e.sum(axis=1, keepdims=True)
            if p_form == "normalised":
                pq = e4m3_round((e / l).astype(np.float32)).astype(np.float64)
                o[b, h, r0:r1] = (pq @ vv[b, h // g]) * vs[b, h // g]
            else:
                pq = e4m3_round(e.astype(np.float32)).astype(np.float64)
                o[b, h, r0:r1] = (pq @ vv[b, h // g]) * vs[b, h // g] / l
    return o
