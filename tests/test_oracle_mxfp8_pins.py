"""Pins for the MXFP8 emulation (oracle/mxfp8.py): the conversion rule on
closed-form blocks, the range and error bound it implies, and the attention
assembly against exact attention."""

import math

import numpy as np
import pytest

import oracle
from oracle import mxfp8 as mx
from oracle.fp8 import E4M3_MAX, fp8_attention_forward, naive_fp8_attention_forward
from synthetic import attention_inputs, bf16_bits_to_f32, sign_vector


def _rng(seed):
    return np.random.default_rng(seed)


# --- the conversion rule -------------------------------------------------------

def test_closed_form_blocks():
    """amax 1 -> e = 0 - 8, codes = v * 2^8; amax 3 -> e = 1 - 8 (3 * 2^7 =
    384, on the grid); amax 7.5 -> e = 2 - 8 and 7.5 * 2^6 = 480 clamps to 448
    (dequantised 7.0)."""
    x = np.zeros((3, 32))
    x[0, :4] = [1.0, 0.5, -0.25, 0.125]
    x[1, :2] = [3.0, -1.5]
    x[2, :2] = [7.5, 1.0]
    codes, e = mx.mx_quantize(x)
    np.testing.assert_array_equal(e[:, 0], [-8, -7, -6])
    np.testing.assert_array_equal(codes[0, :4], [256.0, 128.0, -64.0, 32.0])
    np.testing.assert_array_equal(codes[1, :2], [384.0, -192.0])
    np.testing.assert_array_equal(codes[2, :2], [448.0, 64.0])
    back = mx.mx_dequantize(codes, e)
    assert back[2, 0] == 7.0 and back[1, 0] == 3.0


def test_fit_rule_differs_only_above_significand_1_75():
    """The "fit" exponent is the specification's plus one exactly when amax's
    significand exceeds 1.75; then nothing is clamped (7.5 -> e = 3 - 8,
    7.5 * 2^5 = 240 on the grid)."""
    x = np.zeros((4, 32))
    x[:, 0] = [1.75, 1.7500001, 7.5, 1.0]
    c_ocp, e_ocp = mx.mx_quantize(x, rule="ocp")
    c_fit, e_fit = mx.mx_quantize(x, rule="fit")
    np.testing.assert_array_equal(e_fit[:, 0] - e_ocp[:, 0], [0, 1, 1, 0])
    assert c_fit[2, 0] == 240.0 and mx.mx_dequantize(c_fit, e_fit)[2, 0] == 7.5
    assert c_ocp[1, 0] == 448.0                      # clamped under the specification's rule
    y = _rng(12).standard_normal((256, 64)) * 3
    cf, ef = mx.mx_quantize(y, rule="fit")
    scale = np.repeat(np.ldexp(1.0, ef), 32, axis=-1)
    assert np.all(np.abs(y / scale) <= E4M3_MAX)    # no element needs the clamp
    top = np.max(np.abs(cf.reshape(256, 2, 32)), axis=-1)
    assert np.all((top >= 224) & (top <= E4M3_MAX))


def test_zero_block_and_ragged_tail():
    x = np.zeros((2, 40))
    x[1, 33] = 2.0                       # only in the ragged second block of row 1
    codes, e = mx.mx_quantize(x)
    assert e.shape == (2, 2)
    assert e[0, 0] == e[0, 1] == e[1, 0] == -127 and e[1, 1] == 1 - 8
    assert np.all(codes[0] == 0) and codes[1, 33] == 256.0 and np.count_nonzero(codes) == 1


def test_exponent_clamped_to_the_e8m0_range():
    """E8M0 holds exponents -127..127. A block with amax 2^-130 (reachable from
    bf16 subnormals) takes e = -127, not -138, and keeps its value as the
    code 2^-3; a block with amax 2^140 takes e = 127 and its code saturates
    at 448. Both rules (the significand is 1)."""
    x = np.zeros((2, 32))
    x[0, 0] = 2.0 ** -130
    x[1, 0] = 2.0 ** 140
    for rule in ("ocp", "fit"):
        codes, e = mx.mx_quantize(x, rule=rule)
        np.testing.assert_array_equal(e[:, 0], [-127, 127])
        assert codes[0, 0] == 0.125 and codes[1, 0] == E4M3_MAX
        assert mx.mx_dequantize(codes, e)[0, 0] == 2.0 ** -130


def test_scales_are_powers_of_two_and_largest_code_in_range():
    """Per block the largest |code| lies in [256, 448]: 2^8 <= amax / 2^e <
    2^9, clamped at 448."""
    x = _rng(1).standard_normal((64, 96)) * np.exp(_rng(2).uniform(-20, 20, (64, 1)))
    codes, e = mx.mx_quantize(x, axis=-1)
    top = np.max(np.abs(codes.reshape(64, 3, 32)), axis=-1)
    assert np.all((top >= 256) & (top <= E4M3_MAX))
    assert e.dtype.kind == "i"


def test_blocks_are_independent_and_follow_the_axis():
    x = _rng(3).standard_normal((32, 64))
    c0, e0 = mx.mx_quantize(x, axis=0)
    y = x.copy()
    y[:, 5] *= 1000.0                    # one column: only its (axis-0) block changes
    c1, e1 = mx.mx_quantize(y, axis=0)
    changed = np.nonzero(np.any(e0 != e1, axis=0))[0]
    np.testing.assert_array_equal(changed, [5])
    np.testing.assert_array_equal(np.delete(c0, 5, axis=1), np.delete(c1, 5, axis=1))


def test_element_error_bound():
    """Away from the clamp, |v - deq| <= 2^-4 |v| (half a quantum of a 3-bit
    mantissa) or, below E4M3's normal range, half the subnormal step 2^(e-10)."""
    x = _rng(4).standard_normal((128, 64)) * np.exp(_rng(5).uniform(-5, 5, (128, 64)))
    codes, e = mx.mx_quantize(x)
    back = mx.mx_dequantize(codes, e)
    scale = np.repeat(np.ldexp(1.0, e), 32, axis=-1)
    clamped = np.abs(x / scale) > E4M3_MAX
    err = np.abs(x - back)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, scale * 2.0 ** -10)
    assert np.all(err[~clamped] <= bound[~clamped] * (1 + 1e-12))


# --- attention ------------------------------------------------------------------

def _representable(shape, seed):
    """Values k/4, |k| <= 7: every 32-block quantises exactly (at most 3 bits of
    significand within a 2^9 range)."""
    return _rng(seed).integers(-7, 8, size=shape) / 4.0


@pytest.mark.parametrize("causal", [False, True])
def test_exact_when_operands_representable_and_p_unquantised(causal):
    """With Q, K, V on the MX grid and P left unquantised, the emulation is
    exact attention: pins the block-scaled score assembly (which operand is
    blocked along which axis) and the tile recurrence."""
    q, k, v = _representable((1, 2, 200, 64), 6), _representable((1, 1, 200, 64), 7), _representable((1, 1, 200, 64), 8)
    o_ref, lse_ref = oracle.attention_forward(q, k, v, causal, 0.125)
    for rule in ("ocp", "fit"):
        o, lse = mx.mxfp8_attention_forward(q, k, v, causal, 0.125, quantize_p=False, rule=rule)
        # P is held in float32 (relative error <= 2^-24 per value)
        np.testing.assert_allclose(o, o_ref, atol=2e-7)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-9)


def test_p_quantisation_error_bound():
    """With exact operands, quantising P moves O by at most
    sum_j |P_j - P^_j| |V_j| / l; each P^_j is within 2^-4 P_j, or within the
    subnormal floor 2^-9 of a block whose largest P is at most 1, so
    |O - O_exact| <= max|V| (2^-4 + 2^-9)."""
    q, k, v = _representable((1, 1, 256, 64), 9), _representable((1, 1, 256, 64), 10), _representable((1, 1, 256, 64), 11)
    o, _ = mx.mxfp8_attention_forward(q, k, v, False, 0.25)
    o_ref, _ = oracle.attention_forward(q, k, v, False, 0.25)
    assert np.max(np.abs(o - o_ref)) <= np.max(np.abs(v)) * (2.0 ** -4 + 2.0 ** -9)
    assert np.max(np.abs(o - o_ref)) > 0        # P really was quantised


def test_v_is_blocked_along_the_keys():
    """Q = 0 makes every P exactly 1 (a code of 256 at scale 2^-8), so O is the
    mean of the quantised V over the keys. V[0, 0] = 1e4 sets the scale of its
    block to 2^5; the rest of key 0's row holds 2^-5, which a 2^5 scale flushes
    to zero (2^-10 is half E4M3's smallest step) while a block of its own
    column (largest value 1.75, scale 2^-8) keeps it exactly. Blocked along the
    keys, every column but 0 of O is therefore exact."""
    v = _representable((1, 1, 64, 64), 13)
    v[0, 0, 0, 1:] = 2.0 ** -5
    v[0, 0, 0, 0] = 1.0e4
    q = np.zeros((1, 1, 64, 64))
    k = _representable((1, 1, 64, 64), 14)
    o, _ = mx.mxfp8_attention_forward(q, k, v, False, 0.125)
    exact = v[0, 0].mean(axis=0)
    np.testing.assert_array_equal(o[0, 0, :, 1:], np.broadcast_to(exact[1:], (64, 63)))


def test_k_is_blocked_along_d():
    """K[0, 0] = -1e4 against Q[:, 0] = 1 drives key 0's probability to 0; the
    other keys hold 2^-5 in column 0, kept exactly by blocks along d (their own
    rows) and flushed by a block along the keys that contains K[0, 0]. With P
    unquantised the emulation must then equal exact attention."""
    q = _representable((1, 1, 64, 64), 15)
    q[0, 0, :, 0] = 1.0
    k = _representable((1, 1, 64, 64), 16)
    k[0, 0, :, 0] = 2.0 ** -5
    k[0, 0, 0, 0] = -1.0e4
    v = _representable((1, 1, 64, 64), 17)
    o, _ = mx.mxfp8_attention_forward(q, k, v, False, 0.5, quantize_p=False)
    o_ref, _ = oracle.attention_forward(q, k, v, False, 0.5)
    np.testing.assert_allclose(o, o_ref, atol=2e-7)


def test_q_is_blocked_along_d():
    """Q[0, 0] = 1e4 and Q[i, 0] = 2^-5 for the other rows, against a column
    0 of K that varies by key (so the term does not cancel in the softmax):
    blocks along d keep rows 1.. exact, a block along the query rows that
    contains Q[0, 0] would flush their 2^-5. Row 0 itself is coarsened and
    left out."""
    q = _representable((1, 1, 64, 64), 18)
    q[0, 0, :, 0] = 2.0 ** -5
    q[0, 0, 0, 0] = 1.0e4
    k = _representable((1, 1, 64, 64), 19)
    v = _representable((1, 1, 64, 64), 20)
    o, _ = mx.mxfp8_attention_forward(q, k, v, False, 0.5, quantize_p=False)
    o_ref, _ = oracle.attention_forward(q, k, v, False, 0.5)
    np.testing.assert_allclose(o[0, 0, 1:], o_ref[0, 0, 1:], atol=2e-7)


def test_each_query_row_depends_only_on_its_own_q():
    """Q is blocked along d and P along the keys of one row, so a row's
    output does not depend on the other query rows: changing rows 1.. leaves
    row 0 as it was. (P blocked along the query rows would take each key's
    block exponent from 32 rows' probabilities and move row 0 with them.)"""
    rng = _rng(31)
    q, k, v = (rng.standard_normal((1, 1, 64, 64)) for _ in range(3))
    q2 = q.copy()
    q2[0, 0, 1:] = 4.0 * rng.standard_normal((63, 64))
    for rule in ("ocp", "fit"):
        o1, l1 = mx.mxfp8_attention_forward(q, k, v, False, 0.125, rule=rule)
        o2, l2 = mx.mxfp8_attention_forward(q2, k, v, False, 0.125, rule=rule)
        np.testing.assert_allclose(o2[0, 0, 0], o1[0, 0, 0], rtol=0, atol=1e-12)
        assert abs(l2[0, 0, 0] - l1[0, 0, 0]) <= 1e-12
        assert np.max(np.abs(o2[0, 0, 1:] - o1[0, 0, 1:])) > 1e-3


def test_gqa_equals_repeated_kv_heads():
    """Query head h reads KV head h // (Hq / Hkv): four query heads over two KV
    heads give what four KV heads 0, 0, 1, 1 give (the quantised copies of a
    KV head are the same whichever query head reads them)."""
    rng = _rng(32)
    q = rng.standard_normal((1, 4, 96, 64))
    k, v = (rng.standard_normal((1, 2, 96, 64)) for _ in range(2))
    rep = lambda t: np.repeat(t, 2, axis=1)
    for causal in (False, True):
        o, lse = mx.mxfp8_attention_forward(q, k, v, causal, 0.125, rule="fit", tile=32, tau=4.0)
        o2, lse2 = mx.mxfp8_attention_forward(q, rep(k), rep(v), causal, 0.125, rule="fit", tile=32, tau=4.0)
        np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [21, 22, 23])
def test_accuracy_on_the_fp8_input_recipe(seed):
    """On the FP8 workload's input recipe (0.1 % of entries x 10), with the
    rotation: both rules beat per-tensor FP8; the clamp-free rule beats the
    specification's; and it is within 10 % of one exact-amax scale per 64
    rows x d (the FP8 path's reading)."""
    bits = attention_inputs(1, 2, 2, 512, 128, seed=seed, outlier_rate=0.001, with_dout=False)
    q, k, v = (bf16_bits_to_f32(bits[n]).astype(np.float64) for n in ("q", "k", "v"))
    exact, _ = oracle.attention_forward(q, k, v, False, 128 ** -0.5)
    rms = lambda a: math.sqrt(float(np.mean(a ** 2)))
    sigma = sign_vector(3, 128)
    e_ocp = rms(mx.mxfp8_attention_forward(q, k, v, False, 128 ** -0.5, sigma=sigma, rule="ocp")[0] - exact)
    e_fit = rms(mx.mxfp8_attention_forward(q, k, v, False, 128 ** -0.5, sigma=sigma, rule="fit")[0] - exact)
    e_64 = rms(fp8_attention_forward(q, k, v, False, 128 ** -0.5, sigma=sigma)[0] - exact)
    e_naive = rms(naive_fp8_attention_forward(q, k, v, False, 128 ** -0.5) - exact)
    assert max(e_ocp, e_fit) < e_naive
    assert e_fit < e_ocp
    assert e_fit < 1.1 * e_64
    assert e_fit < 0.1 * rms(exact)


def test_mxfp8_deferred_max_two_tile_closed_form():
    """Two keys visited one per tile, log2-domain scores 0 and 0.5 (scale =
    ln 2; Q = e_0, K_1 = 0.5 e_0: codes 256 and 256 with exact block scales).
    With tau = 8 the second tile's max does not raise m = 0, so that tile's P
    is 2^0.5, one block whose exponent is floor(log2 2^0.5) - 8 = -8 (both
    rules: the significand 1.414 is below 1.75): code 362.04 -> 352 (quantum
    32), P^ = 1.375, O = (V_0 + 1.375 V_1) / (1 + 2^0.5). With tau = 0 every
    code is exact and O is the softmax's. V's columns are exact in MX (blocks
    of 32 keys: amax 2, 2, 2, 0.25)."""
    q = np.zeros((1, 1, 2, 32))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, 2, 32))
    k[0, 0, 1, 0] = 0.5
    v = np.zeros((1, 1, 2, 32))
    v[0, 0, 0, :4] = [2.0, -1.0, 0.5, 0.0]
    v[0, 0, 1, :4] = [1.0, 2.0, -2.0, 0.25]
    for rule in ("ocp", "fit"):
        o8, _ = mx.mxfp8_attention_forward(q, k, v, False, math.log(2.0), None, tile=1, rule=rule, tau=8.0)
        want = (v[0, 0, 0] + 1.375 * v[0, 0, 1]) / (1 + 2 ** 0.5)
        np.testing.assert_allclose(o8[0, 0, 0], want, rtol=1e-7, atol=1e-12)   # P and l in float32
        o0, _ = mx.mxfp8_attention_forward(q, k, v, False, math.log(2.0), None, tile=1, rule=rule, tau=0.0)
        exact = (2 ** -0.5 * v[0, 0, 0] + v[0, 0, 1]) / (1 + 2 ** -0.5)
        np.testing.assert_allclose(o0[0, 0, 0], exact, rtol=1e-7, atol=1e-12)


def test_mxfp8_deferred_max_keeps_accuracy_and_lse():
    """tau = 8 rounds different multiples of the same P; the LSE does not
    depend on when m is raised (up to P's float32 rounding), and the accuracy
    against exact attention stays within 10 %."""
    rng = np.random.default_rng(41)
    q, k, v = (rng.standard_normal((1, 2, 384, 64)) for _ in range(3))
    exact, _ = oracle.attention_forward(q, k, v, True, 0.125)
    o0, l0 = mx.mxfp8_attention_forward(q, k, v, True, 0.125, rule="fit", tau=0.0)
    o8, l8 = mx.mxfp8_attention_forward(q, k, v, True, 0.125, rule="fit", tau=8.0)
    rms = lambda a: math.sqrt(np.mean(a ** 2))
    # the same except for P's float32 rounding at a different scale
    np.testing.assert_allclose(l0, l8, rtol=0, atol=1e-6)
    assert abs(rms(o0 - exact) - rms(o8 - exact)) <= 0.1 * rms(o0 - exact)
    assert rms(o0 - o8) < 0.5 * rms(o0 - exact)
