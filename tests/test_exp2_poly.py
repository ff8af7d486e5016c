"""The FMA-pipe exp2 used for part of the FP8 softmax's exponentials: its
coefficients reproduce from the committed fit, and a step-by-step float32
emulation of the device function (same range reduction and Horner steps; an
fp32 FMA is emulated as the exact product-sum rounded once) stays within the
fitted error bound of the exact 2^x over the range the kernels use."""

import os
import re

import numpy as np

from exact_tiled_attention_42_b200 import fit_exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def device_coefficients():
    text = open(os.path.join(ROOT, "exact_tiled_attention_42_b200", "csrc", "common.cuh")).read()
    body = text[text.index("float exp2_poly"):]
    vals = re.search(r"C0 = ([^,]+)f, C1 = ([^,]+)f, C2 = ([^,]+)f, C3 = ([^;]+)f;", body).groups()
    return [np.float32(float.fromhex(v)) for v in vals]


def fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def emulate(x):
    c0, c1, c2, c3 = device_coefficients()
    shift = np.float32(12582912.0)
    x = np.maximum(np.float32(x), np.float32(-126.0))
    t = np.float32(x + shift)
    f = np.float32(x - np.float32(t - shift))
    p = fma32(fma32(fma32(c3, f, c2), f, c1), f, c0)
    j = (t.view(np.int32).astype(np.int64) - shift.view(np.int32).astype(np.int64)).astype(np.int64)
    bits = (p.view(np.uint32).astype(np.int64) + (j << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_match_the_fit():
    fitted = fit_exp2_poly.fit()
    np.testing.assert_array_equal(np.array(device_coefficients(), np.float32), fitted)
    assert fitted[0] == 1.0
    assert fit_exp2_poly.max_rel_error(fitted) < 1.5e-4


def test_emulated_device_function_error():
    # results below 2^-125 land in the subnormal range, where the exponent-bit
    # addition loses the implicit bit; those values are far below any P that
    # matters (the row maximum contributes at least 2^-8)
    x = np.concatenate([np.linspace(-125, 8, 400001), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 8) + 0.5]).astype(np.float32)
    y = np.array([emulate(v) for v in x[::7]] + [emulate(v) for v in x[-300:]], np.float64)
    xs = np.concatenate([x[::7], x[-300:]]).astype(np.float64)
    rel = np.abs(y - np.exp2(xs)) / np.exp2(xs)
    assert rel.max() < 1.5e-4, rel.max()


def test_masked_scores_vanish():
    for x in (-np.inf, -1e30, -127.0, -200.0):
        y = float(emulate(np.float32(x)))
        assert 0.0 <= y <= 2.0 ** -125
    assert float(emulate(np.float32(0.0))) == 1.0   # a row's largest score: P = 1 exactly
    for j in range(-20, 8):
        assert float(emulate(np.float32(j))) == 2.0 ** j
