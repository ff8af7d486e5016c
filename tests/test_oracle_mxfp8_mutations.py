"""The MXFP8 pins catch plausible mistakes: each case plants one error in a
copy of oracle/mxfp8.py (never in the oracle itself), swaps the copy's
functions in, and expects at least one named pin to fail."""

import importlib.util
import os
import sys

import pytest

import oracle.mxfp8 as mxmod

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import test_oracle_mxfp8_pins as pins  # noqa: E402

SRC = open(mxmod.__file__).read().replace("from .fp8 import", "from oracle.fp8 import")

MUTATIONS = [
    ("max raised on every increase despite tau", "m_new = np.where(tmax > m + tau, np.maximum(m, tmax), m)",
     "m_new = np.maximum(m, tmax)", [pins.test_mxfp8_deferred_max_two_tile_closed_form]),
    ("shared exponent off by one", "e = E - 1 - E4M3_EMAX", "e = E - E4M3_EMAX",
     [pins.test_closed_form_blocks]),
    ("fit rule at the boundary", "e = e + (m > 0.875)", "e = e + (m >= 0.875)",
     [pins.test_fit_rule_differs_only_above_significand_1_75]),
    ("V blocked along d", "vh = mx_roundtrip(v.astype(np.float32), axis=-2, rule=rule)",
     "vh = mx_roundtrip(v.astype(np.float32), axis=-1, rule=rule)",
     [pins.test_v_is_blocked_along_the_keys]),
    ("recurrence without rescale", "acc = acc * alpha[:, None] + pq @ vh[b, kvh, j0:j1]",
     "acc = acc + pq @ vh[b, kvh, j0:j1]",
     [lambda: pins.test_exact_when_operands_representable_and_p_unquantised(False)]),
    ("rotation's 1/d not folded", "sfac = scale / d", "sfac = scale",
     [lambda: pins.test_accuracy_on_the_fp8_input_recipe(21)]),
    ("K blocked along the keys", "kh = mx_roundtrip(k.astype(np.float32), axis=-1, rule=rule)",
     "kh = mx_roundtrip(k.astype(np.float32), axis=-2, rule=rule)",
     [pins.test_k_is_blocked_along_d]),
    ("Q blocked along the query rows", "qh = mx_roundtrip(q.astype(np.float32), axis=-1, rule=rule)",
     "qh = mx_roundtrip(q.astype(np.float32), axis=-2, rule=rule)",
     [pins.test_q_is_blocked_along_d]),
    ("P blocked along the query rows", "pq = mx_roundtrip(p, axis=-1, rule=rule)",
     "pq = mx_roundtrip(p, axis=0, rule=rule)", [pins.test_each_query_row_depends_only_on_its_own_q]),
    ("exponent not clamped to E8M0", "e = np.clip(e, E8M0_MIN, E8M0_MAX).astype(np.int64)", "e = e.astype(np.int64)",
     [pins.test_exponent_clamped_to_the_e8m0_range]),
    ("GQA head map", "kvh = h // g", "kvh = h % Hkv", [pins.test_gqa_equals_repeated_kv_heads]),
    ("row sum of the quantised P",
     "                l = l * alpha + p.sum(axis=1)\n                pq = mx_roundtrip(p, axis=-1, rule=rule) if quantize_p else p\n",
     "                pq = mx_roundtrip(p, axis=-1, rule=rule) if quantize_p else p\n                l = l * alpha + pq.sum(axis=1)\n",
     [pins.test_mxfp8_deferred_max_two_tile_closed_form]),
    ("causal mask off by one", "s = np.where(np.arange(j0, j1)[None, :] > rows[:, None], -np.inf, s)",
     "s = np.where(np.arange(j0, j1)[None, :] >= rows[:, None], -np.inf, s)",
     [lambda: pins.test_exact_when_operands_representable_and_p_unquantised(True)]),
    ("LSE left in log2", "lse[b, h] = (m + np.log2(l)) * math.log(2.0)", "lse[b, h] = (m + np.log2(l))",
     [lambda: pins.test_exact_when_operands_representable_and_p_unquantised(False)]),
    ("zero block given the exponent of its zero amax", "e = np.where(amax > 0, e, E8M0_MIN)", "e = e",
     [pins.test_zero_block_and_ragged_tail]),
    ("V rotated with Q and K", "    qh = mx_roundtrip(q.astype(np.float32), axis=-1, rule=rule)",
     "    v = rotate_rows(v, sigma) / d if sigma is not None else v\n"
     "    qh = mx_roundtrip(q.astype(np.float32), axis=-1, rule=rule)",
     [lambda: pins.test_accuracy_on_the_fp8_input_recipe(21)]),
]


def _mutated_module(old, new):
    assert SRC.count(old) >= 1, old
    spec = importlib.util.spec_from_loader("mxfp8_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(SRC.replace(old, new), "mxfp8_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, old, new, catchers):
    mod = _mutated_module(old, new)
    for fn in ("mx_quantize", "mx_dequantize", "mx_roundtrip", "mxfp8_attention_forward"):
        monkeypatch.setattr(mxmod, fn, getattr(mod, fn))
    caught = 0
    for pin in catchers:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake: {name}"
