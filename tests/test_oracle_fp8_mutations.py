"""The FP8 oracle's pins catch plausible mistakes: each case plants one error
in a copy of oracle/fp8.py (never in the oracle itself), swaps the copy's
functions into the ``oracle`` package, and expects at least one named pin to
fail."""

import importlib.util
import os
import sys

import pytest

import oracle
import oracle.fp8 as fp8mod

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import test_oracle_fp8_pins as pins  # noqa: E402

SRC = open(fp8mod.__file__).read()

MUTATIONS = [
    ("ties away from zero", "r = np.round(ax / quantum) * quantum", "r = np.floor(ax / quantum + 0.5) * quantum",
     [pins.test_e4m3_ties_go_to_even_and_saturate, pins.test_e4m3_round_matches_torch_in_range]),
    ("no saturation", "r = np.minimum(r, E4M3_MAX)", "r = r",
     [pins.test_e4m3_ties_go_to_even_and_saturate]),
    ("block scale inverted", "scales[..., bi] = np.where(nz, safe / np.float32(E4M3_MAX)",
     "scales[..., bi] = np.where(nz, np.float32(E4M3_MAX) / safe", [pins.test_block_quantize_properties]),
    ("sign vector ignored", "return (x * sigma) @ hadamard(x.shape[-1])", "return x @ hadamard(x.shape[-1])",
     [pins.test_rotation_preserves_scores_up_to_d]),
    ("rotation's 1/d not folded", "sfac = scale / d", "sfac = scale",
     [lambda: pins.test_fp8_emulation_within_e4m3_error_of_exact(True)]),
    ("V's block scale not folded into P", "wkey = _expand_rows(vs[b, kvh], N, block_rows) / vref * p_lift",
     "wkey = np.full(N, p_lift)",
     [lambda: pins.test_fp8_emulation_within_e4m3_error_of_exact(False)]),
    ("O not rescaled when the max grows", "acc = acc * alpha[:, None] + pq @ vv[b, kvh, j0:j1].astype(np.float64)",
     "acc = acc + pq @ vv[b, kvh, j0:j1].astype(np.float64)",
     [lambda: pins.test_fp8_emulation_within_e4m3_error_of_exact(False)]),
    ("emulated P not rounded", "pq = e4m3_round((p * wkey[None, j0:j1]).astype(np.float32)).astype(np.float64)",
     "pq = p * wkey[None, j0:j1]",
     [lambda: pins.test_fp8_emulation_within_p_rounding_of_softmax_on_dequantised_operands(128, False, 0.8)]),
    ("emulated P rounded against a stale max", "p = np.exp2(s - m_new[:, None])", "p = np.exp2(s - np.maximum(m, -60.0)[:, None])",
     [lambda: pins.test_fp8_emulation_within_p_rounding_of_softmax_on_dequantised_operands(128, False, 0.8),
      lambda: pins.test_fp8_emulation_within_e4m3_error_of_exact(False)]),
    ("max raised on every increase despite tau", "m_new = np.where(tmax > m + tau, np.maximum(m, tmax), m)",
     "m_new = np.maximum(m, tmax)", [pins.test_fp8_deferred_max_two_tile_closed_form]),
    ("naive: P not rounded", "pq = e4m3_round(e.astype(np.float32)).astype(np.float64)", "pq = e",
     [pins.test_naive_fp8_two_key_closed_form_unnormalised,
      lambda: pins.test_naive_fp8_within_p_rounding_of_exact_on_grid("unnormalised")]),
    ("naive: normalised P not rounded", "pq = e4m3_round((e / l).astype(np.float32)).astype(np.float64)",
     "pq = e / l", [pins.test_naive_fp8_two_key_closed_form_normalised]),
    ("naive: per-head instead of per-tensor amax", "amax = np.max(np.abs(x32)).astype(np.float32)",
     "amax = np.max(np.abs(x32), axis=(-2, -1), keepdims=True).astype(np.float32)",
     [pins.test_naive_fp8_two_key_closed_form_unnormalised]),
    ("naive: V scale not applied", "o[b, h, r0:r1] = (pq @ vv[b, h // g]) * vs[b, h // g] / l",
     "o[b, h, r0:r1] = (pq @ vv[b, h // g]) / l", [pins.test_naive_fp8_two_key_closed_form_unnormalised]),
    ("naive: row sum of the rounded P", "o[b, h, r0:r1] = (pq @ vv[b, h // g]) * vs[b, h // g] / l",
     "o[b, h, r0:r1] = (pq @ vv[b, h // g]) * vs[b, h // g] / pq.sum(axis=1, keepdims=True)",
     [pins.test_naive_fp8_two_key_closed_form_unnormalised]),
    ("per-tensor scale inverted", "s = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float64)",
     "s = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float64)",
     [pins.test_per_tensor_quantize_closed_form]),
    ("emulation: GQA head map", "            kvh = h // g\n            vref", "            kvh = h % Hkv\n            vref",
     [lambda: pins.test_fp8_emulation_and_naive_gqa_equal_repeated_kv_heads(False)]),
    ("naive: GQA head map", "s = scale * (qh[b, h, r0:r1] @ kh[b, h // g].T)",
     "s = scale * (qh[b, h, r0:r1] @ kh[b, h % kh.shape[1]].T)",
     [lambda: pins.test_fp8_emulation_and_naive_gqa_equal_repeated_kv_heads(False)]),
    ("emulation: causal mask off by one",
     "s = np.where(np.arange(j0, j1)[None, :] > np.arange(N)[:, None], -np.inf, s)",
     "s = np.where(np.arange(j0, j1)[None, :] >= np.arange(N)[:, None], -np.inf, s)",
     [lambda: pins.test_fp8_emulation_within_p_rounding_of_softmax_on_dequantised_operands(128, True, 0.0)]),
    ("emulation: V's block weight not undone", "o[b, h] = acc * (vref / p_lift) / l[:, None]",
     "o[b, h] = acc / p_lift / l[:, None]", [pins.test_fp8_deferred_max_two_tile_closed_form]),
    ("e4m3 codes: exponent bias 8", "exp_field = np.where(normal, e + 7, 0)", "exp_field = np.where(normal, e + 8, 0)",
     [pins.test_e4m3_codes_match_torch_bit_patterns]),
    ("e4m3 rounding: no subnormal floor", "e = np.maximum(E - 1, _E4M3_MIN_NORMAL_EXP)", "e = E - 1",
     [pins.test_e4m3_round_matches_torch_in_range]),
]

SWAPPED = ("hadamard", "rotate_rows", "e4m3_round", "e4m3_encode", "e4m3_decode", "block_quantize",
           "per_tensor_quantize", "fp8_attention_forward", "naive_fp8_attention_forward")


def _mutated_module(old, new):
    assert SRC.count(old) == 1, old
    spec = importlib.util.spec_from_loader("fp8_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(SRC.replace(old, new), "fp8_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, old, new, catchers):
    mod = _mutated_module(old, new)
    for fn in SWAPPED:
        monkeypatch.setattr(oracle, fn, getattr(mod, fn))
    caught = 0
    for pin in catchers:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake: {name}"
