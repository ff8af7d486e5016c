"""The pins catch plausible mistakes: each case plants one error in a copy of
the oracle's source (never in the oracle itself), swaps the copy in, and
expects at least one of the named pin tests to fail."""

import importlib.util
import os
import sys

import pytest

import oracle
import oracle.attention as att

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import test_oracle_pins as pins  # noqa: E402

SRC = open(att.__file__).read()

MUTATIONS = [
    ("scale dropped", "s = scale * (qh[row0:row1] @ kh.T)", "s = (qh[row0:row1] @ kh.T)",
     [pins.test_two_key_closed_form, pins.test_lse_identity_without_max_shift]),
    ("causal mask flipped", "s = np.where(j > i, -np.inf, s)", "s = np.where(j < i, -np.inf, s)",
     [pins.test_causal_first_row_is_v0]),
    ("dS sign", "ds = p * (dp - D)", "ds = p * (D - dp)",
     [lambda: pins.test_backward_matches_finite_differences(False, 2, 2)]),
    ("dV untransposed", "dv[b, kv] += p.T @ do", "dv[b, kv] += p @ do",
     [lambda: pins.test_backward_matches_finite_differences(False, 2, 2)]),
    ("D term dropped", "ds = p * (dp - D)", "ds = p * dp",
     [lambda: pins.test_backward_matches_finite_differences(False, 2, 2)]),
    ("GQA head map", "kh, vh = k[b, h // g], v[b, h // g]", "kh, vh = k[b, h % Hkv], v[b, h % Hkv]",
     [pins.test_gqa_equals_repeated_heads]),
    ("recurrence without rescale", "acc = acc * alpha[:, None] + p @ vh[j0:j1]", "acc = acc + p @ vh[j0:j1]",
     [lambda: pins.test_online_softmax_recurrence_is_exact(32, 0.0, False)]),
    ("LSE without max", "return e / l, (m + np.log(l))[:, 0]", "return e / l, (np.log(l))[:, 0]",
     [pins.test_lse_identity_without_max_shift]),
    ("probabilities: GQA head map", "p[b, h], _ = _softmax_rows(_scores(q[b, h], k[b, h // g], scale, causal, 0, N))",
     "p[b, h], _ = _softmax_rows(_scores(q[b, h], k[b, h % Hkv], scale, causal, 0, N))",
     [lambda: pins.test_probabilities_times_v_is_the_forward_under_gqa(False)]),
    ("decode alignment dropped", "i = np.arange(row0, row1)[:, None] + (kh.shape[0] - qh.shape[0])",
     "i = np.arange(row0, row1)[:, None]", [lambda: pins.test_query_suffix_equals_rows_of_square_problem(True)]),
    ("dK overwritten, not summed over the group", "dk[b, kv] += scale * (ds.T @ q[b, h, r0:r1])",
     "dk[b, kv] = scale * (ds.T @ q[b, h, r0:r1])", [pins.test_gqa_equals_repeated_heads]),
    ("dQ from P instead of dS", "dq[b, h, r0:r1] = scale * (ds @ kh)", "dq[b, h, r0:r1] = scale * (p @ kh)",
     [lambda: pins.test_backward_matches_finite_differences(False, 2, 2)]),
    ("row subset end off by one", "lo, hi = (0, N) if rows is None else rows\n    o = np.full",
     "lo, hi = (0, N) if rows is None else (rows[0], rows[1] - 1)\n    o = np.full",
     [pins.test_row_subset_matches_full_result]),
]


def _mutated_module(old, new):
    assert SRC.count(old) >= 1, old
    spec = importlib.util.spec_from_loader("oracle_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(SRC.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, old, new, catchers):
    mod = _mutated_module(old, new)
    for fn in ("attention_forward", "attention_backward", "attention_probabilities", "online_softmax_forward"):
        monkeypatch.setattr(oracle, fn, getattr(mod, fn))
    caught = 0
    for pin in catchers:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake: {name}"


import oracle.fp8 as fp8  # noqa: E402
import test_oracle_fp8_pins as fpins  # noqa: E402

FSRC = open(fp8.__file__).read()

FP8_MUTATIONS = [
    ("round half up", "r = np.round(ax / quantum) * quantum", "r = np.floor(ax / quantum + 0.5) * quantum",
     [fpins.test_e4m3_round_matches_torch_in_range, fpins.test_e4m3_ties_go_to_even_and_saturate]),
    ("no saturation", "r = np.minimum(r, E4M3_MAX)", "r = r",
     [fpins.test_e4m3_ties_go_to_even_and_saturate]),
    ("scale off by 2", "inv = np.where(nz, np.float32(E4M3_MAX) / safe", "inv = np.where(nz, np.float32(224.0) / safe",
     [fpins.test_block_quantize_properties]),
    ("rotation without signs", "return (x * sigma) @ hadamard(x.shape[-1])", "return x @ hadamard(x.shape[-1])",
     [fpins.test_rotation_preserves_scores_up_to_d]),
]


@pytest.mark.parametrize("name,old,new,catchers", FP8_MUTATIONS, ids=[m[0] for m in FP8_MUTATIONS])
def test_fp8_pins_catch_planted_mistake(monkeypatch, name, old, new, catchers):
    assert FSRC.count(old) >= 1, old
    spec = importlib.util.spec_from_loader("fp8_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(FSRC.replace(old, new), "fp8_mutant", "exec"), mod.__dict__)
    for fn in ("e4m3_round", "block_quantize", "rotate_rows", "fp8_attention_forward", "naive_fp8_attention_forward"):
        monkeypatch.setattr(oracle, fn, getattr(mod, fn))
    caught = 0
    for pin in catchers:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake: {name}"
