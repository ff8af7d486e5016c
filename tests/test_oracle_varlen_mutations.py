"""The varlen oracle's pins catch plausible mistakes: each case plants one
error in a copy of oracle/varlen.py (never in the oracle itself), swaps the
copy's functions into the ``oracle`` package, and expects a named pin to
fail."""

import importlib.util
import os
import sys

import pytest

import oracle
import oracle.varlen as vmod

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
import test_oracle_varlen_pins as pins  # noqa: E402

SRC = open(vmod.__file__).read()

MUTATIONS = [
    ("keys of the whole batch", "qh, kh, vh = q[s0:s1, h], k[s0:s1, h // g], v[s0:s1, h // g]",
     "qh, kh, vh = q[s0:s1, h], k[:, h // g], v[:, h // g]",
     [lambda: pins.test_each_sequence_equals_the_fixed_length_oracle(False),
      pins.test_other_sequences_do_not_move_the_result]),
    ("causal mask off by one", "                s[np.triu_indices(n, 1)] = -np.inf\n            m = s.max",
     "                s[np.triu_indices(n, 0)] = -1e9\n            m = s.max",
     [lambda: pins.test_uniform_scores_average_within_the_sequence_only(True)]),
    ("dK overwritten, not summed over the group", "dk[s0:s1, kv] += scale * (ds.T @ qh)",
     "dk[s0:s1, kv] = scale * (ds.T @ qh)",
     [lambda: pins.test_each_sequence_equals_the_fixed_length_oracle(True)]),
    ("D from dO alone instead of dO * O", "ds = p * (dp - np.sum(do * o, axis=1, keepdims=True))",
     "ds = p * (dp - np.sum(do * do, axis=1, keepdims=True))",
     [pins.test_varlen_backward_finite_differences]),
    ("LSE of the wrong rows", "lse[h, s0:s1] = (m + np.log(l))[:, 0]", "lse[h, s0:s1] = m[:, 0]",
     [lambda: pins.test_uniform_scores_average_within_the_sequence_only(False)]),
    ("dQ without the scale", "dq[s0:s1, h] = scale * (ds @ kh)", "dq[s0:s1, h] = ds @ kh",
     [pins.test_varlen_backward_finite_differences]),
    ("decreasing offsets accepted", "np.any(np.diff(cu) < 0)", "False", [pins.test_bad_offsets_are_rejected]),
    ("backward GQA head map", "            kv = h // g\n            qh, kh, vh, do", "            kv = h % Hkv\n            qh, kh, vh, do",
     [lambda: pins.test_each_sequence_equals_the_fixed_length_oracle(True)]),
    ("an empty sequence ends the batch", "        if n == 0:\n            continue\n        for h in range(Hq):\n            qh, kh",
     "        if n == 0:\n            break\n        for h in range(Hq):\n            qh, kh",
     [pins.test_other_sequences_do_not_move_the_result]),
]


def _mutated_module(old, new):
    assert SRC.count(old) == 1, old
    spec = importlib.util.spec_from_loader("varlen_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(SRC.replace(old, new), "varlen_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, old, new, catchers):
    mod = _mutated_module(old, new)
    for fn in ("varlen_forward", "varlen_backward"):
        monkeypatch.setattr(oracle, fn, getattr(mod, fn))
    caught = 0
    for pin in catchers:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake: {name}"
