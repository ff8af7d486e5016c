"""Pins for the packed variable-length oracle (oracle/varlen.py): it agrees
with the fixed-length oracle on every sequence unpacked, with closed forms
that restart at sequence boundaries, with finite differences, and one
sequence's tokens never move another sequence's results."""

import numpy as np
import pytest

import oracle

LENS = [0, 1, 129, 7, 300, 128]


def _packed(lens, Hq, Hkv, d, seed):
    rng = np.random.default_rng(seed)
    T = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q = rng.standard_normal((T, Hq, d))
    k = rng.standard_normal((T, Hkv, d))
    v = rng.standard_normal((T, Hkv, d))
    do = rng.standard_normal((T, Hq, d))
    return cu, q, k, v, do


def _unpack(x, s0, s1):
    return np.ascontiguousarray(np.transpose(x[s0:s1], (1, 0, 2))[None])   # [1, H, n, d]


@pytest.mark.parametrize("causal", [False, True])
def test_each_sequence_equals_the_fixed_length_oracle(causal):
    cu, q, k, v, do = _packed(LENS, 4, 2, 16, seed=1)
    scale = 0.3
    o, lse = oracle.varlen_forward(q, k, v, cu, causal, scale)
    dq, dk, dv = oracle.varlen_backward(q, k, v, do, cu, causal, scale)
    for b in range(len(LENS)):
        s0, s1 = cu[b], cu[b + 1]
        if s1 == s0:
            continue
        args = [_unpack(x, s0, s1) for x in (q, k, v)]
        o_ref, lse_ref = oracle.attention_forward(*args, causal, scale)
        np.testing.assert_allclose(_unpack(o, s0, s1), o_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[:, s0:s1], lse_ref[0], rtol=1e-12, atol=1e-12)
        grads = oracle.attention_backward(*args, _unpack(do, s0, s1), causal, scale)
        for got, ref in zip((dq, dk, dv), grads):
            np.testing.assert_allclose(_unpack(got, s0, s1), ref, rtol=1e-10, atol=1e-12)


def test_equal_lengths_pack_to_the_batched_layout():
    """B sequences of one length packed token-major are the [B, H, N, d]
    problem with the axes moved."""
    B, H, N, d = 3, 2, 50, 8
    rng = np.random.default_rng(2)
    q, k, v = (rng.standard_normal((B, H, N, d)) for _ in range(3))
    pack = lambda x: np.transpose(x, (0, 2, 1, 3)).reshape(B * N, H, d)
    cu = np.arange(B + 1) * N
    o, lse = oracle.varlen_forward(pack(q), pack(k), pack(v), cu, True, 0.25)
    o_ref, lse_ref = oracle.attention_forward(q, k, v, True, 0.25)
    np.testing.assert_allclose(o, pack(o_ref), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, np.transpose(lse_ref, (1, 0, 2)).reshape(H, B * N), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores_average_within_the_sequence_only(causal):
    """Q = 0: every visible key scores 0, so O_i is the mean of V over the
    keys row i sees (its own sequence's first i+1 tokens when causal, all of
    its sequence otherwise) and LSE_i = log(#keys): both restart at every
    boundary."""
    cu, q, k, v, _ = _packed(LENS, 2, 1, 8, seed=3)
    o, lse = oracle.varlen_forward(np.zeros_like(q), k, v, cu, causal, 1.0)
    for b in range(len(LENS)):
        s0, s1 = cu[b], cu[b + 1]
        for i in range(s0, s1):
            hi = i + 1 if causal else s1
            np.testing.assert_allclose(o[i], np.broadcast_to(v[s0:hi, 0].mean(axis=0), (2, 8)), rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse[:, i], np.log(hi - s0), rtol=0, atol=1e-12)


def test_other_sequences_do_not_move_the_result():
    cu, q, k, v, do = _packed(LENS, 2, 2, 8, seed=4)
    o1, l1 = oracle.varlen_forward(q, k, v, cu, True, 0.5)
    g1 = oracle.varlen_backward(q, k, v, do, cu, True, 0.5)
    s0, s1 = cu[4], cu[5]             # change every input of sequence 4 only
    for x in (q, k, v, do):
        x[s0:s1] += 3.0
    o2, l2 = oracle.varlen_forward(q, k, v, cu, True, 0.5)
    g2 = oracle.varlen_backward(q, k, v, do, cu, True, 0.5)
    keep = np.r_[0:s0, s1:cu[-1]]
    np.testing.assert_array_equal(o1[keep], o2[keep])
    np.testing.assert_array_equal(l1[:, keep], l2[:, keep])
    for a, b in zip(g1, g2):
        np.testing.assert_array_equal(a[keep], b[keep])
    assert np.max(np.abs(o1[s0:s1] - o2[s0:s1])) > 0.1


def test_varlen_backward_finite_differences():
    """Central differences of f = sum(dO * O) at a few entries of Q, K, V."""
    cu, q, k, v, do = _packed([3, 5, 4], 2, 1, 4, seed=5)
    scale = 0.7
    f = lambda q_, k_, v_: np.sum(do * oracle.varlen_forward(q_, k_, v_, cu, True, scale)[0])
    dq, dk, dv = oracle.varlen_backward(q, k, v, do, cu, True, scale)
    rng = np.random.default_rng(6)
    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for _ in range(8):
            args = [q.copy(), k.copy(), v.copy()]
            idx = tuple(rng.integers(0, s) for s in args[which].shape)
            args[which][idx] += h
            fp = f(*args)
            args[which][idx] -= 2 * h
            fm = f(*args)
            fd = (fp - fm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


def test_bad_offsets_are_rejected():
    cu, q, k, v, _ = _packed([2, 3], 1, 1, 4, seed=7)
    for bad in ([1, 2, 5], [0, 3, 2, 5], [0, 2, 4]):
        with pytest.raises(ValueError, match="cu_seqlens"):   # rejected by the check, not by a later failure
            oracle.varlen_forward(q, k, v, bad, False, 1.0)
