"""Pins for the fp64 oracle: closed forms, invariants, brute force and finite
differences, each chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them."""

import math

import numpy as np
import pytest

import oracle
from synthetic import attention_inputs, bf16_bits_to_f32


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# --- softmax rows -----------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    q, k = _rand((1, 2, 37, 16), 1), _rand((1, 2, 37, 16), 2)
    p = oracle.attention_probabilities(q, k, causal, 0.25)
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14, rtol=0)
    if causal:
        assert np.all(np.triu(p[0, 0], 1) == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_probabilities_times_v_is_the_forward_under_gqa(causal):
    """P from attention_probabilities, multiplied by the V head each query head
    reads (h // (Hq / Hkv)), is the forward's O."""
    q, k, v = _rand((1, 4, 29, 16), 41), _rand((1, 2, 29, 16), 42), _rand((1, 2, 29, 16), 43)
    p = oracle.attention_probabilities(q, k, causal, 0.25)
    o, _ = oracle.attention_forward(q, k, v, causal, 0.25)
    np.testing.assert_allclose(p @ np.repeat(v, 2, axis=1), o, atol=1e-13, rtol=0)


# --- closed forms -----------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores_give_mean_of_v(causal):
    """Q = 0 makes every score 0: O_i is the mean of V over the visible keys
    and LSE_i = log(number of visible keys)."""
    N, d = 33, 8
    q = np.zeros((1, 1, N, d))
    k = _rand((1, 1, N, d), 3)
    v = _rand((1, 1, N, d), 4)
    o, lse = oracle.attention_forward(q, k, v, causal, 0.5)
    vv = v[0, 0]
    if causal:
        expect = np.cumsum(vv, axis=0) / np.arange(1, N + 1)[:, None]
        expect_lse = np.log(np.arange(1, N + 1))
    else:
        expect = np.broadcast_to(vv.mean(0), (N, d))
        expect_lse = np.full(N, math.log(N))
    np.testing.assert_allclose(o[0, 0], expect, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], expect_lse, atol=1e-14)


def test_one_hot_scores_select_a_v_row():
    """K = identity rows, Q_i = alpha e_{pi(i)} with alpha*scale = 50: row i
    puts weight 1/(1 + (N-1) e^-50) on key pi(i), so O_i = V_{pi(i)} to within
    about N e^-50 and LSE_i = 50 + log(1 + (N-1) e^-50)."""
    N = d = 16
    scale = 0.125
    alpha = 50.0 / scale
    perm = np.random.default_rng(5).permutation(N)
    q = np.zeros((1, 1, N, d))
    q[0, 0, np.arange(N), perm] = alpha
    k = np.eye(N)[None, None]
    v = _rand((1, 1, N, d), 6)
    o, lse = oracle.attention_forward(q, k, v, False, scale)
    np.testing.assert_allclose(o[0, 0], v[0, 0, perm], atol=1e-18 + N * math.exp(-50) * np.abs(v).max())
    np.testing.assert_allclose(lse[0, 0], 50 + math.log1p((N - 1) * math.exp(-50)), rtol=1e-15)
    # causal: row i sees keys 0..i; the chosen key is visible iff perm[i] <= i
    oc, _ = oracle.attention_forward(q, k, v, True, scale)
    for i in range(N):
        if perm[i] <= i:
            np.testing.assert_allclose(oc[0, 0, i], v[0, 0, perm[i]], atol=1e-18 + N * math.exp(-50) * np.abs(v).max())
        else:  # all visible scores are 0: mean of the visible V rows
            np.testing.assert_allclose(oc[0, 0, i], v[0, 0, :i + 1].mean(0), atol=1e-13)


def test_causal_first_row_is_v0():
    q, k, v = _rand((2, 3, 20, 8), 7), _rand((2, 3, 20, 8), 8), _rand((2, 3, 20, 8), 9)
    scale = 0.3
    o, lse = oracle.attention_forward(q, k, v, True, scale)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-15)
    s00 = scale * np.sum(q[:, :, 0] * k[:, :, 0], axis=-1)
    np.testing.assert_allclose(lse[:, :, 0], s00, atol=1e-14)


def test_lse_identity_without_max_shift():
    q, k, v = _rand((1, 2, 24, 8), 10, 0.3), _rand((1, 2, 24, 8), 11, 0.3), _rand((1, 2, 24, 8), 12)
    scale = 0.5
    for causal in (False, True):
        _, lse = oracle.attention_forward(q, k, v, causal, scale)
        for h in range(2):
            for i in range(24):
                js = range(i + 1) if causal else range(24)
                direct = math.log(sum(math.exp(scale * float(q[0, h, i] @ k[0, h, j])) for j in js))
                assert abs(lse[0, h, i] - direct) < 1e-13


def test_two_key_closed_form():
    """N = 2, d = 1: P row 0 = softmax(scale*[q0 k0, q0 k1]) written out."""
    q = np.array([2.0, -1.0]).reshape(1, 1, 2, 1)
    k = np.array([0.5, 1.5]).reshape(1, 1, 2, 1)
    v = np.array([3.0, -2.0]).reshape(1, 1, 2, 1)
    scale = 0.7
    o, lse = oracle.attention_forward(q, k, v, False, scale)
    for i, qi in enumerate([2.0, -1.0]):
        a, b = math.exp(scale * qi * 0.5), math.exp(scale * qi * 1.5)
        assert abs(o[0, 0, i, 0] - (3.0 * a - 2.0 * b) / (a + b)) < 1e-15
        assert abs(lse[0, 0, i] - math.log(a + b)) < 1e-15


# --- brute force: scalar loops vs numpy ---------------------------------------

def _tiny_inputs():
    x = attention_inputs(1, 2, 2, 128, 64, seed=42)
    return {n: bf16_bits_to_f32(a).astype(np.float64) for n, a in x.items()}


@pytest.mark.parametrize("causal", [False, True])
def test_loops_match_numpy_forward(causal):
    x = _tiny_inputs()
    o1, l1 = oracle.attention_forward(x["q"], x["k"], x["v"], causal, 64 ** -0.5)
    o2, l2 = oracle.attention_forward_loops(x["q"], x["k"], x["v"], causal, 64 ** -0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_loops_match_numpy_backward(causal):
    x = attention_inputs(1, 4, 2, 24, 16, seed=3)
    x = {n: bf16_bits_to_f32(a).astype(np.float64) for n, a in x.items()}
    g1 = oracle.attention_backward(x["q"], x["k"], x["v"], x["do"], causal, 0.25)
    g2 = oracle.attention_backward_loops(x["q"], x["k"], x["v"], x["do"], causal, 0.25)
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(a, b, atol=1e-12)


# --- finite differences --------------------------------------------------------

@pytest.mark.parametrize("causal,Hq,Hkv", [(False, 2, 2), (True, 4, 2)])
def test_backward_matches_finite_differences(causal, Hq, Hkv):
    rng = np.random.default_rng(13)
    N, d, scale = 12, 8, 0.35
    q = rng.standard_normal((1, Hq, N, d))
    k = rng.standard_normal((1, Hkv, N, d))
    v = rng.standard_normal((1, Hkv, N, d))
    do = rng.standard_normal((1, Hq, N, d))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal, scale)

    def f(q_, k_, v_):
        o, _ = oracle.attention_forward(q_, k_, v_, causal, scale)
        return float(np.sum(do * o))

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(20):
            idx = tuple(rng.integers(0, s) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd = (f(args_p["q"], args_p["k"], args_p["v"]) - f(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(g[idx])), (name, idx, fd, g[idx])


# --- GQA ----------------------------------------------------------------------

def test_gqa_equals_repeated_heads():
    rng = np.random.default_rng(14)
    B, Hkv, grp, N, d = 2, 2, 3, 10, 8
    q = rng.standard_normal((B, Hkv * grp, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    do = rng.standard_normal((B, Hkv * grp, N, d))
    krep, vrep = np.repeat(k, grp, axis=1), np.repeat(v, grp, axis=1)
    for causal in (False, True):
        o1, l1 = oracle.attention_forward(q, k, v, causal, 0.4)
        o2, l2 = oracle.attention_forward(q, krep, vrep, causal, 0.4)
        np.testing.assert_allclose(o1, o2, atol=1e-15)
        np.testing.assert_allclose(l1, l2, atol=1e-15)
        dq1, dk1, dv1 = oracle.attention_backward(q, k, v, do, causal, 0.4)
        dq2, dk2, dv2 = oracle.attention_backward(q, krep, vrep, do, causal, 0.4)
        np.testing.assert_allclose(dq1, dq2, atol=1e-14)
        np.testing.assert_allclose(dk1, dk2.reshape(B, Hkv, grp, N, d).sum(2), atol=1e-13)
        np.testing.assert_allclose(dv1, dv2.reshape(B, Hkv, grp, N, d).sum(2), atol=1e-13)


def test_row_subset_matches_full_result():
    q, k, v, do = (_rand((1, 2, 50, 8), s) for s in (24, 25, 26, 27))
    full = oracle.attention_forward(q, k, v, True, 0.3)
    part = oracle.attention_forward(q, k, v, True, 0.3, row_chunk=4, rows=(13, 31))
    np.testing.assert_array_equal(part[0][:, :, 13:31], full[0][:, :, 13:31])
    assert np.isnan(part[0][:, :, :13]).all() and np.isnan(part[1][:, :, 31:]).all()
    g_full = oracle.attention_backward(q, k, v, do, True, 0.3)
    g_a = oracle.attention_backward(q, k, v, do, True, 0.3, rows=(0, 20))
    g_b = oracle.attention_backward(q, k, v, do, True, 0.3, rows=(20, 50))
    for x, a, b in zip(g_full, g_a, g_b):
        np.testing.assert_allclose(a + b, x, atol=1e-13)


def test_row_chunking_does_not_change_result():
    q, k, v, do = (_rand((1, 2, 50, 8), s) for s in (20, 21, 22, 23))
    a = oracle.attention_forward(q, k, v, True, 0.3, row_chunk=7)
    b = oracle.attention_forward(q, k, v, True, 0.3, row_chunk=1000)
    np.testing.assert_allclose(a[0], b[0], atol=1e-15)
    ga = oracle.attention_backward(q, k, v, do, True, 0.3, row_chunk=7)
    gb = oracle.attention_backward(q, k, v, do, True, 0.3, row_chunk=1000)
    for x, y in zip(ga, gb):
        np.testing.assert_allclose(x, y, atol=1e-13)


# --- the tiled recurrence -----------------------------------------------------------

@pytest.mark.parametrize("block", [16, 32, 128])
@pytest.mark.parametrize("tau", [0.0, 8.0])
@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_recurrence_is_exact(block, tau, causal):
    x = _tiny_inputs()
    o1, l1 = oracle.attention_forward(x["q"], x["k"], x["v"], causal, 64 ** -0.5)
    o2, l2 = oracle.online_softmax_forward(x["q"], x["k"], x["v"], causal, 64 ** -0.5, block, tau)
    np.testing.assert_allclose(o2, o1, atol=1e-13)
    np.testing.assert_allclose(l2, l1, atol=1e-13)


def test_online_softmax_large_scores_with_stale_max():
    """Scores spread over hundreds of log2 units: the stale-max recurrence must
    stay finite and exact."""
    q, k, v = _rand((1, 1, 64, 8), 30, 6.0), _rand((1, 1, 64, 8), 31, 6.0), _rand((1, 1, 64, 8), 32)
    o1, l1 = oracle.attention_forward(q, k, v, False, 1.0)
    o2, l2 = oracle.online_softmax_forward(q, k, v, False, 1.0, 8, 8.0)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=1e-13)


# --- fewer query rows than keys ------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_query_suffix_equals_rows_of_square_problem(causal):
    """Nq < Nk: the last Nq queries of a square problem, run alone against all
    Nk keys, give exactly those rows of the square result (the causal mask is
    aligned to the end of the key sequence)."""
    q, k, v = _rand((2, 4, 40, 8), 40), _rand((2, 2, 40, 8), 41), _rand((2, 2, 40, 8), 42)
    full_o, full_l = oracle.attention_forward(q, k, v, causal, 0.3)
    for nq in (1, 3, 17, 40):
        o, l = oracle.attention_forward(q[:, :, 40 - nq:], k, v, causal, 0.3)
        np.testing.assert_allclose(o, full_o[:, :, 40 - nq:], atol=1e-14)
        np.testing.assert_allclose(l, full_l[:, :, 40 - nq:], atol=1e-14)


def test_single_query_uniform_scores():
    """One query with Q = 0 against Nk keys: O is the mean of all V rows and
    LSE = log Nk, causal or not (the query is the last position)."""
    k, v = _rand((1, 1, 25, 8), 43), _rand((1, 1, 25, 8), 44)
    for causal in (False, True):
        o, l = oracle.attention_forward(np.zeros((1, 1, 1, 8)), k, v, causal, 0.7)
        np.testing.assert_allclose(o[0, 0, 0], v[0, 0].mean(0), atol=1e-14)
        assert abs(l[0, 0, 0] - math.log(25)) < 1e-14
