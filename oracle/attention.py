"""Plain fp64 exact softmax attention (forward, log-sum-exp, backward).

TEST INFRASTRUCTURE ONLY: see the package docstring for who may import this.

What it follows:
* "FlashAttention: The Algorithm That Made Long-Context AI Possible"
  (promptingindex.com), section "The quadratic bottleneck in standard
  attention": the score matrix S = Q K^T and the output O = softmax(S) V.
  This module writes that definition out directly, with the full N x N score
  matrix, which is exactly the computation the tiled method avoids
  materialising.
* Same page, section "What tiling changes": the tiled method keeps a running
  maximum and a running sum of exponentials and arrives at the same result.
  ``online_softmax_forward`` restates that recurrence separately, so a test can
  check that it reaches the one-shot softmax.
* "FlashAttention-2: Faster Attention with Better Parallelism and Work
  Partitioning" (abstract): grouped-query attention, whose head mapping the
  pages do not give. Reading used here: query head h reads KV head
  h // (Hq // Hkv), so consecutive query heads share a KV head.

Readings where the pages are silent (the method's definition is fixed by the
workload statement, not by the pages): scale multiplies Q K^T; the causal mask
keeps key j for query i iff j <= i; LSE is the natural log of the row's sum of
exp(scale * S); the backward is the analytic gradient of O with respect to Q,
K and V (dK and dV summed over the query heads sharing a KV head). For fewer
query rows than keys (Nq < Nk, decoding against a cache) the forward treats
the queries as the last Nq positions: query i keeps keys j <= i + Nk - Nq.

Inputs are float arrays [B, H, N, d] (Q and dO with Hq heads, K and V with Hkv
heads); every computation runs in float64.
"""

from __future__ import annotations

import math

import numpy as np


def _heads(q, k):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return B, Hq, Hkv, N, d, Hq // Hkv


def _scores(qh, kh, scale, causal, row0, row1):
    """Rows row0..row1-1 of S = scale * Q K^T, with -inf where the causal mask
    removes a key. With Nq query rows and Nk >= Nq keys, query i sits at key
    position i + Nk - Nq (the queries are the last Nq positions of the
    sequence, as when decoding against a cache); with Nq = Nk this is j <= i."""
    s = scale * (qh[row0:row1] @ kh.T)
    if causal:
        i = np.arange(row0, row1)[:, None] + (kh.shape[0] - qh.shape[0])
        j = np.arange(kh.shape[0])[None, :]
        s = np.where(j > i, -np.inf, s)
    return s


def _softmax_rows(s):
    """Explicit row softmax of a score block plus the natural-log LSE."""
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def attention_probabilities(q, k, causal: bool, scale: float) -> np.ndarray:
    """The full softmax matrix P [B, Hq, N, N] (small inputs only)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    B, Hq, Hkv, N, d, g = _heads(q, k)
    p = np.empty((B, Hq, N, N))
    for b in range(B):
        for h in range(Hq):
            p[b, h], _ = _softmax_rows(_scores(q[b, h], k[b, h // g], scale, causal, 0, N))
    return p


def attention_forward(q, k, v, causal: bool, scale: float, row_chunk: int = 2048, rows=None):
    """O = softmax(scale * Q K^T [+ causal mask]) V and LSE, in float64.

    Rows of S are formed ``row_chunk`` at a time so that large N fits in host
    memory; every row still sees its full set of scores, so this is the plain
    definition, not a tiling of the key dimension. ``rows = (r0, r1)`` limits
    the work to query rows r0..r1-1 (other rows of the result are left as
    NaN); it changes which rows are computed, not how.
    Returns (O [B,Hq,N,d], LSE [B,Hq,N]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, Hkv, N, d, g = _heads(q, k)
    lo, hi = (0, N) if rows is None else rows
    o = np.full((B, Hq, N, d), np.nan)
    lse = np.full((B, Hq, N), np.nan)
    for b in range(B):
        for h in range(Hq):
            kh, vh = k[b, h // g], v[b, h // g]
            for r0 in range(lo, hi, row_chunk):
                r1 = min(hi, r0 + row_chunk)
                p, lse[b, h, r0:r1] = _softmax_rows(_scores(q[b, h], kh, scale, causal, r0, r1))
                o[b, h, r0:r1] = p @ vh
    return o, lse


def attention_backward(q, k, v, dout, causal: bool, scale: float, row_chunk: int = 2048, rows=None):
    """Analytic gradients (dQ, dK, dV) of O = attention(Q, K, V) against dO.

    With P the softmax matrix:  dV = P^T dO;  dP = dO V^T;
    D_i = sum_t dO[i,t] O[i,t];  dS = P * (dP - D);  dQ = scale dS K;
    dK = scale dS^T Q.  dK and dV are summed over the query heads that share
    a KV head. P and O are recomputed here from the definition.
    ``rows = (r0, r1)`` keeps only the terms of query rows r0..r1-1 (their dQ
    rows and their share of dK and dV).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dout = np.asarray(dout, np.float64)
    B, Hq, Hkv, N, d, g = _heads(q, k)
    dq = np.zeros((B, Hq, N, d))
    dk = np.zeros((B, Hkv, N, d))
    dv = np.zeros((B, Hkv, N, d))
    lo, hi = (0, N) if rows is None else rows
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            kh, vh = k[b, kv], v[b, kv]
            for r0 in range(lo, hi, row_chunk):
                r1 = min(hi, r0 + row_chunk)
                p, _ = _softmax_rows(_scores(q[b, h], kh, scale, causal, r0, r1))
                do = dout[b, h, r0:r1]
                o = p @ vh
                dv[b, kv] += p.T @ do
                dp = do @ vh.T
                D = np.sum(do * o, axis=1, keepdims=True)
                ds = p * (dp - D)
                dq[b, h, r0:r1] = scale * (ds @ kh)
                dk[b, kv] += scale * (ds.T @ q[b, h, r0:r1])
    return dq, dk, dv


# ---------------------------------------------------------------------------
# Pure-Python loop versions (tiny inputs): the same definitions, one scalar at
# a time, with no library matmul, used to cross-check the numpy versions.
# ---------------------------------------------------------------------------

def _loop_head_forward(Q, K, V, causal, scale):
    N, d = len(Q), len(Q[0])
    O, L, P = [], [], []
    for i in range(N):
        s = []
        for j in range(N):
            if causal and j > i:
                s.append(-math.inf)
                continue
            acc = 0.0
            for t in range(d):
                acc += Q[i][t] * K[j][t]
            s.append(scale * acc)
        m = max(s)
        e = [math.exp(x - m) if x != -math.inf else 0.0 for x in s]
        z = sum(e)
        p = [x / z for x in e]
        row = [0.0] * d
        for j in range(N):
            if p[j] != 0.0:
                for t in range(d):
                    row[t] += p[j] * V[j][t]
        O.append(row)
        L.append(m + math.log(z))
        P.append(p)
    return O, L, P


def attention_forward_loops(q, k, v, causal: bool, scale: float):
    """Scalar-loop forward: returns (O, LSE) as float64 arrays."""
    q = np.asarray(q, np.float64)
    B, Hq, Hkv, N, d, g = _heads(q, np.asarray(k))
    o = np.empty((B, Hq, N, d))
    lse = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            O, L, _ = _loop_head_forward(q[b, h].tolist(), np.asarray(k, np.float64)[b, h // g].tolist(),
                                         np.asarray(v, np.float64)[b, h // g].tolist(), causal, scale)
            o[b, h] = O
            lse[b, h] = L
    return o, lse


def attention_backward_loops(q, k, v, dout, causal: bool, scale: float):
    """Scalar-loop backward: returns (dQ, dK, dV) as float64 arrays."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dout = np.asarray(dout, np.float64)
    B, Hq, Hkv, N, d, g = _heads(q, k)
    dq = np.zeros((B, Hq, N, d))
    dk = np.zeros((B, Hkv, N, d))
    dv = np.zeros((B, Hkv, N, d))
    for b in range(B):
        for h in range(Hq):
            kv = h // g
            Q, K, V, dO = q[b, h].tolist(), k[b, kv].tolist(), v[b, kv].tolist(), dout[b, h].tolist()
            O, _, P = _loop_head_forward(Q, K, V, causal, scale)
            for i in range(N):
                D = 0.0
                for t in range(d):
                    D += dO[i][t] * O[i][t]
                for j in range(N):
                    if P[i][j] == 0.0:
                        continue
                    dp = 0.0
                    for t in range(d):
                        dp += dO[i][t] * V[j][t]
                    ds = P[i][j] * (dp - D)
                    for t in range(d):
                        dv[b, kv, j, t] += P[i][j] * dO[i][t]
                        dq[b, h, i, t] += scale * ds * K[j][t]
                        dk[b, kv, j, t] += scale * ds * Q[i][t]
    return dq, dk, dv


# ---------------------------------------------------------------------------
# The tiled recurrence itself, in fp64.
# ---------------------------------------------------------------------------

def online_softmax_forward(q, k, v, causal: bool, scale: float, block: int, tau: float = 0.0):
    """Tile-by-tile forward with a running row max and running row sum.

    Follows "FlashAttention: The Algorithm That Made Long-Context AI Possible",
    section "What tiling changes": keys are visited ``block`` at a time; each
    row keeps a running maximum m and a running sum l of exponentials, and the
    partial output is rescaled whenever m moves. Scores are kept in base 2
    (c = scale * log2(e)). The maximum is only raised when the block's maximum
    exceeds it by more than ``tau`` (log2 units); a stale maximum is exact in
    real arithmetic because the same m is used for l and for O. ``tau = 0``
    raises it on any increase. Normalisation by l happens once, at the end.
    Returns (O, LSE).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, Hkv, N, d, g = _heads(q, k)
    c = scale * math.log2(math.e)
    o = np.empty((B, Hq, N, d))
    lse = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            kh, vh = k[b, h // g], v[b, h // g]
            m = np.full(N, -np.inf)
            l = np.zeros(N)
            acc = np.zeros((N, d))
            for j0 in range(0, N, block):
                j1 = min(N, j0 + block)
                s = c * (q[b, h] @ kh[j0:j1].T)
                if causal:
                    s = np.where(np.arange(j0, j1)[None, :] > np.arange(N)[:, None], -np.inf, s)
                bmax = np.max(s, axis=1)
                raise_m = (bmax > m + tau) | np.isneginf(m)
                m_new = np.where(raise_m, np.maximum(m, bmax), m)
                with np.errstate(invalid="ignore"):
                    alpha = np.where(np.isneginf(m), 0.0, np.exp2(m - m_new))
                m_safe = np.where(np.isneginf(m_new), 0.0, m_new)
                p = np.exp2(s - m_safe[:, None])
                l = l * alpha + p.sum(axis=1)
                acc = acc * alpha[:, None] + p @ vh[j0:j1]
                m = m_new
            o[b, h] = acc / l[:, None]
            lse[b, h] = (m + np.log2(l)) * math.log(2.0)
    return o, lse
