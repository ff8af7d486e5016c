"""fp64 exact attention over packed variable-length batches.

TEST INFRASTRUCTURE ONLY: see the package docstring for who may import this.

The blog page ("FlashAttention: The Algorithm That Made Long-Context AI
Possible", section "Version 2 in 2023 and version 3 in 2024") notes that the
method was taken up widely by training and serving stacks; batches there pack
sequences of different lengths end to end. The pages give no interface for
this, so the reading here is the plain one: every sequence is its own
attention problem, exactly as if it were run alone.

Layout (packed, token-major): Q, O, dO are [T, Hq, d], K, V are [T, Hkv, d],
with T = cu_seqlens[-1] tokens; sequence b owns tokens
cu_seqlens[b] .. cu_seqlens[b+1]-1 (a sequence may be empty). LSE is
[Hq, T]. Within a sequence the causal mask keeps key j for query i iff
j <= i (positions local to the sequence); nothing crosses a sequence
boundary. Query head h reads KV head h // (Hq // Hkv).

This module restates the definition directly, per sequence and head, with its
own score/softmax/gradient lines; the pins compare it against the fixed-length
oracle on sequences unpacked into [1, H, n, d], against closed forms that
would cross a boundary if the packing leaked, and against independence under
changes to other sequences.
"""

from __future__ import annotations

import numpy as np


def _check(q, k, cu_seqlens):
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    cu = np.asarray(cu_seqlens, np.int64)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    if cu.ndim != 1 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, end at T and not decrease")
    return cu, Hq, Hkv, d


def varlen_forward(q, k, v, cu_seqlens, causal: bool, scale: float):
    """O [T, Hq, d] and LSE [Hq, T] of every packed sequence on its own."""
    cu, Hq, Hkv, d = _check(q, k, cu_seqlens)
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    g = Hq // Hkv
    T = q.shape[0]
    o = np.zeros((T, Hq, d))
    lse = np.zeros((Hq, T))
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        n = s1 - s0
        if n == 0:
            continue
        for h in range(Hq):
            qh, kh, vh = q[s0:s1, h], k[s0:s1, h // g], v[s0:s1, h // g]
            s = scale * (qh @ kh.T)
            if causal:
                s[np.triu_indices(n, 1)] = -np.inf
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            o[s0:s1, h] = (e / l) @ vh
            lse[h, s0:s1] = (m + np.log(l))[:, 0]
    return o, lse


def varlen_backward(q, k, v, dout, cu_seqlens, causal: bool, scale: float):
    """dQ [T, Hq, d], dK and dV [T, Hkv, d] (dK, dV summed over the query
    heads sharing a KV head), each sequence on its own: dV = P^T dO,
    dP = dO V^T, D = rowsum(dO * O), dS = P * (dP - D), dQ = scale dS K,
    dK = scale dS^T Q."""
    cu, Hq, Hkv, d = _check(q, k, cu_seqlens)
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    dout = np.asarray(dout, np.float64)
    g = Hq // Hkv
    T = q.shape[0]
    dq = np.zeros((T, Hq, d))
    dk = np.zeros((T, Hkv, d))
    dv = np.zeros((T, Hkv, d))
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        n = s1 - s0
        if n == 0:
            continue
        for h in range(Hq):
            kv = h // g
            qh, kh, vh, do = q[s0:s1, h], k[s0:s1, kv], v[s0:s1, kv], dout[s0:s1, h]
            s = scale * (qh @ kh.T)
            if causal:
                s[np.triu_indices(n, 1)] = -np.inf
            e = np.exp(s - s.max(axis=1, keepdims=True))
            p = e / e.sum(axis=1, keepdims=True)
            o = p @ vh
            dv[s0:s1, kv] += p.T @ do
            dp = do @ vh.T
            ds = p * (dp - np.sum(do * o, axis=1, keepdims=True))
            dq[s0:s1, h] = scale * (ds @ kh)
            dk[s0:s1, kv] += scale * (ds.T @ qh)
    return dq, dk, dv
