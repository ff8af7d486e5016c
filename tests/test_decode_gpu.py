"""Decode-shaped forward (few query rows against a long key sequence, split
over the keys and merged by log-sum-exp) against the fp64 oracle on the same
seeded inputs: O max-abs <= 2e-2, LSE max-abs <= 1e-3."""

import numpy as np
import pytest
import torch

import oracle
from synthetic import WORKLOADS, attention_inputs, bf16_bits_to_f32

from _helpers import LSE_MAX_ABS, O_MAX_ABS, to_device_bf16, to_f64

pytestmark = pytest.mark.gpu


def inputs(B, Hq, Hkv, Nq, Nk, d, seed):
    kv = attention_inputs(B, Hkv, Hkv, Nk, d, seed, with_dout=False)
    qq = attention_inputs(B, Hq, Hq, Nq, d, seed + 1000, with_dout=False)
    dev = {"q": to_device_bf16(qq["q"]), "k": to_device_bf16(kv["k"]), "v": to_device_bf16(kv["v"])}
    host = {"q": bf16_bits_to_f32(qq["q"]).astype(np.float64), "k": bf16_bits_to_f32(kv["k"]).astype(np.float64),
            "v": bf16_bits_to_f32(kv["v"]).astype(np.float64)}
    return dev, host


def run(dev, causal, ctas=0, scale=None):
    import exact_tiled_attention_42_b200 as fa
    o, lse = fa.fa_fwd_decode(dev["q"], dev["k"], dev["v"], causal=causal, num_ctas=ctas, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return to_f64(o), lse.cpu().numpy().astype(np.float64)


def check(o, lse, o_ref, lse_ref):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(o - o_ref)) <= O_MAX_ABS, np.max(np.abs(o - o_ref))
    assert np.max(np.abs(lse - lse_ref)) <= LSE_MAX_ABS, np.max(np.abs(lse - lse_ref))


@pytest.mark.parametrize("Nk", [1, 63, 64, 65, 1000, 4097])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_single_query_gqa(Nk, d, causal):
    dev, host = inputs(2, 8, 2, 1, Nk, d, seed=300 + Nk + d)
    o, lse = run(dev, causal)
    o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], causal, d ** -0.5)
    check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("Hq,Hkv,Nq,Nk", [(4, 1, 4, 700), (2, 2, 8, 333), (16, 16, 1, 2000), (8, 1, 2, 129),
                                           (1, 1, 16, 16), (1, 1, 5, 5)])
@pytest.mark.parametrize("causal", [False, True])
def test_several_query_rows(Hq, Hkv, Nq, Nk, causal):
    dev, host = inputs(1, Hq, Hkv, Nq, Nk, 128, seed=400 + Nq + Nk)
    o, lse = run(dev, causal)
    o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], causal, 128 ** -0.5)
    check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("ctas", [1, 2, 3, 7, 64, 95, 10000])
def test_cta_count_does_not_change_the_result(ctas):
    """2 x 2 KV heads x 47 key tiles shared by 1 .. 94 CTAs (10000 is capped
    at one tile per CTA): ranges that end mid-head, cover a whole head, or
    span a head boundary."""
    dev, host = inputs(2, 8, 2, 2, 3000, 128, seed=501)
    o, lse = run(dev, True, ctas)
    o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], True, 128 ** -0.5)
    check(o, lse, o_ref, lse_ref)


def test_large_scale_scores():
    dev, host = inputs(1, 4, 1, 4, 1500, 64, seed=502)
    for scale in (0.05, 2.0):
        o, lse = run(dev, False, 0, scale)
        o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], False, scale)
        check(o, lse, o_ref, lse_ref)


def test_decode_workload_sampled():
    """The decode workload at full size (B=16, Hq=32, Hkv=8, one query row,
    16384 keys): two KV groups checked against the oracle."""
    w = WORKLOADS["decode"]
    dev, host = inputs(w.B, w.Hq, w.Hkv, w.nq, w.N, w.d, w.seed)
    o, lse = run(dev, True)
    g = w.Hq // w.Hkv
    for b, kv in ((0, 0), (w.B - 1, w.Hkv - 1)):
        hs = slice(kv * g, (kv + 1) * g)
        o_ref, lse_ref = oracle.attention_forward(host["q"][b:b + 1, hs], host["k"][b:b + 1, kv:kv + 1],
                                                  host["v"][b:b + 1, kv:kv + 1], True, w.scale)
        check(o[b:b + 1, hs], lse[b:b + 1, hs], o_ref, lse_ref)


def test_split_that_some_rows_cannot_see():
    """Nk = 129 as three 64-key tiles on three CTAs: with the causal mask
    aligned to the sequence end, query rows 0..14 see no key of the last tile
    (its partial log-sum-exp is -inf and must drop out of the merge)."""
    dev, host = inputs(1, 1, 1, 16, 129, 128, seed=503)
    o, lse = run(dev, True, 3)
    o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], True, 128 ** -0.5)
    check(o, lse, o_ref, lse_ref)
