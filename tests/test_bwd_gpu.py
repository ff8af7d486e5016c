"""Backward parity: dQ, dK, dV from the CUDA path (through the C ABI, fed
with the CUDA forward's O and LSE) against the fp64 oracle's analytic
gradients on the same seeded inputs. Tolerance: relative L2 error <= 1e-2 for
each of dQ, dK, dV."""

import numpy as np
import pytest
import torch

import oracle
from synthetic import WORKLOADS

from _helpers import GRAD_REL_L2, make_inputs, rel_l2, to_f64

pytestmark = pytest.mark.gpu


def run_bwd(dev, causal, scale=None, workspace_fill=None):
    import exact_tiled_attention_42_b200 as fa
    o, lse = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal, scale=scale)
    ws = None
    if workspace_fill is not None:
        B, Hq, N, d = dev["q"].shape
        n = fa.fa_bwd_workspace_size(B, Hq, dev["k"].shape[1], N, d)
        ws = torch.full((n // 4,), workspace_fill, dtype=torch.float32, device="cuda")
    dq, dk, dv = fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal=causal, scale=scale,
                           workspace=ws)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return to_f64(dq), to_f64(dk), to_f64(dv)


def check(got, ref, what=""):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.all(np.isfinite(g)), f"{what} {name} has non-finite values"
        e = rel_l2(g, r)
        assert e <= GRAD_REL_L2, f"{what} {name} relative L2 error {e}"


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_workload(causal):
    w = WORKLOADS["tiny"]
    dev, host = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed)
    got = run_bwd(dev, causal)
    ref = oracle.attention_backward(host["q"], host["k"], host["v"], host["do"], causal, w.scale)
    check(got, ref, "tiny")


@pytest.mark.parametrize("N", [1, 17, 127, 128, 129, 255, 257, 383, 1000])
@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_edge_sizes(N, d, causal):
    dev, host = make_inputs(1, 2, 2, N, d, seed=2000 + N + d)
    got = run_bwd(dev, causal)
    ref = oracle.attention_backward(host["q"], host["k"], host["v"], host["do"], causal, d ** -0.5)
    check(got, ref, f"N={N} d={d}")


@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (8, 2), (3, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_small(Hq, Hkv, causal):
    dev, host = make_inputs(2, Hq, Hkv, 300, 128, seed=177 + Hq)
    got = run_bwd(dev, causal)
    ref = oracle.attention_backward(host["q"], host["k"], host["v"], host["do"], causal, 128 ** -0.5)
    check(got, ref, "gqa")


def test_workspace_contents_do_not_matter():
    dev, _ = make_inputs(1, 4, 2, 333, 64, seed=8)
    a = run_bwd(dev, True, workspace_fill=0.0)
    b = run_bwd(dev, True, workspace_fill=float("nan"))
    c = run_bwd(dev, True, workspace_fill=1e30)
    for x, y, z in zip(a, b, c):
        np.testing.assert_array_equal(x, y)
        np.testing.assert_array_equal(x, z)


def test_large_scale_scores():
    dev, host = make_inputs(1, 2, 2, 384, 64, seed=15)
    for scale in (0.05, 1.0):
        got = run_bwd(dev, True, scale)
        ref = oracle.attention_backward(host["q"], host["k"], host["v"], host["do"], True, scale)
        check(got, ref, f"scale={scale}")


@pytest.mark.parametrize("name", ["gpt2", "long128", "gqa"])
def test_full_size_workloads_sampled(name):
    """Full-size launch; the gradients of two KV groups (batch 0 group 0, and
    the last group of the last batch) are checked against the oracle run on
    exactly those heads."""
    w = WORKLOADS[name]
    dev, host = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed)
    g = w.Hq // w.Hkv
    for causal in w.causal:
        dq, dk, dv = run_bwd(dev, causal)
        for b, kv in ((0, 0), (w.B - 1, w.Hkv - 1)):
            hs = slice(kv * g, (kv + 1) * g)
            ref = oracle.attention_backward(host["q"][b:b + 1, hs], host["k"][b:b + 1, kv:kv + 1],
                                            host["v"][b:b + 1, kv:kv + 1], host["do"][b:b + 1, hs], causal, w.scale)
            got = (dq[b:b + 1, hs], dk[b:b + 1, kv:kv + 1], dv[b:b + 1, kv:kv + 1])
            check(got, ref, f"{name} causal={causal} b={b} kv={kv}")
