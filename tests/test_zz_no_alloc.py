"""fa_bwd_noalloc: the backward for callers that cannot allocate device
memory at the call (it takes its scratch from a fixed array inside the
library). Called through the C ABI and checked against fa_bwd, the entry
point with a caller-provided workspace, on two calls in a row with different
inputs, so the second call starts from the scratch the first one left; on a
tiny case against the fp64 oracle directly; and at the exact size limit.
Collected last so that a stopping run has already run every other test."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from _helpers import GRAD_REL_L2, make_inputs, rel_l2, to_f64

pytestmark = pytest.mark.gpu

MAX_BYTES = 32 * 1024 * 1024   # FA_BWD_NOALLOC_MAX_BYTES


def _c_bwd_noalloc(lib, dev, o, lse, causal, scale):
    B, Hq, N, d = dev["q"].shape
    Hkv = dev["k"].shape[1]
    dq, dk, dv = torch.empty_like(dev["q"]), torch.empty_like(dev["k"]), torch.empty_like(dev["v"])
    st = lib.fa_bwd_noalloc(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(), o.data_ptr(),
                            lse.data_ptr(), dev["do"].data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                            B, Hq, Hkv, N, d, int(causal), float(scale),
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, st
    return dq, dk, dv


def test_noalloc_matches_workspace_entry_point_twice():
    import exact_tiled_attention_42_b200 as fa
    from exact_tiled_attention_42_b200 import _lib
    lib = _lib.load()
    cases = [(1, 4, 2, 777, 128, True, 31), (2, 2, 2, 300, 64, False, 32)]
    for B, Hq, Hkv, N, d, causal, seed in cases:
        dev, _ = make_inputs(B, Hq, Hkv, N, d, seed)
        scale = d ** -0.5
        o, lse = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal)
        ref = fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal=causal)
        got = _c_bwd_noalloc(lib, dev, o, lse, causal, scale)
        torch.cuda.synchronize()
        assert fa.fa_last_device_status() == 0
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            g, r = to_f64(g), to_f64(r)
            assert np.all(np.isfinite(g))
            assert rel_l2(g, r) <= GRAD_REL_L2, (name, rel_l2(g, r))


def test_noalloc_matches_the_oracle_on_a_tiny_case():
    """The tiny workload's shape (B=1, H=2, N=128, d=64), causal and not,
    against the fp64 oracle's gradients."""
    import exact_tiled_attention_42_b200 as fa
    from exact_tiled_attention_42_b200 import _lib
    lib = _lib.load()
    for causal in (False, True):
        dev, host = make_inputs(1, 2, 2, 128, 64, seed=33)
        o, lse = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal)
        got = _c_bwd_noalloc(lib, dev, o, lse, causal, 0.125)
        torch.cuda.synchronize()
        assert fa.fa_last_device_status() == 0
        exact = oracle.attention_backward(host["q"], host["k"], host["v"], host["do"], causal, 0.125)
        for name, g, r in zip(("dq", "dk", "dv"), got, exact):
            assert rel_l2(to_f64(g), r) <= GRAD_REL_L2, (causal, name, rel_l2(to_f64(g), r))


def test_noalloc_at_its_exact_size_limit():
    """B=2, Hq=64, Hkv=16, N=992, d=64 needs exactly FA_BWD_NOALLOC_MAX_BYTES of
    scratch: accepted, equal to fa_bwd, and the first and last KV groups
    equal to the oracle's gradients. One more query head past the limit is
    rejected with FA_ERR_WORKSPACE."""
    import exact_tiled_attention_42_b200 as fa
    from exact_tiled_attention_42_b200 import _lib
    lib = _lib.load()
    B, Hq, Hkv, N, d = 2, 64, 16, 992, 64
    assert fa.fa_bwd_workspace_size(B, Hq, Hkv, N, d) == MAX_BYTES
    dev, host = make_inputs(B, Hq, Hkv, N, d, seed=34)
    o, lse = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=True)
    got = _c_bwd_noalloc(lib, dev, o, lse, True, d ** -0.5)
    ref = fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert rel_l2(to_f64(g), to_f64(r)) <= GRAD_REL_L2, name
    g = Hq // Hkv
    for b, kvh in ((0, 0), (B - 1, Hkv - 1)):
        qs, ks = slice(kvh * g, (kvh + 1) * g), slice(kvh, kvh + 1)
        exact = oracle.attention_backward(host["q"][b:b + 1, qs], host["k"][b:b + 1, ks], host["v"][b:b + 1, ks],
                                          host["do"][b:b + 1, qs], True, d ** -0.5)
        for name, t, r, sl in zip(("dq", "dk", "dv"), got, exact, (qs, ks, ks)):
            assert rel_l2(to_f64(t[b:b + 1, sl]), r) <= GRAD_REL_L2, (b, kvh, name)
    P = torch.empty(16, dtype=torch.uint8, device="cuda").data_ptr()
    assert fa.fa_bwd_workspace_size(1, 129, 129, N, d) > MAX_BYTES
    assert lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 1, 129, 129, N, d, 1, 0.125, None) == 4


def test_noalloc_rejects_problems_larger_than_its_scratch():
    from exact_tiled_attention_42_b200 import _lib
    lib = _lib.load()
    P = torch.empty(16, dtype=torch.uint8, device="cuda").data_ptr()
    # 64 heads x 8192 rows x 128 fp32 = 256 MiB of dQ accumulator alone
    st = lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 2, 32, 8, 8192, 128, 1, 0.088, None)
    assert st == 4  # FA_ERR_WORKSPACE, nothing launched
