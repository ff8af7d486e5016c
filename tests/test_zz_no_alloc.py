"""fa_bwd_noalloc: the backward for callers that cannot allocate device
memory at the call (it takes its scratch from a fixed array inside the
library). Called through the C ABI and checked against fa_bwd, the entry
point with a caller-provided workspace, on two calls in a row with different
inputs, so the second call starts from the scratch the first one left.
Collected last so that a stopping run has already run every other test."""

import ctypes

import numpy as np
import pytest
import torch

from _helpers import GRAD_REL_L2, make_inputs, rel_l2, to_f64

pytestmark = pytest.mark.gpu


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


def test_noalloc_rejects_problems_larger_than_its_scratch():
    from exact_tiled_attention_42_b200 import _lib
    lib = _lib.load()
    P = torch.empty(16, dtype=torch.uint8, device="cuda").data_ptr()
    # 64 heads x 8192 rows x 128 fp32 = 256 MiB of dQ accumulator alone
    st = lib.fa_bwd_noalloc(P, P, P, P, P, P, P, P, P, 2, 32, 8, 8192, 128, 1, 0.088, None)
    assert st == 4  # FA_ERR_WORKSPACE, nothing launched
