"""Bounds checks of every computed global index, on the GPU.

The debug library (libfa_b200_debug.so, built with FA_DEBUG_BOUNDS) checks
each global index a kernel computes against its buffer before the access and
records FA_ERR_BOUNDS | (96 + site) << 8 in the status word instead of
touching memory out of range (the stand-in for a device bounds checker,
which is not available here). Every entry point runs through the debug
library at small, odd sizes (ragged tiles, packed batches with an empty
sequence, GQA, both masks): no check may fire, and the results must equal
the release library's (bit for bit where the arithmetic order is fixed; dQ
is an fp32 sum of reduce-adds that land in any order, rounded to bf16, so
the odd element may sit one bf16 step away: within 2^-7 relative)."""

import numpy as np
import pytest
import torch

from _helpers import make_inputs
from test_wait_timeout_gpu import _debug_lib

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg():
    return _debug_lib()


def both(dbg, fn):
    """fn() through the release library, then through the debug library;
    returns (release results, debug results) as float64 arrays."""
    import exact_tiled_attention_42_b200 as fa
    from exact_tiled_attention_42_b200 import _lib
    rel = [t.float().cpu().numpy() for t in fn()]
    assert fa.fa_last_device_status() == 0
    release_load = _lib.load
    _lib.load = lambda: dbg
    try:
        out = [t.float().cpu().numpy() for t in fn()]
        torch.cuda.synchronize()
        status = dbg.fa_last_device_status()
    finally:
        _lib.load = release_load
    assert status == 0, f"debug library status {status:#x}"
    return rel, out


def same(a, b):
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 64), (77, 96), (300, 128), (137, 192), (129, 256)])
def test_forward(dbg, N, d, causal):
    import exact_tiled_attention_42_b200 as fa
    dev, _ = make_inputs(2, 4, 2, N, d, seed=N + d, with_dout=False)
    rel, out = both(dbg, lambda: fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal))
    for a, b in zip(rel, out):
        same(a, b)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(77, 64), (300, 96), (257, 128)])
def test_backward(dbg, N, d, causal):
    import exact_tiled_attention_42_b200 as fa
    dev, _ = make_inputs(2, 4, 2, N, d, seed=3 * N + d, with_dout=True)
    o, lse = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal)
    rel, out = both(dbg, lambda: fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal=causal))
    np.testing.assert_allclose(out[0], rel[0], rtol=2 ** -7, atol=1e-6)   # dQ: one bf16 step
    same(rel[1], out[1])                                               # dK
    same(rel[2], out[2])                                               # dV


@pytest.mark.parametrize("d", [64, 128, 256])
def test_packed_batch(dbg, d):
    import exact_tiled_attention_42_b200 as fa
    lens = [150, 0, 77, 300]
    T = sum(lens)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    dev, _ = make_inputs(1, 4, 4, T, d, seed=11 + d, with_dout=True)
    tok = {n: t[0].transpose(0, 1).contiguous() for n, t in dev.items()}   # [T, H, d]
    q, k, v, do = tok["q"], tok["k"][:, :2].contiguous(), tok["v"][:, :2].contiguous(), tok["do"]
    rel, out = both(dbg, lambda: fa.fa_fwd_varlen(q, k, v, cu, max_seqlen=300, causal=True))
    for a, b in zip(rel, out):
        same(a, b)
    if d <= 128:
        o, lse = fa.fa_fwd_varlen(q, k, v, cu, max_seqlen=300, causal=True)
        rel, out = both(dbg, lambda: fa.fa_bwd_varlen(q, k, v, o, lse, do, cu, max_seqlen=300, causal=True))
        np.testing.assert_allclose(out[0], rel[0], rtol=2 ** -7, atol=1e-6)
        same(rel[1], out[1])
        same(rel[2], out[2])


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_and_mxfp8(dbg, causal):
    import exact_tiled_attention_42_b200 as fa
    dev, _ = make_inputs(1, 4, 2, 333, 128, seed=21, outlier_rate=0.001, with_dout=False)
    rel, out = both(dbg, lambda: fa.fa_fwd_fp8(dev["q"], dev["k"], dev["v"], causal=causal, rotation_seed=5))
    for a, b in zip(rel, out):
        same(a, b)
    for rule in ("fit", "ocp"):
        rel, out = both(dbg, lambda: fa.fa_fwd_mxfp8(dev["q"], dev["k"], dev["v"], causal=causal, rotation_seed=5,
                                                     scale_rule=rule))
        for a, b in zip(rel, out):
            same(a, b)


@pytest.mark.parametrize("Nq,Nk", [(1, 1000), (3, 4097)])
def test_decode(dbg, Nq, Nk):
    import exact_tiled_attention_42_b200 as fa
    qd, _ = make_inputs(2, 8, 8, Nq, 128, seed=31, with_dout=False)
    kv, _ = make_inputs(2, 2, 2, Nk, 128, seed=32, with_dout=False)
    rel, out = both(dbg, lambda: fa.fa_fwd_decode(qd["q"], kv["k"], kv["v"], causal=True))
    for a, b in zip(rel, out):
        same(a, b)
