"""A bounded wait that runs out: the abort path, on the GPU, without a fault.

The debug variant of the library (libfa_b200_debug.so: the same sources with
a 1 ms bound on every wait and a switch, fa_debug_withhold_first_v, that keeps
the forward's producer from issuing its first V tile) is called through its C
ABI. With the switch on, the MMA warp of every CTA waits for a copy that never
comes; the wait gives up after 1 ms, raises the CTA's abort flag, every role
leaves its loop, in-flight copies and MMAs drain, tensor memory is freed and
the kernel returns. The host then reads FA_ERR_TIMEOUT with the site of the
wait from fa_last_device_status. The same context must keep working: the
next call with the switch off, and the release library, match the oracle."""

import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
from _helpers import LSE_MAX_ABS, O_MAX_ABS, make_inputs, to_f64

pytestmark = pytest.mark.gpu

FA_ERR_TIMEOUT = 6
# The waits on the withheld tile's chain; whichever started first gives up
# first: the MMA warp's wait for the V tile, the producer's wait for the slot
# that tile never frees, and the softmax warps' wait for the next S, which the
# MMA warp never issues.
SITE_V_FULL = 3
SITE_V_EMPTY = 5
SITE_S_FULL = 6


def _debug_lib():
    from exact_tiled_attention_42_b200 import _lib
    path = os.path.join(os.path.dirname(_lib.LIB_PATH), "libfa_b200_debug.so")
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m exact_tiled_attention_42_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _lib.SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    lib.fa_debug_withhold_first_v.restype = None
    lib.fa_debug_withhold_first_v.argtypes = [ctypes.c_int]
    return lib


def _fwd(lib, dev, o, lse, causal):
    B, Hq, N, d = dev["q"].shape
    return lib.fa_fwd(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(), o.data_ptr(), lse.data_ptr(),
                      B, Hq, dev["k"].shape[1], N, d, int(causal), d ** -0.5,
                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_withheld_copy_times_out_and_the_context_survives():
    import exact_tiled_attention_42_b200 as fa
    dbg = _debug_lib()
    assert dbg.fa_last_device_status() == 0          # clean start
    B, Hq, Hkv, N, d = 1, 2, 1, 300, 128
    dev, host = make_inputs(B, Hq, Hkv, N, d, seed=61, with_dout=False)
    exact, lse_exact = oracle.attention_forward(host["q"], host["k"], host["v"], True, d ** -0.5)
    o = torch.zeros_like(dev["q"])
    lse = torch.zeros((B, Hq, N), dtype=torch.float32, device="cuda")

    dbg.fa_debug_withhold_first_v(1)
    try:
        assert _fwd(dbg, dev, o, lse, True) == 0     # the launch itself is fine
        status = dbg.fa_last_device_status()         # synchronises: the kernel returned
    finally:
        dbg.fa_debug_withhold_first_v(0)
    assert status & 0xFF == FA_ERR_TIMEOUT, hex(status)
    assert status >> 8 in (SITE_V_FULL, SITE_V_EMPTY, SITE_S_FULL), hex(status)
    assert dbg.fa_last_device_status() == 0          # reading cleared it

    # same context, switch off: a normal result
    assert _fwd(dbg, dev, o, lse, True) == 0
    assert dbg.fa_last_device_status() == 0
    assert np.max(np.abs(to_f64(o) - exact)) <= O_MAX_ABS
    assert np.max(np.abs(lse.cpu().numpy() - lse_exact)) <= LSE_MAX_ABS

    # and the release library in the same process
    o2, lse2 = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=True)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert np.max(np.abs(to_f64(o2) - exact)) <= O_MAX_ABS
    assert np.max(np.abs(lse2.cpu().numpy() - lse_exact)) <= LSE_MAX_ABS
