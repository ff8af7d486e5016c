"""MXFP8 path parity.

* The pre-pass is byte work decided in float32: its e4m3 codes and E8M0
  exponents must equal the oracle quantiser's (``oracle.mx_quantize``) bit for
  bit, for both scale rules, with and without the rotation; V's exponents are
  per 32 keys of a column, stored one 4-byte word per 96-key tile (bytes 0-2
  its blocks, byte 3 zero); blocks past N (up to a whole tile) hold the
  exponent of zeros.
* The forward is compared with the oracle's fp64 emulation of the same steps
  (blocks of 32 along each contraction, P quantised per 32 keys of each
  96-key tile -- the kernel's key tile -- the running max raised only past 4
  in log2 units). What may
  differ is what differs in the per-block FP8 path, with the same gates:
  bf16 rounding of O, fp32 scores and P against fp64, and hence the odd P
  code rounded to the neighbouring e4m3 value (at most 2^-3 P_ij |V_jc| per
  flipped key). A flipped block exponent moves no code in the normal range
  (E4M3's relative grid is the same at every power-of-two scale); it only
  changes a clamped top value (rule "ocp"; under 2^-3 of it) or codes in the
  subnormal range (below 2^-17 of the block's largest value).
* The kernel must be as accurate as the emulation (RMS against exact fp64
  attention within 10 %), and no worse than naive per-tensor FP8.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from synthetic import sign_vector

from _helpers import make_inputs, to_f64
from test_fp8_gpu import check_against_emulation

pytestmark = pytest.mark.gpu

TAU = 4.0   # the kernel's deferred-max threshold (log2 units)
TILE = 96   # the kernel's key tile


def up1024(x):
    return (x + 1023) // 1024 * 1024


def run_mx(dev, causal, seed, rotate, rule):
    import exact_tiled_attention_42_b200 as fa
    B, Hq, N, d = dev["q"].shape
    Hkv = dev["k"].shape[1]
    ws = torch.empty(fa.fa_mxfp8_workspace_size(B, Hq, Hkv, N, d), dtype=torch.uint8, device="cuda")
    o, lse = fa.fa_fwd_mxfp8(dev["q"], dev["k"], dev["v"], causal=causal, rotation_seed=seed,
                             use_rotation=rotate, scale_rule=rule, workspace=ws)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return to_f64(o), lse.cpu().numpy().astype(np.float64), ws.cpu().numpy()


def split_workspace(ws, B, Hq, Hkv, N, d):
    """The documented layout: codes Q, K, V; exponent bytes Q [BHq, N, 4],
    K [BHkv, N, 4], V [BHkv, d, nb] with nb = 4 ceil(N / 96); each region
    1024-byte aligned."""
    nb = 4 * (-(-N // TILE))
    sizes = [B * Hq * N * d, B * Hkv * N * d, B * Hkv * N * d, B * Hq * N * 4, B * Hkv * N * 4, B * Hkv * d * nb]
    out, off = [], 0
    for n in sizes:
        out.append(ws[off:off + n])
        off += up1024(n)
    codes = [out[0].reshape(B, Hq, N, d), out[1].reshape(B, Hkv, N, d), out[2].reshape(B, Hkv, N, d)]
    exps = [out[3].reshape(B, Hq, N, 4).astype(np.int64) - 127, out[4].reshape(B, Hkv, N, 4).astype(np.int64) - 127,
            out[5].reshape(B, Hkv, d, nb).astype(np.int64) - 127]
    return codes, exps


@pytest.mark.parametrize("rule", ["fit", "ocp"])
@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("N", [1, 33, 300])
def test_prepass_codes_and_exponents_bit_exact(rule, rotate, N):
    B, Hq, Hkv, d = 1, 4, 2, 128
    dev, host = make_inputs(B, Hq, Hkv, N, d, seed=150 + N, outlier_rate=0.01, with_dout=False)
    seed = 777 + N
    _, _, ws = run_mx(dev, False, seed, rotate, rule)
    codes, exps = split_workspace(ws, B, Hq, Hkv, N, d)
    sigma = sign_vector(seed, d)
    for t, name in enumerate(("q", "k", "v")):
        x = host[name]
        if rotate and name != "v":
            x = oracle.rotate_rows(x, sigma)
        x = x.astype(np.float32)
        axis = -2 if name == "v" else -1
        vals, e = oracle.mx_quantize(x, axis=axis, rule=rule)
        ref = oracle.e4m3_encode(vals)
        got = codes[t]
        same = (got == ref) | (((got & 0x7F) == 0) & ((ref & 0x7F) == 0))
        assert same.all(), f"{name}: {np.count_nonzero(~same)} codes differ"
        if name == "v":
            nb = e.shape[-2]                                # blocks of 32 keys: [B, H, nb, d]
            words = exps[2].reshape(B, Hkv, d, -1, 4)       # [B, H, d, tiles, 4]
            blocks = words[..., :3].reshape(B, Hkv, d, -1)  # the tiles' three blocks in order
            np.testing.assert_array_equal(blocks[..., :nb], np.swapaxes(e, -1, -2))
            assert np.all(blocks[..., nb:] == -127)
            assert np.all(words[..., 3] == -127)            # byte 3 of each word is 0
        else:
            np.testing.assert_array_equal(exps[t], e)


@pytest.mark.parametrize("rule", ["fit", "ocp"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,Hq,Hkv", [(1, 2, 2), (200, 2, 2), (385, 4, 2), (1000, 2, 1)])
def test_forward_matches_emulation(rule, causal, N, Hq, Hkv):
    d = 128
    dev, host = make_inputs(1, Hq, Hkv, N, d, seed=170 + N, outlier_rate=0.001, with_dout=False)
    seed = 99
    sigma = sign_vector(seed, d)
    o, lse, _ = run_mx(dev, causal, seed, True, rule)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    o_emu, lse_emu = oracle.mxfp8_attention_forward(host["q"], host["k"], host["v"], causal, d ** -0.5, sigma,
                                                    tile=TILE, rule=rule, tau=TAU)
    check_against_emulation(o, lse, o_emu, lse_emu, host["q"], host["k"], host["v"], causal, d ** -0.5, sigma,
                            single_tile=lambda: oracle.mxfp8_attention_forward(
                                host["q"], host["k"], host["v"], causal, d ** -0.5, sigma, tile=1 << 30,
                                rule=rule)[0])


def test_forward_without_rotation_matches_emulation():
    d = 128
    dev, host = make_inputs(1, 2, 2, 640, d, seed=171, outlier_rate=0.001, with_dout=False)
    o, lse, _ = run_mx(dev, False, 5, False, "fit")
    o_emu, lse_emu = oracle.mxfp8_attention_forward(host["q"], host["k"], host["v"], False, d ** -0.5, None,
                                                    tile=TILE, rule="fit", tau=TAU)
    check_against_emulation(o, lse, o_emu, lse_emu, host["q"], host["k"], host["v"], False, d ** -0.5, None,
                            single_tile=lambda: oracle.mxfp8_attention_forward(
                                host["q"], host["k"], host["v"], False, d ** -0.5, None, tile=1 << 30,
                                rule="fit")[0])


def test_mxfp8_error_report_against_fp8_and_naive():
    """One head of the FP8 workload's recipe (N = 4096, 0.1 % entry outliers):
    RMS error against exact fp64 attention of the MXFP8 kernel (both rules),
    the per-block FP8 kernel and naive per-tensor FP8 (reported; MXFP8 must
    beat the naive baseline)."""
    import exact_tiled_attention_42_b200 as fa
    d, N = 128, 4096
    dev, host = make_inputs(1, 1, 1, N, d, seed=4243, outlier_rate=0.001, with_dout=False)
    exact, _ = oracle.attention_forward(host["q"], host["k"], host["v"], False, d ** -0.5)
    naive = oracle.naive_fp8_attention_forward(host["q"], host["k"], host["v"], False, d ** -0.5)
    o8, _ = fa.fa_fwd_fp8(dev["q"], dev["k"], dev["v"], rotation_seed=3)
    rms = lambda a: math.sqrt(np.mean((a - exact) ** 2))
    r = {"naive": rms(naive), "fp8 64-row blocks": rms(to_f64(o8))}
    for rule in ("fit", "ocp"):
        o, _, _ = run_mx(dev, False, 3, True, rule)
        r[f"mxfp8 {rule}"] = rms(o)
    print("RMS error vs exact: " + ", ".join(f"{k} {v:.3e}" for k, v in r.items()))
    assert r["mxfp8 fit"] < r["naive"] and r["mxfp8 ocp"] < r["naive"]
