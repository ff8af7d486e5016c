"""FP8 path parity.

* The pre-pass is integer/byte work decided in float32: its e4m3 codes and
  float32 block scales must equal the oracle quantiser's bit for bit (the
  rotated values are exact fp64 sums rounded once to fp32 on both sides).
* The FP8 forward is compared with the oracle's fp64 emulation of the same
  steps ("FlashAttention-3: Fast and Accurate Attention with Asynchrony and
  Low-precision", abstract: block quantisation and incoherent processing).
  What may differ, and the gates derived from it:
  - O is bf16 (half an ulp: at most 2^-9 |O|), the emulation fp64: on the
    test inputs this is an RMS of about 3 % of the emulation's own RMS error
    against exact attention.
  - The kernel forms P~ w in fp32 (one FFMA, MUFU ex2.approx, one FMUL);
    its scores agree with the emulation's to about 1e-6 (LSE within 1e-5 on
    every case measured). Where P~ w of one key lies that close to an e4m3
    rounding boundary the two sides pick neighbouring codes: O_ic moves by
    at most 2^-3 P_ij |V_jc| per flipped key (e4m3 has 3 mantissa bits).
  Gates: per element |O - O_emu| <= 2e-2 + 1/4 M_ic, with M_ic the largest
  single term max_j P_ij |V_jc| of the row's own sum (two flips on its
  largest terms; the floor covers the bf16 half-ulp and flips of small
  terms); LSE within 1e-4 (ten times the largest measured gap); and the RMS
  of O - O_emu at most 0.1 of the emulation's RMS error against exact
  attention over all rows but the max(2, 0.1 %) rows with the largest
  difference: a flip of a row's dominant probability moves a whole row (one
  such event in a 400-row case alone is 0.34 of the RMS), and those rows are
  still held to the element bound.
* The kernel must be as accurate as the method: its RMS error against exact
  fp64 attention may exceed the 128-key emulation's, and the single-tile
  emulation's (P rounded against the row's final maximum), by at most 10 %.
* Its error against exact fp64 attention is reported next to the naive
  per-tensor FP8 baseline's (rounding the unnormalised P~ = exp(S - m), and
  the normalised probabilities), and must not be worse than either.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from synthetic import WORKLOADS, sign_vector

from _helpers import O_MAX_ABS, make_inputs, to_f64

pytestmark = pytest.mark.gpu


FP8_LSE_MAX_ABS = 1e-4
FP8_RMS_RATIO = 0.1
FLIP_ROW_SHARE = 1e-3


def attended_max(q, k, v, scale, causal, lse, top=32, chunk=1024):
    """Upper bound of M_ic = max_j P_ij |V_jc| (the largest single term of
    O_ic's sum): exact over each row's `top` most probable keys, and
    P_(top+1) max_j |V_jc| for all the others."""
    B, H, N, d = q.shape
    g = H // k.shape[1]
    out = np.empty((B, H, N, d))
    for b in range(B):
        for h in range(H):
            vabs = np.abs(v[b, h // g])
            vmax = vabs.max(axis=0)
            kk = min(top, N)
            for r0 in range(0, N, chunk):
                r1 = min(N, r0 + chunk)
                s = scale * (q[b, h, r0:r1] @ k[b, h // g].T)
                if causal:
                    s = np.where(np.arange(N)[None, :] > np.arange(r0, r1)[:, None], -np.inf, s)
                p = np.exp(s - lse[b, h, r0:r1, None])
                if kk < N:
                    idx = np.argpartition(-p, kk - 1, axis=1)[:, :kk]
                else:
                    idx = np.tile(np.arange(N), (r1 - r0, 1))
                ptop = np.take_along_axis(p, idx, axis=1)
                m = np.max(ptop[:, :, None] * vabs[idx], axis=1)
                if kk < N:
                    rest = -np.partition(-p, kk, axis=1)[:, kk]
                    m = np.maximum(m, rest[:, None] * vmax[None, :])
                out[b, h, r0:r1] = m
    return out


def check_against_emulation(o, lse, o_emu, lse_emu, q, k, v, causal, scale, sigma=None, single_tile=None):
    exact, lse_exact = oracle.attention_forward(q, k, v, causal, scale)
    M = attended_max(q, k, v, scale, causal, lse_exact)
    bound = O_MAX_ABS + 0.25 * M
    err = np.abs(o - o_emu)
    assert np.all(err <= bound), f"{np.count_nonzero(err > bound)} elements past the flip bound, max {err.max()}"
    assert np.max(np.abs(lse - lse_emu)) <= FP8_LSE_MAX_ABS, np.max(np.abs(lse - lse_emu))
    d = o.shape[-1]
    row_ms = np.mean((o - o_emu).reshape(-1, d) ** 2, axis=1)
    drop = max(2, int(math.ceil(FLIP_ROW_SHARE * row_ms.size)))
    kept = np.sort(row_ms)[:max(1, row_ms.size - drop)]
    rms_diff = math.sqrt(np.mean(kept))
    rms_emu = math.sqrt(np.mean((o_emu - exact) ** 2))
    rms_gpu = math.sqrt(np.mean((o - exact) ** 2))
    assert rms_diff <= FP8_RMS_RATIO * rms_emu, (rms_diff, rms_emu)
    assert rms_gpu <= 1.1 * rms_emu + 1e-4, (rms_gpu, rms_emu)
    if single_tile is None:
        o_one, _ = oracle.fp8_attention_forward(q, k, v, causal, scale, sigma, tile=1 << 30)
    else:
        o_one = single_tile()
    rms_one = math.sqrt(np.mean((o_one - exact) ** 2))
    assert rms_gpu <= 1.1 * rms_one + 1e-4, (rms_gpu, rms_one)
    return exact


def up1024(x):
    return (x + 1023) // 1024 * 1024


def run_fp8(dev, causal, seed, rotate):
    import exact_tiled_attention_42_b200 as fa
    B, Hq, N, d = dev["q"].shape
    Hkv = dev["k"].shape[1]
    ws = torch.empty(fa.fa_fp8_workspace_size(B, Hq, Hkv, N, d), dtype=torch.uint8, device="cuda")
    o, lse = fa.fa_fwd_fp8(dev["q"], dev["k"], dev["v"], causal=causal, rotation_seed=seed,
                           use_rotation=rotate, workspace=ws)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return to_f64(o), lse.cpu().numpy().astype(np.float64), ws.cpu().numpy()


def split_workspace(ws, B, Hq, Hkv, N, d):
    """The documented layout: codes Q, K, V then scales Q, K, V, each region
    1024-byte aligned."""
    nb = -(-N // 64)
    sizes = [B * Hq * N * d, B * Hkv * N * d, B * Hkv * N * d, B * Hq * nb * 4, B * Hkv * nb * 4, B * Hkv * nb * 4]
    out, off = [], 0
    for i, n in enumerate(sizes):
        out.append(ws[off:off + n])
        off += up1024(n)
    codes = [out[0].reshape(B, Hq, N, d), out[1].reshape(B, Hkv, N, d), out[2].reshape(B, Hkv, N, d)]
    scales = [out[3].view(np.float32).reshape(B, Hq, nb), out[4].view(np.float32).reshape(B, Hkv, nb),
              out[5].view(np.float32).reshape(B, Hkv, nb)]
    return codes, scales


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("N", [1, 64, 65, 300])
def test_prepass_codes_and_scales_bit_exact(rotate, N):
    B, Hq, Hkv, d = 1, 4, 2, 128
    dev, host = make_inputs(B, Hq, Hkv, N, d, seed=50 + N, outlier_rate=0.01, with_dout=False)
    seed = 1234 + N
    _, _, ws = run_fp8(dev, False, seed, rotate)
    codes, scales = split_workspace(ws, B, Hq, Hkv, N, d)
    sigma = sign_vector(seed, d)
    for t, name in enumerate(("q", "k", "v")):
        x = host[name]
        if rotate and name != "v":
            x = oracle.rotate_rows(x, sigma)
        vals, sc = oracle.block_quantize(x, 64)
        ref = oracle.e4m3_encode(vals)
        got = codes[t]
        same = (got == ref) | (((got & 0x7F) == 0) & ((ref & 0x7F) == 0))
        assert same.all(), f"{name}: {np.count_nonzero(~same)} codes differ"
        np.testing.assert_array_equal(scales[t], sc)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,Hq,Hkv", [(1, 2, 2), (200, 2, 2), (385, 4, 2), (1000, 2, 1)])
def test_forward_matches_emulation(causal, N, Hq, Hkv):
    d = 128
    dev, host = make_inputs(1, Hq, Hkv, N, d, seed=70 + N, outlier_rate=0.001, with_dout=False)
    seed = 99
    o, lse, _ = run_fp8(dev, causal, seed, True)
    o_emu, lse_emu = oracle.fp8_attention_forward(host["q"], host["k"], host["v"], causal, d ** -0.5,
                                                  sign_vector(seed, d))
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    check_against_emulation(o, lse, o_emu, lse_emu, host["q"], host["k"], host["v"], causal, d ** -0.5,
                            sign_vector(seed, d))


def test_forward_without_rotation_matches_emulation():
    d = 128
    dev, host = make_inputs(1, 2, 2, 640, d, seed=71, outlier_rate=0.001, with_dout=False)
    o, lse, _ = run_fp8(dev, False, 5, False)
    o_emu, lse_emu = oracle.fp8_attention_forward(host["q"], host["k"], host["v"], False, d ** -0.5, None)
    check_against_emulation(o, lse, o_emu, lse_emu, host["q"], host["k"], host["v"], False, d ** -0.5, None)


def test_full_fp8_workload_sampled_error_report():
    """The FP8 workload at full size (B=1, H=16, N=16384, d=128, 0.1% entry
    outliers): heads 0 and 15 against the emulation, and the error of the
    kernel vs exact fp64 attention compared with the naive per-tensor FP8
    baseline on the same heads (reported; block scales + rotation must not be
    worse)."""
    w = WORKLOADS["fp8"]
    dev, host = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, outlier_rate=w.outlier_rate, with_dout=False)
    seed = 4242
    o, lse, _ = run_fp8(dev, False, seed, True)
    sigma = sign_vector(seed, w.d)
    heads = [(0, 0), (0, w.Hq - 1)]
    naive_all = oracle.naive_fp8_attention_forward(host["q"], host["k"], host["v"], False, w.scale, heads=heads)
    naive_norm = oracle.naive_fp8_attention_forward(host["q"], host["k"], host["v"], False, w.scale, heads=heads,
                                                    p_form="normalised")
    for _, h in heads:
        sl = slice(h, h + 1)
        q, k, v = host["q"][:, sl], host["k"][:, sl], host["v"][:, sl]
        o_emu, lse_emu = oracle.fp8_attention_forward(q, k, v, False, w.scale, sigma)
        exact = check_against_emulation(o[:, sl], lse[:, sl], o_emu, lse_emu, q, k, v, False, w.scale, sigma)
        rmse_ours = math.sqrt(np.mean((o[:, sl] - exact) ** 2))
        rmse_naive = math.sqrt(np.mean((naive_all[:, sl] - exact) ** 2))   # per-tensor scales: amax over every head
        rmse_norm = math.sqrt(np.mean((naive_norm[:, sl] - exact) ** 2))
        print(f"head {h}: RMSE fp8 kernel {rmse_ours:.3e}; naive per-tensor fp8 {rmse_naive:.3e} "
              f"(ratio {rmse_naive / rmse_ours:.2f}), with normalised P {rmse_norm:.3e} "
              f"(ratio {rmse_norm / rmse_ours:.2f})")
        assert rmse_ours < rmse_naive and rmse_ours < rmse_norm


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("causal", [False, True])
def test_quantize_then_forward_equals_one_call(rotate, causal):
    """fa_fp8_quantize followed by fa_fwd_fp8_quantized runs the same kernels
    on the same data as fa_fwd_fp8: identical bits; and a second forward
    from the same workspace gives them again (the workspace is only read)."""
    import exact_tiled_attention_42_b200 as fa
    dev, _ = make_inputs(1, 4, 2, 640, 128, seed=611)
    o1, lse1, ws1 = run_fp8(dev, causal, 17, rotate)
    ws = fa.fa_fp8_quantize(dev["q"], dev["k"], dev["v"], rotation_seed=17, use_rotation=rotate)
    shape = (1, 4, 2, 640, 128)
    for _ in range(2):
        o2, lse2 = fa.fa_fwd_fp8_quantized(ws, shape, causal=causal, use_rotation=rotate)
        torch.cuda.synchronize()
        assert fa.fa_last_device_status() == 0
        np.testing.assert_array_equal(to_f64(o2), o1)
        np.testing.assert_array_equal(lse2.cpu().numpy().astype(np.float64), lse1)
    # the documented regions (the padding between them is never written)
    c1, s1 = split_workspace(ws1, *shape)
    c2, s2 = split_workspace(ws.cpu().numpy(), *shape)
    for a, b in zip(c1 + s1, c2 + s2):
        np.testing.assert_array_equal(a, b)
