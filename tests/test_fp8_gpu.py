"""FP8 path parity.

* The pre-pass is integer/byte work decided in float32: its e4m3 codes and
  float32 block scales must equal the oracle quantiser's bit for bit (the
  rotated values are exact fp64 sums rounded once to fp32 on both sides).
* The FP8 forward is compared with the oracle's fp64 emulation of the same
  steps. The kernel's scores come from the FP8 tensor-core product, which is
  not exact to fp64 (relative error of order 1e-4 in the log2-domain scores);
  near an e4m3 rounding boundary that flips P's code by one step (up to 1/8
  of its value), and in a peaked row one flip moves O visibly. The emulation
  itself moves by the same amount (0.06 max, 3e-4 RMS on a 385-row case) when
  its scores are perturbed by 1e-4 relative. So the bound per element is
  2e-2 + 1/4 * Pmax_i * max|V| (one step on the row's two largest
  probabilities; Pmax_i the exact largest probability of row i) and LSE must
  agree within 1e-2. The RMS of kernel - emulation must stay under half the
  emulation's own RMS error against exact attention, and the kernel's RMS
  error against exact attention may exceed the emulation's by at most 10 %:
  the kernel must be as accurate as the emulated method, not equal to it.
* The kernel's error against exact fp64 attention is reported next to the
  naive per-tensor FP8 baseline's, and must not be worse.
"""

FP8_LSE_MAX_ABS = 1e-2


def row_pmax(q, k, scale, causal, lse, chunk=2048):
    """Largest softmax probability of each row: exp(max_j S_ij - LSE_i)."""
    B, H, N, d = q.shape
    g = H // k.shape[1]
    out = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, chunk):
                r1 = min(N, r0 + chunk)
                s = scale * (q[b, h, r0:r1] @ k[b, h // g].T)
                if causal:
                    s = np.where(np.arange(N)[None, :] > np.arange(r0, r1)[:, None], -np.inf, s)
                out[b, h, r0:r1] = np.exp(s.max(axis=1) - lse[b, h, r0:r1])
    return out


def check_against_emulation(o, lse, o_emu, lse_emu, q, k, v, causal, scale):
    exact, lse_exact = oracle.attention_forward(q, k, v, causal, scale)
    pmax = row_pmax(q, k, scale, causal, lse_exact)
    bound = O_MAX_ABS + 0.25 * pmax[..., None] * np.abs(v).max()
    err = np.abs(o - o_emu)
    assert np.all(err <= bound), f"{np.count_nonzero(err > bound)} elements past the flip bound, max {err.max()}"
    rms_diff = math.sqrt(np.mean((o - o_emu) ** 2))
    rms_emu = math.sqrt(np.mean((o_emu - exact) ** 2))
    rms_gpu = math.sqrt(np.mean((o - exact) ** 2))
    assert rms_diff <= 0.5 * rms_emu, (rms_diff, rms_emu)
    assert rms_gpu <= 1.1 * rms_emu + 1e-4, (rms_gpu, rms_emu)
    assert np.max(np.abs(lse - lse_emu)) <= FP8_LSE_MAX_ABS, np.max(np.abs(lse - lse_emu))
    return exact

import math

import numpy as np
import pytest
import torch

import oracle
from synthetic import WORKLOADS, sign_vector

from _helpers import O_MAX_ABS, make_inputs, to_f64

pytestmark = pytest.mark.gpu


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
    check_against_emulation(o, lse, o_emu, lse_emu, host["q"], host["k"], host["v"], causal, d ** -0.5)


def test_forward_without_rotation_matches_emulation():
    d = 128
    dev, host = make_inputs(1, 2, 2, 640, d, seed=71, outlier_rate=0.001, with_dout=False)
    o, lse, _ = run_fp8(dev, False, 5, False)
    o_emu, lse_emu = oracle.fp8_attention_forward(host["q"], host["k"], host["v"], False, d ** -0.5, None)
    check_against_emulation(o, lse, o_emu, lse_emu, host["q"], host["k"], host["v"], False, d ** -0.5)


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
    for _, h in heads:
        sl = slice(h, h + 1)
        q, k, v = host["q"][:, sl], host["k"][:, sl], host["v"][:, sl]
        o_emu, lse_emu = oracle.fp8_attention_forward(q, k, v, False, w.scale, sigma)
        exact = check_against_emulation(o[:, sl], lse[:, sl], o_emu, lse_emu, q, k, v, False, w.scale)
        naive = naive_all[:, sl]  # per-tensor scales: amax over every head
        rmse_ours = math.sqrt(np.mean((o[:, sl] - exact) ** 2))
        rmse_naive = math.sqrt(np.mean((naive - exact) ** 2))
        print(f"head {h}: RMSE fp8 kernel {rmse_ours:.3e}, naive per-tensor fp8 {rmse_naive:.3e}, "
              f"ratio {rmse_naive / rmse_ours:.2f}")
        assert rmse_ours < rmse_naive


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
