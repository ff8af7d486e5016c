"""Forward parity: the CUDA path through the C ABI against the fp64 oracle on
the same seeded bf16 inputs. Tolerances: O max-abs <= 2e-2, LSE max-abs
<= 1e-3."""

import numpy as np
import pytest
import torch

import oracle
from synthetic import WORKLOADS

from _helpers import LSE_MAX_ABS, O_MAX_ABS, make_inputs, to_f64

pytestmark = pytest.mark.gpu


def run_fwd(dev, causal, scale=None):
    import exact_tiled_attention_42_b200 as fa
    o, lse = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    return to_f64(o), lse.cpu().numpy().astype(np.float64)


def check(o, lse, o_ref, lse_ref):
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    err_o = np.max(np.abs(o - o_ref))
    err_l = np.max(np.abs(lse - lse_ref))
    assert err_o <= O_MAX_ABS, f"O max-abs error {err_o}"
    assert err_l <= LSE_MAX_ABS, f"LSE max-abs error {err_l}"


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_workload(causal):
    w = WORKLOADS["tiny"]
    dev, host = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, with_dout=False)
    o, lse = run_fwd(dev, causal)
    o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], causal, w.scale)
    check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("N", [1, 17, 127, 128, 129, 255, 256, 257, 383, 1000])
@pytest.mark.parametrize("d", [64, 96, 128, 192, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_edge_sizes(N, d, causal):
    dev, host = make_inputs(1, 2, 2, N, d, seed=1000 + N + d, with_dout=False)
    o, lse = run_fwd(dev, causal)
    o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], causal, d ** -0.5)
    check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (8, 2), (3, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_small(Hq, Hkv, causal):
    dev, host = make_inputs(2, Hq, Hkv, 300, 128, seed=77 + Hq, with_dout=False)
    o, lse = run_fwd(dev, causal)
    o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], causal, 128 ** -0.5)
    check(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("d", [192, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_wide_heads_gqa_and_many_key_tiles(d, causal):
    """The wide-head kernel (one query tile, 64-key tiles, two score
    buffers) over many key tiles with GQA and a ragged end, plus large
    scores that make the running maximum move."""
    dev, host = make_inputs(2, 4, 2, 1100, d, seed=91 + d, with_dout=False)
    for scale in (d ** -0.5, 0.5):
        o, lse = run_fwd(dev, causal, scale)
        o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], causal, scale)
        check(o, lse, o_ref, lse_ref)


def test_scale_and_large_scores():
    """A large scale spreads scores over many log2 units, which exercises the
    deferred rescale of O (the running max moves by more than the threshold)."""
    dev, host = make_inputs(1, 2, 2, 640, 64, seed=5, with_dout=False)
    for scale in (0.05, 1.0, 3.0):
        for causal in (False, True):
            o, lse = run_fwd(dev, causal, scale)
            o_ref, lse_ref = oracle.attention_forward(host["q"], host["k"], host["v"], causal, scale)
            check(o, lse, o_ref, lse_ref)


def test_repeatable_and_output_untouched_outside():
    """Same inputs give bit-identical outputs; the kernel writes nothing past
    the end of O and LSE (guard regions around both stay intact)."""
    import exact_tiled_attention_42_b200 as fa
    dev, _ = make_inputs(1, 2, 2, 200, 64, seed=9, with_dout=False)
    B, H, N, d = 1, 2, 200, 64
    o_buf = torch.full((B * H * N * d + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((B * H * N + 1024,), 7.0, dtype=torch.float32, device="cuda")
    o = o_buf[:B * H * N * d].view(B, H, N, d)
    lse = l_buf[:B * H * N].view(B, H, N)
    fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=True, out=o, lse=lse)
    first = o.clone()
    fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.equal(first, o)
    assert torch.all(o_buf[B * H * N * d:] == 7.0)
    assert torch.all(l_buf[B * H * N:] == 7.0)


def _sampled_heads(w):
    """(b, hq) pairs compared in full: every query head of KV group 0 in batch
    0 (capped at 4), and the last head of the last batch."""
    g = w.Hq // w.Hkv
    heads = [(0, h) for h in range(min(g, 4))]
    heads.append((w.B - 1, w.Hq - 1))
    return heads


@pytest.mark.parametrize("name", ["gpt2", "long128", "gqa"])
def test_full_size_workloads_sampled(name):
    """Full-size launch (the configuration the benchmark times); sampled
    heads are checked against the oracle in full."""
    w = WORKLOADS[name]
    dev, host = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, with_dout=False)
    g = w.Hq // w.Hkv
    for causal in w.causal:
        o, lse = run_fwd(dev, causal)
        for b, h in _sampled_heads(w):
            kv = h // g
            o_ref, lse_ref = oracle.attention_forward(host["q"][b:b + 1, h:h + 1], host["k"][b:b + 1, kv:kv + 1],
                                                      host["v"][b:b + 1, kv:kv + 1], causal, w.scale)
            check(o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], o_ref, lse_ref)
