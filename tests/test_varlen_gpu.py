"""Packed variable-length batches on the GPU against the fp64 oracle.

Sequences of mixed lengths (empty, one token, ragged, several tiles) are
packed token-major ([T, H, d]) with int32 offsets; every sequence must come
out as if it had been run alone: O within 2e-2 and LSE within 1e-3 of the
oracle, dQ, dK, dV within relative L2 1e-2 per sequence. Guard regions around
every output catch a store that strays past a sequence's end into a
neighbour's rows or past the tensor."""

import numpy as np
import pytest
import torch

import oracle
from synthetic import attention_inputs, bf16_bits_to_f32

from _helpers import GRAD_REL_L2, LSE_MAX_ABS, O_MAX_ABS, rel_l2, to_f64

pytestmark = pytest.mark.gpu

CASES = [
    # lengths, Hq, Hkv, d
    ([1, 127, 128, 129, 300], 2, 2, 128),
    ([0, 64, 1000, 5, 256], 4, 2, 128),
    ([200, 7, 385], 2, 1, 64),
    ([130, 0, 250], 2, 2, 96),
    ([513], 2, 2, 128),
]


def _packed_inputs(lens, Hq, Hkv, d, seed):
    T = int(sum(lens))
    bits = attention_inputs(1, Hq, Hkv, T, d, seed)                 # [1, H, T, d] bits
    to_tok = lambda a: np.ascontiguousarray(np.transpose(a[0], (1, 0, 2)))   # [T, H, d]
    host = {n: bf16_bits_to_f32(to_tok(a)).astype(np.float64) for n, a in bits.items()}
    dev = {n: torch.from_numpy(to_tok(a).view(np.int16)).view(torch.bfloat16).cuda() for n, a in bits.items()}
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return dev, host, cu


def _guarded(shape, dtype, guard=4096):
    """A tensor of `shape` inside a larger buffer whose margins hold a NaN
    pattern: returns (view, whole buffer)."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * guard,), float("nan"), dtype=dtype, device="cuda")
    return buf[guard:guard + n].view(shape), buf, guard


def _margins_intact(buf, guard):
    a = buf.float().cpu().numpy()
    return np.isnan(a[:guard]).all() and np.isnan(a[-guard:]).all()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lens,Hq,Hkv,d", CASES)
def test_varlen_forward_and_backward(lens, Hq, Hkv, d, causal):
    import exact_tiled_attention_42_b200 as fa
    dev, host, cu = _packed_inputs(lens, Hq, Hkv, d, seed=81 + len(lens) + d)
    T = int(cu[-1])
    cu_dev = torch.from_numpy(cu).cuda()
    scale = d ** -0.5
    maxlen = max(lens)
    o, obuf, g = _guarded((T, Hq, d), torch.bfloat16)
    lse, lbuf, gl = _guarded((Hq, T), torch.float32)
    fa.fa_fwd_varlen(dev["q"], dev["k"], dev["v"], cu_dev, maxlen, causal=causal, out=o, lse=lse)
    dq, qbuf, gq = _guarded((T, Hq, d), torch.bfloat16)
    dk, kbuf, gk = _guarded((T, Hkv, d), torch.bfloat16)
    dv, vbuf, gv = _guarded((T, Hkv, d), torch.bfloat16)
    fa.fa_bwd_varlen(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], cu_dev, maxlen, causal=causal,
                     dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    for buf, gg in ((obuf, g), (lbuf, gl), (qbuf, gq), (kbuf, gk), (vbuf, gv)):
        assert _margins_intact(buf, gg)
    o_ref, lse_ref = oracle.varlen_forward(host["q"], host["k"], host["v"], cu, causal, scale)
    grads = oracle.varlen_backward(host["q"], host["k"], host["v"], host["do"], cu, causal, scale)
    o_got, lse_got = to_f64(o), lse.cpu().numpy().astype(np.float64)
    got = [to_f64(t) for t in (dq, dk, dv)]
    assert np.all(np.isfinite(o_got)) and np.all(np.isfinite(lse_got))
    assert np.max(np.abs(o_got - o_ref)) <= O_MAX_ABS
    assert np.max(np.abs(lse_got - lse_ref)) <= LSE_MAX_ABS
    for b in range(len(lens)):
        s0, s1 = cu[b], cu[b + 1]
        if s1 == s0:
            continue
        for name, gt, ref in zip(("dq", "dk", "dv"), got, grads):
            assert np.all(np.isfinite(gt[s0:s1]))
            assert rel_l2(gt[s0:s1], ref[s0:s1]) <= GRAD_REL_L2, (b, name, rel_l2(gt[s0:s1], ref[s0:s1]))


@pytest.mark.parametrize("d", [192, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_wide_heads_forward(d, causal):
    """The wide-head forward on a packed batch (its backward is not built)."""
    import exact_tiled_attention_42_b200 as fa
    lens = [70, 0, 300, 129]
    dev, host, cu = _packed_inputs(lens, 4, 2, d, seed=93 + d)
    T = int(cu[-1])
    o, obuf, g = _guarded((T, 4, d), torch.bfloat16)
    lse, lbuf, gl = _guarded((4, T), torch.float32)
    fa.fa_fwd_varlen(dev["q"], dev["k"], dev["v"], torch.from_numpy(cu).cuda(), max(lens), causal=causal,
                     out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0
    assert _margins_intact(obuf, g) and _margins_intact(lbuf, gl)
    o_ref, lse_ref = oracle.varlen_forward(host["q"], host["k"], host["v"], cu, causal, d ** -0.5)
    assert np.max(np.abs(to_f64(o) - o_ref)) <= O_MAX_ABS
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= LSE_MAX_ABS


def test_varlen_equal_lengths_match_the_batched_entry_points():
    """Equal lengths packed: the same numbers as fa_fwd / fa_bwd on the
    [B, H, N, d] layout, within the bf16 tolerances."""
    import exact_tiled_attention_42_b200 as fa
    B, H, N, d = 3, 2, 300, 128
    bits = attention_inputs(B, H, H, N, d, seed=90)
    dev4 = {n: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for n, a in bits.items()}
    pack = lambda t: t.permute(0, 2, 1, 3).reshape(B * N, H, d).contiguous()
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    o4, l4 = fa.fa_fwd(dev4["q"], dev4["k"], dev4["v"], causal=True)
    g4 = fa.fa_bwd(dev4["q"], dev4["k"], dev4["v"], o4, l4, dev4["do"], causal=True)
    op, lp = fa.fa_fwd_varlen(pack(dev4["q"]), pack(dev4["k"]), pack(dev4["v"]), cu, N, causal=True)
    gp = fa.fa_bwd_varlen(pack(dev4["q"]), pack(dev4["k"]), pack(dev4["v"]), op, lp, pack(dev4["do"]), cu, N,
                          causal=True)
    torch.cuda.synchronize()
    assert np.max(np.abs(to_f64(op) - to_f64(pack(o4)))) <= O_MAX_ABS
    assert np.max(np.abs(lp.cpu().numpy() - l4.permute(1, 0, 2).reshape(H, B * N).cpu().numpy())) <= LSE_MAX_ABS
    for a, b_ in zip(gp, g4):
        assert rel_l2(to_f64(a), to_f64(pack(b_))) <= GRAD_REL_L2


def test_varlen_bad_offsets_reported_on_the_device():
    """Offsets the host cannot see (they live on the device) are checked by
    the kernels: a length above max_seqlen or offsets past T give
    FA_ERR_INVALID_ARG in the device status word, and nothing is written."""
    import exact_tiled_attention_42_b200 as fa
    dev, _, cu = _packed_inputs([100, 100], 2, 2, 64, seed=91)
    o = torch.zeros_like(dev["q"])
    bad = torch.tensor([0, 150, 200], dtype=torch.int32, device="cuda")    # length 150 > max_seqlen 100
    fa.fa_fwd_varlen(dev["q"], dev["k"], dev["v"], bad, 100, out=o)
    st = fa.fa_last_device_status()
    assert st & 0xFF == 1 and st >> 8 == 64, hex(st)
    assert torch.count_nonzero(o[:150]).item() == 0
    good = torch.from_numpy(cu).cuda()
    fa.fa_fwd_varlen(dev["q"], dev["k"], dev["v"], good, 100, out=o)
    assert fa.fa_last_device_status() == 0
