"""Every entry point writes exactly its outputs: each output tensor and each
workspace sits inside a larger buffer whose margins hold a fixed pattern
(NaN for floating outputs, 0xA5 for workspaces), at ragged sizes. After the
call the margins are unchanged and every output element was written (no NaN
left inside). Stands in for a device-side bounds checker, which is not
available on this machine."""

import numpy as np
import pytest
import torch

from _helpers import make_inputs

pytestmark = pytest.mark.gpu

GUARD = 4096


def guarded(shape, dtype):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), float("nan"), dtype=dtype, device="cuda")
    return buf[GUARD:GUARD + n].view(shape), buf


def guarded_ws(nbytes):
    buf = torch.full((nbytes + 2 * GUARD,), 0xA5, dtype=torch.uint8, device="cuda")
    return buf[GUARD:GUARD + nbytes], buf


def check_output(view, buf):
    torch.cuda.synchronize()
    a = buf.float().cpu().numpy()
    assert np.isnan(a[:GUARD]).all() and np.isnan(a[-GUARD:]).all(), "write outside the output"
    assert not torch.isnan(view.float()).any(), "output element left unwritten"


def check_ws(buf):
    torch.cuda.synchronize()
    a = buf.cpu().numpy()
    assert (a[:GUARD] == 0xA5).all() and (a[-GUARD:] == 0xA5).all(), "write outside the workspace"


@pytest.mark.parametrize("d", [64, 96, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_outputs_and_workspace(d, causal):
    import exact_tiled_attention_42_b200 as fa
    B, Hq, Hkv, N = 2, 4, 2, 200
    dev, _ = make_inputs(B, Hq, Hkv, N, d, seed=5 + d, with_dout=True)
    o, lse = fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal)
    dq, bq = guarded((B, Hq, N, d), torch.bfloat16)
    dk, bk = guarded((B, Hkv, N, d), torch.bfloat16)
    dv, bv = guarded((B, Hkv, N, d), torch.bfloat16)
    ws, bw = guarded_ws(fa.fa_bwd_workspace_size(B, Hq, Hkv, N, d))
    fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal=causal, dq=dq, dk=dk, dv=dv, workspace=ws)
    assert fa.fa_last_device_status() == 0
    for view, buf in ((dq, bq), (dk, bk), (dv, bv)):
        check_output(view, buf)
    check_ws(bw)


@pytest.mark.parametrize("d", [192, 256])
def test_wide_forward_outputs(d):
    import exact_tiled_attention_42_b200 as fa
    B, Hq, Hkv, N = 1, 2, 1, 137
    dev, _ = make_inputs(B, Hq, Hkv, N, d, seed=7, with_dout=False)
    o, bo = guarded((B, Hq, N, d), torch.bfloat16)
    lse, bl = guarded((B, Hq, N), torch.float32)
    fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=True, out=o, lse=lse)
    assert fa.fa_last_device_status() == 0
    check_output(o, bo)
    check_output(lse, bl)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_outputs_and_workspace(causal):
    import exact_tiled_attention_42_b200 as fa
    B, Hq, Hkv, N, d = 1, 4, 2, 333, 128
    dev, _ = make_inputs(B, Hq, Hkv, N, d, seed=11, outlier_rate=0.001, with_dout=False)
    o, bo = guarded((B, Hq, N, d), torch.bfloat16)
    lse, bl = guarded((B, Hq, N), torch.float32)
    ws, bw = guarded_ws(fa.fa_fp8_workspace_size(B, Hq, Hkv, N, d))
    fa.fa_fwd_fp8(dev["q"], dev["k"], dev["v"], causal=causal, rotation_seed=3, out=o, lse=lse, workspace=ws)
    assert fa.fa_last_device_status() == 0
    check_output(o, bo)
    check_output(lse, bl)
    check_ws(bw)


@pytest.mark.parametrize("rule", ["fit", "ocp"])
@pytest.mark.parametrize("causal", [False, True])
def test_mxfp8_outputs_and_workspace(rule, causal):
    import exact_tiled_attention_42_b200 as fa
    B, Hq, Hkv, N, d = 1, 4, 2, 333, 128
    dev, _ = make_inputs(B, Hq, Hkv, N, d, seed=13, outlier_rate=0.001, with_dout=False)
    o, bo = guarded((B, Hq, N, d), torch.bfloat16)
    lse, bl = guarded((B, Hq, N), torch.float32)
    ws, bw = guarded_ws(fa.fa_mxfp8_workspace_size(B, Hq, Hkv, N, d))
    fa.fa_fwd_mxfp8(dev["q"], dev["k"], dev["v"], causal=causal, rotation_seed=3, scale_rule=rule, out=o, lse=lse,
                    workspace=ws)
    assert fa.fa_last_device_status() == 0
    check_output(o, bo)
    check_output(lse, bl)
    check_ws(bw)


@pytest.mark.parametrize("Nq,Nk", [(1, 1000), (3, 4097)])
def test_decode_outputs_and_workspace(Nq, Nk):
    import exact_tiled_attention_42_b200 as fa
    B, Hq, Hkv, d = 2, 8, 2, 128
    qd, _ = make_inputs(B, Hq, Hq, Nq, d, seed=17, with_dout=False)
    kv, _ = make_inputs(B, Hkv, Hkv, Nk, d, seed=18, with_dout=False)
    o, bo = guarded((B, Hq, Nq, d), torch.bfloat16)
    lse, bl = guarded((B, Hq, Nq), torch.float32)
    ws, bw = guarded_ws(fa.fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, 0))
    fa.fa_fwd_decode(qd["q"], kv["k"], kv["v"], causal=True, out=o, lse=lse, workspace=ws)
    assert fa.fa_last_device_status() == 0
    check_output(o, bo)
    check_output(lse, bl)
    check_ws(bw)
