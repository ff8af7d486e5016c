"""The Python binding's marshalling, on the host (no GPU): every entry point
passes the C ABI the declared number of arguments, each convertible to its
declared C type, with the tensors' addresses and the sizes in the header's
order; and every tensor the library would write (outputs, workspaces) is
checked for shape, dtype, contiguity and device before the call, so that a
wrong one raises in Python instead of reaching a kernel that indexes it by
the documented shape alone.

The library's compute entry points are replaced by a recorder that checks
each argument against the ctypes signature and returns a chosen status; the
size queries and status strings are the real library's (host arithmetic).
CPU tensors stand in for device tensors."""

import os

import pytest
import torch

import exact_tiled_attention_42_b200 as fa
from exact_tiled_attention_42_b200 import _lib, api

B, HQ, HKV, N, D = 1, 4, 2, 8, 64
BF, F32 = torch.bfloat16, torch.float32


class Recorder:
    def __init__(self, real):
        self.real, self.calls, self.status = real, [], 0

    def __getattr__(self, name):
        if name.endswith("_workspace_size") or name == "fa_status_string":
            return getattr(self.real, name)
        _, argtypes = _lib.SIGNATURES[name]

        def call(*args):
            assert len(args) == len(argtypes), f"{name}: {len(args)} arguments, {len(argtypes)} declared"
            for a, t in zip(args, argtypes):
                t(a)   # ctypes raises TypeError for an argument it cannot convert
            self.calls.append((name, args))
            return self.status
        return call


@pytest.fixture
def rec(monkeypatch):
    if not os.path.exists(_lib.LIB_PATH):
        from exact_tiled_attention_42_b200.build import build
        build()
    r = Recorder(_lib.load())
    monkeypatch.setattr(_lib, "load", lambda: r)
    monkeypatch.setattr(api, "_is_gpu", lambda t: True)
    return r


def z(*shape, dtype=BF):
    return torch.zeros(shape, dtype=dtype)


def ptrs(*ts):
    return tuple(t.data_ptr() for t in ts)


def dense(d=D, n=N):
    return {"q": z(B, HQ, n, d), "k": z(B, HKV, n, d), "v": z(B, HKV, n, d), "o": z(B, HQ, n, d),
            "lse": z(B, HQ, n, dtype=F32), "do": z(B, HQ, n, d)}


def packed():
    T = 2 * N
    return {"q": z(T, HQ, D), "k": z(T, HKV, D), "v": z(T, HKV, D), "o": z(T, HQ, D), "lse": z(HQ, T, dtype=F32),
            "do": z(T, HQ, D), "cu": torch.tensor([0, N, T], dtype=torch.int32)}


# entry point -> (call(**outputs), {output name: a correct tensor of it})
def entries():
    x, x8, p = dense(), dense(128), packed()
    T = 2 * N
    ws8 = torch.zeros(fa.fa_fp8_workspace_size(B, HQ, HKV, N, 128), dtype=torch.uint8)
    return {
        "fa_fwd": (lambda **kw: fa.fa_fwd(x["q"], x["k"], x["v"], stream=0, **kw),
                   {"out": z(B, HQ, N, D), "lse": z(B, HQ, N, dtype=F32)}),
        "fa_bwd": (lambda **kw: fa.fa_bwd(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"], stream=0, **kw),
                   {"dq": z(B, HQ, N, D), "dk": z(B, HKV, N, D), "dv": z(B, HKV, N, D),
                    "workspace": torch.zeros(fa.fa_bwd_workspace_size(B, HQ, HKV, N, D), dtype=torch.uint8)}),
        "fa_bwd_noalloc": (lambda **kw: fa.fa_bwd_noalloc(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"],
                                                          stream=0, **kw),
                           {"dq": z(B, HQ, N, D), "dk": z(B, HKV, N, D), "dv": z(B, HKV, N, D)}),
        "fa_fwd_fp8": (lambda **kw: fa.fa_fwd_fp8(x8["q"], x8["k"], x8["v"], stream=0, **kw),
                       {"out": z(B, HQ, N, 128), "lse": z(B, HQ, N, dtype=F32),
                        "workspace": torch.zeros(fa.fa_fp8_workspace_size(B, HQ, HKV, N, 128), dtype=torch.uint8)}),
        "fa_fwd_mxfp8": (lambda **kw: fa.fa_fwd_mxfp8(x8["q"], x8["k"], x8["v"], stream=0, **kw),
                         {"out": z(B, HQ, N, 128), "lse": z(B, HQ, N, dtype=F32),
                          "workspace": torch.zeros(fa.fa_mxfp8_workspace_size(B, HQ, HKV, N, 128),
                                                   dtype=torch.uint8)}),
        "fa_fp8_quantize": (lambda **kw: fa.fa_fp8_quantize(x8["q"], x8["k"], x8["v"], stream=0, **kw),
                            {"workspace": torch.zeros(ws8.numel(), dtype=torch.uint8)}),
        "fa_fwd_fp8_quantized": (lambda **kw: fa.fa_fwd_fp8_quantized(ws8, (B, HQ, HKV, N, 128), stream=0, **kw),
                                 {"out": z(B, HQ, N, 128), "lse": z(B, HQ, N, dtype=F32)}),
        "fa_fwd_decode": (lambda **kw: fa.fa_fwd_decode(z(B, HQ, 1, D), x["k"], x["v"], causal=True, stream=0, **kw),
                          {"out": z(B, HQ, 1, D), "lse": z(B, HQ, 1, dtype=F32),
                           "workspace": torch.zeros(fa.fa_decode_workspace_size(B, HQ, HKV, 1, N, D, 0),
                                                    dtype=torch.uint8)}),
        "fa_fwd_varlen": (lambda **kw: fa.fa_fwd_varlen(p["q"], p["k"], p["v"], p["cu"], max_seqlen=N, stream=0,
                                                        **kw),
                          {"out": z(T, HQ, D), "lse": z(HQ, T, dtype=F32)}),
        "fa_bwd_varlen": (lambda **kw: fa.fa_bwd_varlen(p["q"], p["k"], p["v"], p["o"], p["lse"], p["do"], p["cu"],
                                                        max_seqlen=N, stream=0, **kw),
                          {"dq": z(T, HQ, D), "dk": z(T, HKV, D), "dv": z(T, HKV, D),
                           "workspace": torch.zeros(fa.fa_bwd_varlen_workspace_size(2, HQ, HKV, T, N, D),
                                                    dtype=torch.uint8)}),
    }


ENTRY_POINTS = sorted(entries())
OUTPUTS = [(e, o) for e, (_, outs) in sorted(entries().items()) for o in sorted(outs)]


@pytest.mark.parametrize("entry", ENTRY_POINTS)
def test_every_entry_point_marshals_its_declared_signature(rec, entry):
    call, outs = entries()[entry]
    call()                       # outputs and workspace allocated by the binding
    call(**outs)                 # the caller's
    assert [c[0] for c in rec.calls] == [entry, entry]
    args = rec.calls[1][1]
    for t in outs.values():      # the caller's buffers reach the library
        assert t.data_ptr() in args


@pytest.mark.parametrize("entry,name", OUTPUTS)
def test_wrong_output_or_workspace_raises_before_the_call(rec, entry, name):
    call, outs = entries()[entry]
    good = outs[name]
    n = good.numel()
    bad = {
        "non-contiguous": torch.zeros(2 * n, dtype=good.dtype)[::2],
        "other device": torch.empty(good.shape, dtype=good.dtype, device="meta"),
    }
    if name != "workspace":
        bad["wrong shape"] = torch.zeros((good.shape[0] + 1,) + tuple(good.shape[1:]), dtype=good.dtype)
        bad["wrong dtype"] = torch.zeros(good.shape, dtype=F32 if good.dtype == BF else BF)
        bad["non-contiguous"] = torch.zeros(tuple(good.shape) + (2,), dtype=good.dtype)[..., 0]
    assert not bad["non-contiguous"].is_contiguous()
    for what, t in bad.items():
        with pytest.raises((ValueError, TypeError)):
            call(**{**outs, name: t})
        assert rec.calls == [], f"{entry}: {name} {what} reached the library"


def test_fwd_argument_order(rec):
    x = dense()
    o, lse = fa.fa_fwd(x["q"], x["k"], x["v"], causal=True, stream=0)
    name, args = rec.calls[0]
    assert name == "fa_fwd"
    assert args[:5] == ptrs(x["q"], x["k"], x["v"], o, lse)
    assert args[5:11] == (B, HQ, HKV, N, D, 1)
    assert args[11] == pytest.approx(D ** -0.5) and args[12] == 0
    assert o.shape == (B, HQ, N, D) and o.dtype == BF and lse.shape == (B, HQ, N) and lse.dtype == F32


def test_bwd_workspace_bytes_from_any_dtype(rec):
    x = dense()
    n = fa.fa_bwd_workspace_size(B, HQ, HKV, N, D)
    ws = torch.zeros(n // 4, dtype=F32)
    dq, dk, dv = fa.fa_bwd(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"], workspace=ws, scale=0.5, stream=0)
    _, args = rec.calls[0]
    assert args[:10] == ptrs(x["q"], x["k"], x["v"], x["o"], x["lse"], x["do"], dq, dk, dv, ws)
    assert args[10] == n and args[11:17] == (B, HQ, HKV, N, D, 0) and args[17] == 0.5


def test_fp8_and_mx_arguments(rec):
    x = dense(128)
    fa.fa_fwd_fp8(x["q"], x["k"], x["v"], rotation_seed=-1, use_rotation=False, stream=0)
    _, args = rec.calls[0]
    assert args[5] == 2 ** 64 - 1 and args[6] == 0      # the seed as its 64-bit pattern; rotation off
    for rule, code in sorted(api.MX_SCALE_RULES.items()):
        fa.fa_fwd_mxfp8(x["q"], x["k"], x["v"], scale_rule=rule, stream=0)
        assert rec.calls[-1][1][7] == code
    with pytest.raises(ValueError):
        fa.fa_fwd_mxfp8(x["q"], x["k"], x["v"], scale_rule="round", stream=0)


def test_decode_and_varlen_sizes(rec):
    x, p = dense(), packed()
    q1 = z(B, HQ, 3, D)
    fa.fa_fwd_decode(q1, x["k"], x["v"], causal=True, num_ctas=5, stream=0)
    _, args = rec.calls[-1]
    assert args[7:14] == (B, HQ, HKV, 3, N, D, 1) and args[15] == 5
    fa.fa_fwd_varlen(p["q"], p["k"], p["v"], p["cu"], max_seqlen=N, causal=True, stream=0)
    _, args = rec.calls[-1]
    assert args[5] == p["cu"].data_ptr() and args[6:13] == (2, HQ, HKV, 2 * N, N, D, 1)


@pytest.mark.parametrize("cu", [torch.tensor([0, 8, 16], dtype=torch.int64), torch.zeros((1, 3), dtype=torch.int32),
                                torch.zeros(0, dtype=torch.int32), torch.zeros(6, dtype=torch.int32)[::2]])
def test_bad_offsets_tensor_raises(rec, cu):
    p = packed()
    with pytest.raises(TypeError):
        fa.fa_fwd_varlen(p["q"], p["k"], p["v"], cu, max_seqlen=N, stream=0)
    assert rec.calls == []


def test_inputs_on_another_device_raise(rec):
    x = dense()
    with pytest.raises(ValueError):
        fa.fa_fwd(x["q"], torch.empty(x["k"].shape, dtype=BF, device="meta"), x["v"], stream=0)
    assert rec.calls == []


def test_library_status_raises_named_error(rec):
    x = dense()
    rec.status = 4
    with pytest.raises(fa.FAError, match=r"fa_fwd returned FA_ERR_WORKSPACE \(4\)"):
        fa.fa_fwd(x["q"], x["k"], x["v"], stream=0)


def test_every_compute_entry_point_is_covered():
    compute = {n for n in _lib.SIGNATURES
               if not n.endswith("_workspace_size") and n not in ("fa_status_string", "fa_last_device_status")}
    assert compute == set(ENTRY_POINTS)


def test_quantized_forward_checks_its_workspace(rec):
    n = fa.fa_fp8_workspace_size(B, HQ, HKV, N, 128)
    with pytest.raises(ValueError):   # the workspace sets the call's device; out and lse must be on it
        fa.fa_fwd_fp8_quantized(torch.zeros(2 * n, dtype=torch.uint8)[::2], (B, HQ, HKV, N, 128), stream=0)
    assert rec.calls == []
