"""Same-named Python entry points over the C ABI (argument marshalling only)."""

from __future__ import annotations

import math

import torch

from . import _lib

FA_OK = 0


class FAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {fa_status_string(status)} ({status})")


def fa_status_string(status: int) -> str:
    return _lib.load().fa_status_string(int(status)).decode()


def fa_last_device_status() -> int:
    """Device status word (0 = no kernel gave up on a bounded wait); clears it."""
    return int(_lib.load().fa_last_device_status())


def fa_bwd_workspace_size(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    return int(_lib.load().fa_bwd_workspace_size(B, Hq, Hkv, N, d))


def fa_fp8_workspace_size(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    return int(_lib.load().fa_fp8_workspace_size(B, Hq, Hkv, N, d))


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _is_gpu(t: torch.Tensor) -> bool:
    return t.is_cuda


def _check(name: str, t: torch.Tensor, dtype, shape, device=None) -> None:
    """Every tensor handed to the library is a contiguous CUDA tensor of the
    documented dtype and shape, on the device of the call's first input: the
    kernels index it by that shape alone."""
    if not isinstance(t, torch.Tensor) or not _is_gpu(t):
        raise TypeError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace_bytes(ws: torch.Tensor, device) -> int:
    """Size in bytes of a caller's workspace (any dtype; contiguous, on the
    call's device). The library checks it against the size it needs."""
    if not isinstance(ws, torch.Tensor) or not _is_gpu(ws):
        raise TypeError("workspace must be a CUDA tensor")
    if ws.device != device:
        raise ValueError(f"workspace is on {ws.device}, expected {device}")
    if not ws.is_contiguous():
        raise ValueError("workspace must be contiguous")
    return ws.numel() * ws.element_size()


def _dims(q, k):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, H, N, d]")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    return B, Hq, Hkv, N, d


def fa_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None, stream=None):
    """O, LSE = attention(q, k, v). q [B,Hq,N,d], k/v [B,Hkv,N,d] bf16 (CUDA);
    returns O bf16 [B,Hq,N,d] and LSE float32 [B,Hq,N]."""
    B, Hq, Hkv, N, d = _dims(q, k)
    _check("q", q, torch.bfloat16, (B, Hq, N, d))
    _check("k", k, torch.bfloat16, (B, Hkv, N, d), q.device)
    _check("v", v, torch.bfloat16, (B, Hkv, N, d), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _check("out", out, torch.bfloat16, (B, Hq, N, d), q.device)
    _check("lse", lse, torch.float32, (B, Hq, N), q.device)
    st = _lib.load().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                            B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream))
    if st != FA_OK:
        raise FAError("fa_fwd", st)
    return out, lse


def fa_bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
           dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of attention(q, k, v) against dout, recomputing P from lse."""
    B, Hq, Hkv, N, d = _dims(q, k)
    for name, t, shp in (("q", q, (B, Hq, N, d)), ("k", k, (B, Hkv, N, d)), ("v", v, (B, Hkv, N, d)),
                         ("o", o, (B, Hq, N, d)), ("dout", dout, (B, Hq, N, d))):
        _check(name, t, torch.bfloat16, shp, q.device)
    _check("lse", lse, torch.float32, (B, Hq, N), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check("dq", dq, torch.bfloat16, (B, Hq, N, d), q.device)
    _check("dk", dk, torch.bfloat16, (B, Hkv, N, d), q.device)
    _check("dv", dv, torch.bfloat16, (B, Hkv, N, d), q.device)
    if workspace is None:
        workspace = torch.empty(fa_bwd_workspace_size(B, Hq, Hkv, N, d), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace_bytes(workspace, q.device)
    st = _lib.load().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                            dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                            workspace.data_ptr(), ws_bytes,
                            B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream))
    if st != FA_OK:
        raise FAError("fa_bwd", st)
    return dq, dk, dv


def fa_bwd_noalloc(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
                   dq=None, dk=None, dv=None, stream=None):
    """fa_bwd without a workspace argument: the library's built-in scratch
    (at most FA_BWD_NOALLOC_MAX_BYTES) is used instead. For callers that
    cannot allocate device memory at the call; calls that may run
    concurrently on the GPU must be serialised because they share the
    scratch."""
    B, Hq, Hkv, N, d = _dims(q, k)
    for name, t, shp in (("q", q, (B, Hq, N, d)), ("k", k, (B, Hkv, N, d)), ("v", v, (B, Hkv, N, d)),
                         ("o", o, (B, Hq, N, d)), ("dout", dout, (B, Hq, N, d))):
        _check(name, t, torch.bfloat16, shp, q.device)
    _check("lse", lse, torch.float32, (B, Hq, N), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check("dq", dq, torch.bfloat16, (B, Hq, N, d), q.device)
    _check("dk", dk, torch.bfloat16, (B, Hkv, N, d), q.device)
    _check("dv", dv, torch.bfloat16, (B, Hkv, N, d), q.device)
    st = _lib.load().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                    dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                    B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream))
    if st != FA_OK:
        raise FAError("fa_bwd_noalloc", st)
    return dq, dk, dv


def fa_fwd_fp8(q, k, v, causal: bool = False, scale: float | None = None, rotation_seed: int = 0,
               use_rotation: bool = True, out=None, lse=None, workspace=None, stream=None):
    """FP8 (e4m3) forward with 64-row block scales and optional Hadamard
    rotation of Q and K; bf16 inputs and output."""
    B, Hq, Hkv, N, d = _dims(q, k)
    _check("q", q, torch.bfloat16, (B, Hq, N, d))
    _check("k", k, torch.bfloat16, (B, Hkv, N, d), q.device)
    _check("v", v, torch.bfloat16, (B, Hkv, N, d), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check("out", out, torch.bfloat16, (B, Hq, N, d), q.device)
    _check("lse", lse, torch.float32, (B, Hq, N), q.device)
    if workspace is None:
        workspace = torch.empty(fa_fp8_workspace_size(B, Hq, Hkv, N, d), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace_bytes(workspace, q.device)
    st = _lib.load().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                int(rotation_seed) & 0xFFFFFFFFFFFFFFFF, int(bool(use_rotation)),
                                workspace.data_ptr(), ws_bytes,
                                B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream))
    if st != FA_OK:
        raise FAError("fa_fwd_fp8", st)
    return out, lse


def fa_mxfp8_workspace_size(B: int, Hq: int, Hkv: int, N: int, d: int) -> int:
    return int(_lib.load().fa_mxfp8_workspace_size(B, Hq, Hkv, N, d))


MX_SCALE_RULES = {"ocp": 0, "fit": 1}


def fa_fwd_mxfp8(q, k, v, causal: bool = False, scale: float | None = None, rotation_seed: int = 0,
                 use_rotation: bool = True, scale_rule: str = "fit", out=None, lse=None, workspace=None,
                 stream=None):
    """MXFP8 forward (e4m3 with one E8M0 exponent per 32 elements along each
    product's contraction, applied by the tensor cores); bf16 inputs and
    output, d = 128. scale_rule "ocp" (the MX specification's exponent) or
    "fit" (one higher where that would saturate)."""
    B, Hq, Hkv, N, d = _dims(q, k)
    _check("q", q, torch.bfloat16, (B, Hq, N, d))
    _check("k", k, torch.bfloat16, (B, Hkv, N, d), q.device)
    _check("v", v, torch.bfloat16, (B, Hkv, N, d), q.device)
    if scale_rule not in MX_SCALE_RULES:
        raise ValueError(f"scale_rule must be one of {sorted(MX_SCALE_RULES)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check("out", out, torch.bfloat16, (B, Hq, N, d), q.device)
    _check("lse", lse, torch.float32, (B, Hq, N), q.device)
    if workspace is None:
        workspace = torch.empty(fa_mxfp8_workspace_size(B, Hq, Hkv, N, d), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace_bytes(workspace, q.device)
    st = _lib.load().fa_fwd_mxfp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  int(rotation_seed) & 0xFFFFFFFFFFFFFFFF, int(bool(use_rotation)),
                                  MX_SCALE_RULES[scale_rule], workspace.data_ptr(), ws_bytes,
                                  B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream))
    if st != FA_OK:
        raise FAError("fa_fwd_mxfp8", st)
    return out, lse


def fa_fp8_quantize(q, k, v, rotation_seed: int = 0, use_rotation: bool = True, workspace=None, stream=None):
    """The FP8 pre-pass alone: rotated (optional) and 64-row block-quantised
    e4m3 copies of q, k, v with their scales, in a workspace (uint8 tensor)
    that fa_fwd_fp8_quantized reads."""
    B, Hq, Hkv, N, d = _dims(q, k)
    _check("q", q, torch.bfloat16, (B, Hq, N, d))
    _check("k", k, torch.bfloat16, (B, Hkv, N, d), q.device)
    _check("v", v, torch.bfloat16, (B, Hkv, N, d), q.device)
    if workspace is None:
        workspace = torch.empty(max(fa_fp8_workspace_size(B, Hq, Hkv, N, d), 16), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace_bytes(workspace, q.device)
    st = _lib.load().fa_fp8_quantize(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                     int(rotation_seed) & 0xFFFFFFFFFFFFFFFF, int(bool(use_rotation)),
                                     workspace.data_ptr(), ws_bytes,
                                     B, Hq, Hkv, N, d, _stream(stream))
    if st != FA_OK:
        raise FAError("fa_fp8_quantize", st)
    return workspace


def fa_fwd_fp8_quantized(workspace, shape, causal: bool = False, scale: float | None = None,
                         use_rotation: bool = True, out=None, lse=None, stream=None):
    """The FP8 forward from a workspace filled by fa_fp8_quantize;
    shape = (B, Hq, Hkv, N, d) of the quantised tensors."""
    B, Hq, Hkv, N, d = (int(x) for x in shape)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = workspace.device
    ws_bytes = _workspace_bytes(workspace, dev)
    out = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=dev) if out is None else out
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev) if lse is None else lse
    _check("out", out, torch.bfloat16, (B, Hq, N, d), dev)
    _check("lse", lse, torch.float32, (B, Hq, N), dev)
    st = _lib.load().fa_fwd_fp8_quantized(workspace.data_ptr(), ws_bytes,
                                          out.data_ptr(), lse.data_ptr(), int(bool(use_rotation)),
                                          B, Hq, Hkv, N, d, int(bool(causal)), float(scale), _stream(stream))
    if st != FA_OK:
        raise FAError("fa_fwd_fp8_quantized", st)
    return out, lse


def fa_decode_workspace_size(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, num_ctas: int = 0) -> int:
    return int(_lib.load().fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_ctas))


def fa_fwd_decode(q, k, v, causal: bool = False, scale: float | None = None, num_ctas: int = 0,
                  out=None, lse=None, workspace=None, stream=None):
    """O, LSE for Nq query rows [B,Hq,Nq,d] against k/v [B,Hkv,Nk,d] (bf16).
    The (KV head, key tile) pairs are shared evenly by ``num_ctas`` CTAs (0 =
    as many as fit on the GPU) and the partial results merged by log-sum-exp."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, H, N, d]")
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    _check("q", q, torch.bfloat16, (B, Hq, Nq, d))
    _check("k", k, torch.bfloat16, (B, Hkv, Nk, d), q.device)
    _check("v", v, torch.bfloat16, (B, Hkv, Nk, d), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check("out", out, torch.bfloat16, (B, Hq, Nq, d), q.device)
    _check("lse", lse, torch.float32, (B, Hq, Nq), q.device)
    if workspace is None:
        n = fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_ctas)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace_bytes(workspace, q.device)
    st = _lib.load().fa_fwd_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                   workspace.data_ptr(), ws_bytes,
                                   B, Hq, Hkv, Nq, Nk, d, int(bool(causal)), float(scale), int(num_ctas),
                                   _stream(stream))
    if st != FA_OK:
        raise FAError("fa_fwd_decode", st)
    return out, lse


def _varlen_dims(q, k, cu_seqlens):
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("packed q and k must be [T, H, d]")
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    if not isinstance(cu_seqlens, torch.Tensor) or not _is_gpu(cu_seqlens) or cu_seqlens.dtype != torch.int32 \
            or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1 or not cu_seqlens.is_contiguous():
        raise TypeError("cu_seqlens must be a contiguous int32 CUDA tensor of B + 1 offsets")
    if cu_seqlens.device != q.device:
        raise ValueError(f"cu_seqlens is on {cu_seqlens.device}, expected {q.device}")
    return cu_seqlens.numel() - 1, T, Hq, Hkv, d


def fa_fwd_varlen(q, k, v, cu_seqlens, max_seqlen: int, causal: bool = False, scale: float | None = None,
                  out=None, lse=None, stream=None):
    """Packed variable-length batch: q [T, Hq, d], k/v [T, Hkv, d] bf16,
    sequence b = tokens cu_seqlens[b]..cu_seqlens[b+1]-1 (int32 CUDA tensor),
    max_seqlen >= every length. Returns O [T, Hq, d] bf16, LSE [Hq, T] fp32."""
    B, T, Hq, Hkv, d = _varlen_dims(q, k, cu_seqlens)
    _check("q", q, torch.bfloat16, (T, Hq, d))
    _check("k", k, torch.bfloat16, (T, Hkv, d), q.device)
    _check("v", v, torch.bfloat16, (T, Hkv, d), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((Hq, T), dtype=torch.float32, device=q.device) if lse is None else lse
    _check("out", out, torch.bfloat16, (T, Hq, d), q.device)
    _check("lse", lse, torch.float32, (Hq, T), q.device)
    st = _lib.load().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                   cu_seqlens.data_ptr(), B, Hq, Hkv, T, int(max_seqlen), d, int(bool(causal)),
                                   float(scale), _stream(stream))
    if st != FA_OK:
        raise FAError("fa_fwd_varlen", st)
    return out, lse


def fa_bwd_varlen_workspace_size(B: int, Hq: int, Hkv: int, total: int, max_seqlen: int, d: int) -> int:
    return int(_lib.load().fa_bwd_varlen_workspace_size(B, Hq, Hkv, total, max_seqlen, d))


def fa_bwd_varlen(q, k, v, o, lse, dout, cu_seqlens, max_seqlen: int, causal: bool = False,
                  scale: float | None = None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of a packed variable-length batch (layouts of fa_fwd_varlen)."""
    B, T, Hq, Hkv, d = _varlen_dims(q, k, cu_seqlens)
    for name, t, shp in (("q", q, (T, Hq, d)), ("k", k, (T, Hkv, d)), ("v", v, (T, Hkv, d)),
                         ("o", o, (T, Hq, d)), ("dout", dout, (T, Hq, d))):
        _check(name, t, torch.bfloat16, shp, q.device)
    _check("lse", lse, torch.float32, (Hq, T), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check("dq", dq, torch.bfloat16, (T, Hq, d), q.device)
    _check("dk", dk, torch.bfloat16, (T, Hkv, d), q.device)
    _check("dv", dv, torch.bfloat16, (T, Hkv, d), q.device)
    if workspace is None:
        n = fa_bwd_varlen_workspace_size(B, Hq, Hkv, T, int(max_seqlen), d)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = _workspace_bytes(workspace, q.device)
    st = _lib.load().fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                   dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cu_seqlens.data_ptr(),
                                   workspace.data_ptr(), ws_bytes,
                                   B, Hq, Hkv, T, int(max_seqlen), d, int(bool(causal)), float(scale), _stream(stream))
    if st != FA_OK:
        raise FAError("fa_bwd_varlen", st)
    return dq, dk, dv
