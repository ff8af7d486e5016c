"""The C-ABI library: it loads, exports every symbol include/fa.h declares,
and rejects bad arguments on the host before launching anything (no GPU
needed for any of these)."""

import ctypes
import json
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    from exact_tiled_attention_42_b200 import _lib
    if not os.path.exists(_lib.LIB_PATH):
        from exact_tiled_attention_42_b200.build import build
        build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:fa_status|size_t|const char\*|int)\s+(fa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_fwd_fp8", "fa_fp8_workspace_size",
                 "fa_fwd_mxfp8", "fa_mxfp8_workspace_size", "fa_status_string", "fa_last_device_status"):
        assert need in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib._name)
    for name in declared_functions():
        assert hasattr(raw, name), name


def test_binding_covers_every_declared_symbol():
    from exact_tiled_attention_42_b200 import _lib
    assert set(declared_functions()) <= set(_lib.SIGNATURES)


def test_status_strings(lib):
    assert lib.fa_status_string(0) == b"FA_OK"
    assert lib.fa_status_string(6) == b"FA_ERR_TIMEOUT"
    assert lib.fa_status_string(99) == b"FA_ERR_UNKNOWN"


P = 0x100000   # an aligned fake device address; never dereferenced by these calls


def fwd(lib, q=P, k=P, v=P, o=P, lse=P, B=1, Hq=2, Hkv=2, N=128, d=64, causal=0, scale=0.125):
    return lib.fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, None)


def test_fwd_rejects_bad_arguments(lib):
    assert fwd(lib, q=None) == 1
    assert fwd(lib, lse=None) == 1
    assert fwd(lib, N=0) == 1
    assert fwd(lib, B=0) == 1
    assert fwd(lib, Hq=3, Hkv=2) == 1
    assert fwd(lib, scale=0.0) == 1
    assert fwd(lib, scale=-1.0) == 1
    assert fwd(lib, scale=float("inf")) == 1
    assert fwd(lib, scale=float("nan")) == 1
    assert fwd(lib, d=80) == 2
    assert fwd(lib, d=112) == 2
    assert fwd(lib, d=320) == 2
    assert fwd(lib, d=160) == 2
    assert fwd(lib, B=65536, Hq=256, Hkv=256, N=16384) == 2  # grid of more than 2^31 - 1 CTAs
    assert fwd(lib, q=P + 8) == 3
    assert fwd(lib, lse=P + 4) == 3


def test_bwd_rejects_bad_arguments(lib):
    ws = lib.fa_bwd_workspace_size(1, 2, 2, 128, 64)
    def bwd(ws_ptr=P, ws_bytes=ws, d=64, dq=P):
        return lib.fa_bwd(P, P, P, P, P, P, dq, P, P, ws_ptr, ws_bytes, 1, 2, 2, 128, d, 0, 0.125, None)
    assert bwd(dq=None) == 1
    assert bwd(d=80) == 2
    assert bwd(d=192) == 2   # the wide-head kernels are forward only
    assert bwd(d=256) == 2
    assert bwd(ws_ptr=None) == 4
    assert bwd(ws_bytes=ws - 1) == 4
    assert bwd(dq=P + 2) == 3


def test_bwd_noalloc_reports_argument_errors_before_its_size_limit(lib):
    """fa_bwd_noalloc checks arguments in fa_bwd's order before the size of
    its built-in scratch: a call that is too large and also wrong in another
    way reports the other error. Sizes: 2 x 32 heads x 8192 rows x 128 needs
    far more than FA_BWD_NOALLOC_MAX_BYTES."""
    big = (2, 32, 8, 8192, 128)
    def nb(dq=P, scale=0.088, sizes=big):
        return lib.fa_bwd_noalloc(P, P, P, P, P, P, dq, P, P, *sizes, 1, scale, None)
    assert lib.fa_bwd_workspace_size(*big) > 32 * 1024 * 1024
    assert nb(dq=None) == 1                    # null pointer
    assert nb(scale=0.0) == 1                  # bad scale
    assert nb(scale=float("nan")) == 1
    assert nb(sizes=(2, 33, 8, 8192, 128)) == 1  # Hq % Hkv != 0
    assert nb(sizes=(2, 32, 8, 8192, 80)) == 2   # head dimension
    assert nb(dq=P + 2) == 3                   # misaligned
    assert nb() == 4                           # only then: larger than the built-in scratch
    # the limit is exact: 2 x 64 heads x 992 rows x 64 needs exactly 32 MiB
    # (launching would need a GPU, so only the size query is checked here)
    assert lib.fa_bwd_workspace_size(2, 64, 16, 992, 64) == 32 * 1024 * 1024
    assert lib.fa_bwd_workspace_size(1, 129, 129, 992, 64) > 32 * 1024 * 1024


def test_varlen_rejects_bad_arguments(lib):
    """Host-side checks of the packed entry points (the offsets themselves
    live on the device and are checked by the kernels)."""
    def fv(cu=P, B=2, Hq=2, Hkv=2, T=300, maxlen=200, d=64, lse=P, scale=0.125):
        return lib.fa_fwd_varlen(P, P, P, P, lse, cu, B, Hq, Hkv, T, maxlen, d, 1, scale, None)
    assert fv(cu=None) == 1
    assert fv(lse=None) == 1
    assert fv(T=-1) == 1
    assert fv(Hq=3) == 1
    assert fv(d=80) == 2
    assert fv(scale=0.0) == 1
    assert fv(cu=P + 2) == 3                  # offsets must be 4-byte aligned
    assert fv(T=0) == 0 and fv(maxlen=0) == 0  # every sequence empty: nothing to do
    ws = lib.fa_bwd_varlen_workspace_size(2, 2, 2, 300, 200, 64)
    assert ws > 0
    def bv(wsp=P, ws_bytes=ws, cu=P, d=64):
        return lib.fa_bwd_varlen(P, P, P, P, P, P, P, P, P, cu, wsp, ws_bytes, 2, 2, 2, 300, 200, d, 1, 0.125, None)
    assert bv(cu=None) == 1
    assert bv(wsp=None) == 4
    assert bv(ws_bytes=ws - 1) == 4
    assert bv(d=80) == 2
    # linear in the tokens and in the longest sequence
    a = lib.fa_bwd_varlen_workspace_size(2, 2, 2, 4096, 2048, 128)
    b = lib.fa_bwd_varlen_workspace_size(2, 2, 2, 8192, 4096, 128)
    assert b <= 2 * a + 512


def test_fp8_rejects_bad_arguments(lib):
    ws = lib.fa_fp8_workspace_size(1, 2, 2, 128, 128)
    assert ws > 0
    assert lib.fa_fwd_fp8(P, P, P, P, P, 1, 1, None, ws, 1, 2, 2, 128, 128, 0, 0.1, None) == 4
    assert lib.fa_fwd_fp8(P, P, P, P, P, 1, 1, P, ws - 1, 1, 2, 2, 128, 128, 0, 0.1, None) == 4
    assert lib.fa_fwd_fp8(P, P, None, P, P, 1, 1, P, ws, 1, 2, 2, 128, 128, 0, 0.1, None) == 1
    # the two halves take the same checks
    assert lib.fa_fp8_quantize(P, P, P, 1, 1, None, ws, 1, 2, 2, 128, 128, None) == 4
    assert lib.fa_fp8_quantize(P, None, P, 1, 1, P, ws, 1, 2, 2, 128, 128, None) == 1
    assert lib.fa_fp8_quantize(P, P, P, 1, 1, P, ws, 1, 2, 2, 128, 64, None) == 2      # d = 64 not built
    assert lib.fa_fwd_fp8_quantized(P, ws - 1, P, P, 1, 1, 2, 2, 128, 128, 0, 0.1, None) == 4
    assert lib.fa_fwd_fp8_quantized(P, ws, None, P, 1, 1, 2, 2, 128, 128, 0, 0.1, None) == 1
    assert lib.fa_fwd_fp8_quantized(P, ws, P + 2, P, 1, 1, 2, 2, 128, 128, 0, 0.1, None) == 3
    assert lib.fa_fwd_fp8_quantized(P, ws, P, P, 1, 1, 3, 2, 128, 128, 0, 0.1, None) == 1  # Hq % Hkv


def test_mxfp8_rejects_bad_arguments(lib):
    ws = lib.fa_mxfp8_workspace_size(1, 2, 2, 300, 128)
    # codes 2*300*128 each (three regions), exponents Q and K 2*300*4 each, V 2*128*(4 per 96-key tile)
    up = lambda x: (x + 1023) // 1024 * 1024
    assert ws == 3 * up(2 * 300 * 128) + 2 * up(2 * 300 * 4) + up(2 * 128 * 4 * 4)
    assert lib.fa_mxfp8_workspace_size(1, 2, 2, 300, 64) == 0                 # d = 128 only
    def mx(q=P, rule=1, wsp=P, wsb=ws, Hq=2, d=128):
        return lib.fa_fwd_mxfp8(q, P, P, P, P, 7, 1, rule, wsp, wsb, 1, Hq, 2, 300, d, 0, 0.1, None)
    assert mx(q=None) == 1
    assert mx(d=64) == 2
    assert mx(rule=2) == 1
    assert mx(rule=-1) == 1
    assert mx(q=P + 8) == 3
    assert mx(wsp=None) == 4
    assert mx(wsb=ws - 1) == 4
    assert mx(wsp=P + 4) == 3
    assert mx(Hq=3) == 1                                                      # Hq % Hkv


def test_fp8_paths_reject_more_than_65535_query_heads(lib):
    """The pre-passes put B * Hq on a grid dimension of at most 65535."""
    for B, Hq in ((1, 65536), (2, 32768)):
        ws8 = lib.fa_fp8_workspace_size(B, Hq, 1, 1, 128)
        wsm = lib.fa_mxfp8_workspace_size(B, Hq, 1, 1, 128)
        assert ws8 > 0 and wsm > 0
        assert lib.fa_fwd_fp8(P, P, P, P, P, 7, 1, P, ws8, B, Hq, 1, 1, 128, 0, 0.1, None) == 2
        assert lib.fa_fp8_quantize(P, P, P, 7, 1, P, ws8, B, Hq, 1, 1, 128, None) == 2
        assert lib.fa_fwd_fp8_quantized(P, ws8, P, P, 1, B, Hq, 1, 1, 128, 0, 0.1, None) == 2
        assert lib.fa_fwd_mxfp8(P, P, P, P, P, 7, 1, 1, P, wsm, B, Hq, 1, 1, 128, 0, 0.1, None) == 2


def test_workspace_sizes_are_linear_in_n(lib):
    """The score matrix the pages size (4,096 tokens -> 16.7 million entries,
    128K -> 16.4 billion) is never stored: workspace grows linearly in N."""
    cases = json.load(open(os.path.join(ROOT, "tests", "golden", "score_matrix_sizes.json")))["cases"]
    for c in cases:
        n = c["tokens"]
        assert abs(n * n - c["entries"]) <= c["rel_tol"] * c["entries"]
        ws = lib.fa_bwd_workspace_size(1, 1, 1, n, 128)
        assert ws < 4 * n * n / 8, (n, ws)
    a = lib.fa_bwd_workspace_size(2, 8, 2, 4096, 128)
    b = lib.fa_bwd_workspace_size(2, 8, 2, 8192, 128)
    assert abs(b / a - 2.0) < 1e-3
    assert lib.fa_bwd_workspace_size(1, 3, 2, 128, 64) == 0
    f1 = lib.fa_fp8_workspace_size(1, 4, 4, 4096, 128)
    f2 = lib.fa_fp8_workspace_size(1, 4, 4, 8192, 128)
    assert abs(f2 / f1 - 2.0) < 1e-2


def test_decode_rejects_bad_arguments(lib):
    ws = lib.fa_decode_workspace_size(2, 8, 2, 1, 4096, 128, 0)
    assert ws > 0
    def dec(Hq=8, Hkv=2, Nq=1, Nk=4096, d=128, causal=1, ws_bytes=ws, wsp=P, q=P, ctas=0):
        return lib.fa_fwd_decode(q, P, P, P, P, wsp, ws_bytes, 2, Hq, Hkv, Nq, Nk, d, causal, 0.08, ctas, None)
    assert dec(q=None) == 1
    assert dec(Nq=8, Nk=4) == 1               # causal with more queries than keys
    assert dec(Hq=8, Hkv=1, Nq=4) == 2        # 32 query rows per KV head
    assert dec(d=96) == 2
    assert dec(wsp=None) == 4
    assert dec(ws_bytes=ws - 1) == 4
    assert dec(ctas=-1) == 1
    # an explicit CTA count needs room for its partials; the automatic one is
    # sized for at most 1024 CTAs, whatever the device
    assert lib.fa_decode_workspace_size(2, 8, 2, 1, 4096, 128, 7) < ws
    assert lib.fa_decode_workspace_size(2, 8, 2, 1, 4096, 128, 4096) == ws
    assert lib.fa_decode_workspace_size(2, 8, 1, 4, 4096, 128, 0) == 0
    # the workspace holds partial rows per split, not an Nq x Nk matrix
    assert lib.fa_decode_workspace_size(16, 32, 8, 1, 131072, 128, 0) < 64 * 2 ** 20


def test_decode_workspace_matches_the_documented_layout(lib):
    """slots = min(CTAs, units) + B*Hkv with the automatic CTA count sized for
    at most 1024; partial rows (d floats) then partial LSEs, each region rounded
    up to 256 bytes. Device independent, so it holds without a GPU."""
    up = lambda x: (x + 255) // 256 * 256
    for B, Hq, Hkv, Nq, Nk, d, ctas in [(16, 32, 8, 1, 16384, 128, 0), (1, 4, 1, 4, 100, 64, 0),
                                        (2, 8, 2, 2, 3000, 128, 7), (2, 8, 2, 2, 3000, 128, 100000),
                                        (64, 8, 8, 1, 64, 128, 0)]:
        R = (Hq // Hkv) * Nq
        units = B * Hkv * ((Nk + 63) // 64)
        slots = min(ctas if ctas > 0 else 1024, units) + B * Hkv
        assert lib.fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, ctas) == up(slots * R * d * 4) + up(slots * R * 4)


def test_header_is_plain_c_and_links(tmp_path):
    """include/fa.h compiles as C99 and a C program linked against the library
    sees the declared behaviour of the host-side entry points."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    from exact_tiled_attention_42_b200 import _lib
    cuda_inc = next((p for p in ("/usr/local/cuda/include",) if os.path.isdir(p)), None)
    if cuda_inc is None:
        pytest.skip("no CUDA headers")
    exe = tmp_path / "c_abi_check"
    libdir = os.path.dirname(_lib.LIB_PATH)
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe), "-L", libdir, "-l:libfa_b200.so",
           "-Wl,-rpath," + libdir]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
