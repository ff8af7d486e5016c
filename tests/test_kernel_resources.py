"""Register and local-memory use of every kernel, from the compiler's own
report (``ptxas -v``), with the product build's flags. No GPU needed.

* The warp-specialised kernels re-divide their registers at run time
  (``setmaxnreg``): the forwards give their two softmax warpgroups 208 and
  the third 88, which needs 168 per thread at launch (256 * 208 + 128 * 88 =
  384 * 168); the backward gives 136 / 152 / 88 to its compute, drain and
  load/MMA warpgroups, which needs 128 at launch (512 threads). The host
  refuses to launch if the compiled count is lower; this checks it at build
  time instead.
* No kernel spills or keeps a stack frame, except the packed-batch variants
  of the bf16 forward, for which the compiler reports a few bytes of spill
  (at most 16 bytes stored and 64 loaded per thread, a 16-byte stack frame);
  the limit here keeps that from growing."""

import concurrent.futures as cf
import glob
import os
import re
import subprocess

import pytest

from exact_tiled_attention_42_b200 import build

SPLIT_AT_LAUNCH = {"fwd_bf16_kernel": 168, "fwd_fp8_kernel": 168, "fwd_mxfp8_kernel": 168, "bwd_bf16_kernel": 128}
PACKED_FWD = re.compile(r"fwd_bf16_kernelILi\d+ELb[01]ELb1E")   # template <D, CAUSAL, VARLEN = true>
PACKED_LIMIT = {"stack": 16, "stores": 16, "loads": 64}


def _report(src, out_dir):
    obj = os.path.join(out_dir, os.path.basename(src) + ".o")
    cmd = [build._nvcc(), *build.ARCH, *build.FLAGS, "-Xptxas=-v", "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return r.stdout + r.stderr


@pytest.fixture(scope="module")
def kernels(tmp_path_factory):
    try:
        build._nvcc()
    except RuntimeError:
        pytest.skip("nvcc not available")
    out = str(tmp_path_factory.mktemp("ptxas"))
    srcs = sorted(glob.glob(os.path.join(build.CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=8) as ex:
        text = "".join(ex.map(lambda s: _report(s, out), srcs))
    found = {}
    for entry in re.split(r"ptxas info\s+: Compiling entry function '", text)[1:]:
        name = entry.split("'")[0]
        frame = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", entry)
        regs = re.search(r"Used (\d+) registers", entry)
        assert frame and regs, name
        found[name] = {"regs": int(regs.group(1)), "stack": int(frame.group(1)), "stores": int(frame.group(2)),
                       "loads": int(frame.group(3))}
    return found


def test_every_kernel_is_reported(kernels):
    for base in ("fwd_bf16_kernel", "fwd_wide_kernel", "fwd_fp8_kernel", "fwd_mxfp8_kernel", "bwd_bf16_kernel",
                 "bwd_pre_kernel", "bwd_post_kernel", "fp8_quant_kernel", "mxfp8_quant_kernel",
                 "decode_split_kernel", "decode_combine_kernel"):
        assert any(base in n for n in kernels), base


def test_register_splits_fit_the_launch_allocation(kernels):
    for base, need in SPLIT_AT_LAUNCH.items():
        got = [(n, k["regs"]) for n, k in kernels.items() if base in n]
        assert got, base
        for n, regs in got:
            assert regs >= need, f"{n}: {regs} registers at launch, the split needs {need}"


def test_no_spills_outside_the_packed_forward(kernels):
    for n, k in kernels.items():
        if PACKED_FWD.search(n):
            for key, limit in PACKED_LIMIT.items():
                assert k[key] <= limit, f"{n}: {key} {k[key]} bytes"
        else:
            assert k["stack"] == k["stores"] == k["loads"] == 0, f"{n}: {k}"
