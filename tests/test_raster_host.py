"""The forwards' grid order groups query heads so that a group's K and V
(about 32 MiB, a quarter of L2) stay in L2 while its CTAs run
(``raster_heads_for`` in csrc/kernels.h, host code). Compiled here with the
host compiler and checked on the workloads' sizes: heads per group = 32 MiB
over the K/V bytes per query head, at least 1, at most every head."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_tiled_attention_42_b200", "csrc")

# (B*Hq, Hq/Hkv, K+V bytes per KV head, heads per group)
CASES = [
    (32, 1, 2 * 8192 * 128 * 2, 8),       # long128: 4 MiB of bf16 K/V per head
    (64, 4, 2 * 8192 * 128 * 2, 32),      # gqa 32/8: four query heads share a KV head
    (128, 1, 2 * 2048 * 64 * 2, 64),      # gpt2: 0.5 MiB per head
    (16, 1, 2 * 16384 * 128, 8),          # the FP8 workload: e4m3 K and V
    (2, 1, 2 * 128 * 64 * 2, 2),          # tiny: every head in one group
    (3, 1, 1 << 40, 1),                   # a head larger than the budget: groups of one
    (7, 7, 7 << 20, 7),                   # one KV head shared by all: all heads
]


@pytest.fixture(scope="module")
def raster_heads_for(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    d = tmp_path_factory.mktemp("raster")
    src, exe = d / "r.cpp", d / "r"
    src.write_text('#include "kernels.h"\n#include <cstdio>\n#include <cstdlib>\n'
                   "int main(int argc, char** argv) {\n"
                   "  for (int i = 1; i + 2 < argc; i += 3)\n"
                   "    std::printf(\"%d\\n\", fa::raster_heads_for(std::atoll(argv[i]), std::atoi(argv[i + 1]),"
                   " std::atoll(argv[i + 2])));\n}\n")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    r = subprocess.run([cxx, "-std=c++17", "-I" + CSRC, "-I" + os.path.join(ROOT, "include"), "-I" + cuda_inc,
                        str(src), "-o", str(exe)], capture_output=True, text=True)
    if r.returncode != 0:
        pytest.skip("kernels.h does not compile as host C++ here: " + r.stderr[:200])

    def call(cases):
        args = [str(x) for c in cases for x in c[:3]]
        out = subprocess.run([str(exe), *args], capture_output=True, text=True, check=True).stdout
        return [int(x) for x in out.split()]
    return call


def test_group_sizes_on_the_workloads(raster_heads_for):
    assert raster_heads_for(CASES) == [c[3] for c in CASES]


def test_groups_stay_within_one_and_every_head(raster_heads_for):
    cases = [(bh, g, b) for bh in (1, 5, 64, 4096) for g in (1, 2, 8) for b in (0, 1, 1 << 20, 1 << 25, 1 << 36)]
    for (bh, _, _), got in zip(cases, raster_heads_for(cases)):
        assert 1 <= got <= bh
