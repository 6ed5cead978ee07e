"""The CUDA path's Philox4x32-10 (csrc/philox.cuh) against the generator's
published known answers, compiled for the host with nvcc (no GPU needed).

The header is the product's own code: its host build differs only in how the
high half of a 32 x 32-bit product is taken.  The oracle implements the same
generator separately (oracle/masked.py); the two share nothing.
"""
import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_54_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include "philox.cuh"
int main(int argc, char** argv) {
  unsigned v[6];
  while (std::scanf("%x %x %x %x %x %x", &v[0], &v[1], &v[2], &v[3], &v[4], &v[5]) == 6) {
    const uint4 r = fa::philox4x32_10(make_uint4(v[0], v[1], v[2], v[3]), v[4], v[5]);
    std::printf("%08x %08x %08x %08x\n", r.x, r.y, r.z, r.w);
  }
  return 0;
}
"""


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


def test_device_philox_known_answers(tmp_path, golden_dir):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not found")
    src = tmp_path / "kat.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "kat"
    subprocess.run([nvcc, "-std=c++17", "-I", CSRC, "-o", str(exe), str(src)], check=True, capture_output=True)
    with open(os.path.join(golden_dir, "philox4x32_10_kat.json")) as f:
        kat = json.load(f)
    lines = "".join(" ".join(vec["counter"] + vec["key"]) + "\n" for vec in kat["vectors"])
    out = subprocess.run([str(exe)], input=lines, capture_output=True, text=True, check=True).stdout.split("\n")
    for vec, got in zip(kat["vectors"], out):
        assert got.split() == vec["out"]
