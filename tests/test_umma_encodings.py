"""The tensor-core encodings of csrc/umma.cuh (host-callable helpers), compiled and run on the
host: the kind::f16 instruction descriptor of the MMA shapes the kernels issue, and the byte
offsets of the 128-byte swizzle.  The expected values are the hardware's field layout written
out by hand (D format fp32 = 1 at bit 4; A and B bf16 = 1 at bits 7 and 10; A / B MN-major at
bits 15 / 16; N / 8 from bit 17; M / 16 from bit 24) and the swizzle's definition (16-byte
chunk c of row r of an 8-row, 1024-byte atom at r * 128 + (c ^ r) * 16); these are the shapes
and layouts a one-CTA GPU probe checked against a CPU product before the kernels used them.
No GPU is needed."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "paged_block_sparse_vt_b200", "csrc", "umma.cuh")

PROGRAM = r"""
#include <cstdio>
#include "umma.cuh"
using namespace vt::umma;
int main() {
  std::printf("%u %u %u %u %u\n", idesc_bf16(64, 32, false, false), idesc_bf16(64, 16, false, false),
              idesc_bf16(128, 32, true, false), idesc_bf16(128, 16, true, false),
              idesc_bf16(128, 256, false, false));
  const int rc[6][2] = {{0, 0}, {0, 7}, {1, 0}, {7, 7}, {9, 3}, {63, 5}};
  for (int i = 0; i < 6; ++i) std::printf("%u ", sw128_off(rc[i][0], rc[i][1]));
  std::printf("\n");
  return 0;
}
"""


def _expected_idesc(M, N, a_mn, b_mn):
    return ((1 << 4) | (1 << 7) | (1 << 10) | (a_mn << 15) | (b_mn << 16) | ((N // 8) << 17)
            | ((M // 16) << 24))


def test_umma_encodings_on_host():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "enc.cu")
        exe = os.path.join(d, "enc")
        with open(src, "w") as f:
            f.write(PROGRAM)
        subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-I", os.path.dirname(HEADER), src, "-o", exe], check=True,
                       capture_output=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    idesc = [int(x) for x in out[0].split()]
    assert idesc == [_expected_idesc(64, 32, 0, 0), _expected_idesc(64, 16, 0, 0),
                     _expected_idesc(128, 32, 1, 0), _expected_idesc(128, 16, 1, 0),
                     _expected_idesc(128, 256, 0, 0)]
    # by hand: row 1 chunk 0 -> 128 + (0 ^ 1) * 16 = 144; row 9 chunk 3 -> 1024 + 128 + 2 * 16;
    # row 63 chunk 5 -> 7 * 1024 + 7 * 128 + (5 ^ 7) * 16
    assert [int(x) for x in out[1].split()] == [0, 112, 144, 896, 1184, 7 * 1024 + 7 * 128 + 32]
