"""The tensor-core operand layout of the saved state and of the forward's [Kt; Qt] tile
(`umma_off` in csrc/carve_umma.cuh), checked on the host against the rules the tensor core
and ldmatrix impose: compiled as host code by nvcc, no GPU involved."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "chunk_gated_delta_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include "carve_umma.cuh"
int main() {
    const int rows_list[3] = {32, 64, 128};
    for (int ri = 0; ri < 3; ++ri) {
        const int rows = rows_list[ri];
        static int seen[128 * 128];
        for (int i = 0; i < rows * 128; ++i) seen[i] = 0;
        for (int r = 0; r < rows; ++r)
            for (int c = 0; c < 128; ++c) {
                const int e = carve::umma_off(r, c, rows);
                if (e < 0 || e >= rows * 128) { printf("range %d %d %d\n", rows, r, c); return 1; }
                ++seen[e];
                const int byte = 2 * e;
                // half h (columns 64h .. 64h + 63) is a block of rows x 128 bytes
                if (byte / (rows * 128) != c / 64) { printf("half %d %d %d\n", rows, r, c); return 1; }
                const int in_half = byte % (rows * 128);
                // row r at r * 128 bytes within its half
                if (in_half / 128 != r) { printf("row %d %d %d\n", rows, r, c); return 1; }
                // elements of one 16-byte chunk stay together and in order
                if (byte % 16 != 2 * (c % 8)) { printf("chunk %d %d %d\n", rows, r, c); return 1; }
                // 128-byte swizzle as the tensor core applies it to a 1024-byte aligned base:
                // stored chunk position (address bits 4-6) = logical chunk ^ address bits 7-9
                if (((byte >> 4) & 7) != (((c % 64) / 8) ^ ((byte >> 7) & 7))) {
                    printf("swizzle %d %d %d\n", rows, r, c); return 1; }
            }
        for (int i = 0; i < rows * 128; ++i)
            if (seen[i] != 1) { printf("bijection %d %d\n", rows, i); return 1; }
        // an 8x8 ldmatrix read (eight consecutive rows, one 16-byte column chunk) touches eight
        // different 16-byte bank groups
        for (int r0 = 0; r0 < rows; r0 += 8)
            for (int c = 0; c < 128; c += 8) {
                int groups = 0;
                for (int x = 0; x < 8; ++x) groups |= 1 << (((2 * carve::umma_off(r0 + x, c, rows)) >> 4) & 7);
                if (groups != 0xff) { printf("banks %d %d %d\n", rows, r0, c); return 1; }
            }
    }
    printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not on PATH")
def test_operand_layout_rules():
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "layout.cu"), os.path.join(d, "layout")
        open(src, "w").write(PROGRAM)
        subprocess.run(["nvcc", "-std=c++17", "-I", CSRC, "-o", exe, src], check=True, capture_output=True)
        out = subprocess.run([exe], capture_output=True, text=True)
        assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout
