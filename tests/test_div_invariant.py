"""The kernels' division by the grid height (column-major order) multiplies by a
constant formed on the host (Granlund and Montgomery, "Division by Invariant Integers
using Multiplication", Figure 4.1).  This compiles a host program against the kernel
header and checks div_by(n, div_inv(d)) == n / d: every n below 70000 for d <= 300,
and sampled n (the 32-bit extremes included) for d up to 20000 and near 2^32.  CPU only
(nvcc compiles host code without a GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "vision_mamba_selective_b200", "csrc")
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include "scan_kernels.cuh"
using namespace vimscan;
static unsigned long long checks = 0, bad = 0;
static void check(unsigned n, unsigned d, const DivInv &v) {
    ++checks;
    if (div_by(n, v) != n / d && ++bad < 10) std::printf("d=%u n=%u: %u\n", d, n, div_by(n, v));
}
int main() {
    uint64_t x = 88172645463325252ull;
    auto next = [&]() { x ^= x << 13; x ^= x >> 7; x ^= x << 17; return (unsigned)x; };
    for (unsigned d = 1; d <= 20000; ++d) {
        const DivInv v = div_inv(d);
        const unsigned edge[] = {0u, 1u, d - 1, d, d + 1, 2 * d - 1, 2 * d, 0x7ffffffeu, 0x7fffffffu, 0xfffffffeu,
                                 0xffffffffu};
        for (unsigned n : edge) check(n, d, v);
        for (int i = 0; i < 200; ++i) check(next() >> (i % 32), d, v);
        if (d <= 300)
            for (unsigned n = 0; n < 70000; ++n) check(n, d, v);
    }
    const unsigned big[] = {0x80000000u, 0x80000001u, 0xfffffffeu, 0xffffffffu, 3000000000u, 196611u, 1u << 20,
                            (1u << 20) + 1};
    for (unsigned d : big) {
        const DivInv v = div_inv(d);
        for (int i = 0; i < 20000; ++i) check(next(), d, v);
    }
    std::printf("%llu %llu\n", checks, bad);
    return bad != 0;
}
"""


@pytest.mark.skipif(not os.path.exists(NVCC), reason="nvcc is not installed")
def test_division_by_invariant_integers(tmp_path):
    src = tmp_path / "div.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "div"
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O2", "-I", CSRC, "-I",
                    os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True, capture_output=True,
                   timeout=600)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout
    checks, bad = map(int, out.stdout.split()[-2:])
    assert bad == 0 and checks > 25_000_000
