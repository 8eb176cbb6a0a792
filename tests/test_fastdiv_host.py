"""The kernels split item indices with FastDiv (csrc/msda_types.h): division by
an invariant divisor as a multiply-high and shifts, after Granlund and
Montgomery, "Division by Invariant Integers using Multiplication" (1994),
Figure 4.1.  This compiles the header's host path with g++ and checks it
against the machine's integer division: every divisor 1..4096 against a grid
of dividends, the divisors next to every power of two, and random pairs over
the whole 32-bit range (the GPU path differs only in computing the
multiply-high with __umulhi, and every GPU parity test runs through it)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "scale_deformable_attention_02_b200", "csrc")

PROGRAM = r"""
#include <cstdio>
#include <cstdint>
#include "msda_types.h"
using msda::FastDiv;

static uint64_t state = 0x9e3779b97f4a7c15ull;
static uint32_t next32() {  // splitmix64, high half
    uint64_t z = (state += 0x9e3779b97f4a7c15ull);
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return (uint32_t)((z ^ (z >> 31)) >> 32);
}

static long long bad = 0, checked = 0;
static void check(uint32_t d, uint32_t n) {
    const FastDiv f = msda::make_fastdiv(d);
    const uint32_t q = msda::fastdiv(f, n);
    ++checked;
    if (q != n / d) {
        if (bad < 10) std::printf("MISMATCH d=%u n=%u got %u want %u\n", d, n, q, n / d);
        ++bad;
    }
}

static void dividends(uint32_t d) {
    const uint32_t edge[] = {0u, 1u, 2u, 3u, 0x7fffffffu, 0x80000000u, 0xfffffffeu, 0xffffffffu};
    for (uint32_t n : edge) check(d, n);
    for (uint32_t k = 0; k < 64; ++k) {  // around multiples of d
        const uint64_t base = (uint64_t)d * (k * 0x1000193ull % 0x100000000ull / d + 0);
        for (int e = -2; e <= 2; ++e) {
            const int64_t n = (int64_t)base + e;
            if (n >= 0 && n <= 0xffffffffll) check(d, (uint32_t)n);
        }
        for (int e = -2; e <= 2; ++e) {
            const int64_t n = (int64_t)d * (int64_t)k + e;
            if (n >= 0 && n <= 0xffffffffll) check(d, (uint32_t)n);
        }
    }
    for (int i = 0; i < 64; ++i) check(d, next32());
}

int main() {
    for (uint32_t d = 1; d <= 4096; ++d) dividends(d);
    for (int b = 1; b < 32; ++b)
        for (int e = -3; e <= 3; ++e) {
            const int64_t d = ((int64_t)1 << b) + e;
            if (d >= 1 && d <= 0xffffffffll) dividends((uint32_t)d);
        }
    dividends(0xffffffffu);
    for (int i = 0; i < 200000; ++i) {
        uint32_t d = next32() >> (next32() % 32);
        if (d == 0) d = 1;
        check(d, next32());
        check(d, next32() >> (next32() % 32));
    }
    std::printf("checked %lld bad %lld\n", checked, bad);
    return bad ? 1 : 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None, reason="no g++")
def test_fastdiv_matches_integer_division(tmp_path):
    src = tmp_path / "fastdiv_check.cpp"
    exe = tmp_path / "fastdiv_check"
    src.write_text(PROGRAM)
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "bad 0" in r.stdout
