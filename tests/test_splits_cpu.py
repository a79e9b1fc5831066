"""The tile splits of the decode call (csrc/splits.h), compiled for the host and
checked exhaustively over small sizes: each split partitions the tiles (every tile
goes to exactly one CTA or warp, in contiguous runs) and balances the ring entries
(two per bf16 tile, one per FP8 tile).  The decode kernel includes the same header,
so these are the functions that run on the device."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mixed_precision_kv_arkv_b200", "csrc")

HARNESS = r"""
#include <cstdio>
#include <cstdlib>
#include "splits.h"
using namespace arkv;
static int fail(const char* what, long long a, long long b, long long c) {
    std::printf("FAIL %s %lld %lld %lld\n", what, a, b, c);
    return 1;
}
int main() {
    // CTA split: n CTAs of a row with T16 bf16 and T8 FP8 tiles
    for (int n = 1; n <= 40; ++n)
        for (int T16 = 0; T16 <= 260; T16 += 1 + T16 / 16)
            for (int T8 = 0; T8 <= 260; T8 += 1 + T8 / 16) {
                if (fp8_tiles_before(T16, T8, n, 0) != 0 || fp8_tiles_before(T16, T8, n, n) != T8)
                    return fail("cta ends", n, T16, T8);
                int lo = 1 << 30, hi = -1;
                for (int c = 0; c < n; ++c) {
                    const int f0 = fp8_tiles_before(T16, T8, n, c), f1 = fp8_tiles_before(T16, T8, n, c + 1);
                    if (f1 < f0) return fail("cta monotone", n, T16, T8);
                    const long long b0 = (long long)T16 * c / n, b1 = (long long)T16 * (c + 1) / n;
                    const int e = (int)(2 * (b1 - b0)) + (f1 - f0);
                    lo = e < lo ? e : lo;
                    hi = e > hi ? e : hi;
                }
                if (T8 >= 2 * n && hi - lo > 1) return fail("cta balance", n, T16, T8);
            }
    // warp split: a CTA's L16 bf16 tiles round robin, its L8 FP8 tiles in runs
    for (int L16 = 0; L16 <= 300; ++L16)
        for (int L8 = 0; L8 <= 300; ++L8) {
            int next = 0, lo = 1 << 30, hi = -1, total = 0;
            for (int w = 0; w < kSplitWarps; ++w) {
                int s, c;
                warp_fp8_share(L16, L8, w, &s, &c);
                if (c < 0 || s != next) return fail("warp runs", L16, L8, w);
                next = s + c;
                total += c;
                const int b = L16 > w ? (L16 - w + kSplitWarps - 1) / kSplitWarps : 0;
                const int e = 2 * b + c;
                lo = e < lo ? e : lo;
                hi = e > hi ? e : hi;
            }
            if (total != L8) return fail("warp total", L16, L8, total);
            // the FP8 tiles can level the warps once they cover the bf16 difference
            const int b0 = L16 > 0 ? (L16 + kSplitWarps - 1) / kSplitWarps : 0, b3 = L16 / kSplitWarps;
            int short_warps = 0;
            for (int w = 0; w < kSplitWarps; ++w)
                short_warps += (L16 > w ? (L16 - w + kSplitWarps - 1) / kSplitWarps : 0) == b3 ? 1 : 0;
            if (L8 >= 2 * (b0 - b3) * short_warps && hi - lo > 1) return fail("warp balance", L16, L8, hi - lo);
        }
    std::printf("ok\n");
    return 0;
}
"""


def test_tile_splits_partition_and_balance(tmp_path):
    src = tmp_path / "splits_check.cpp"
    exe = tmp_path / "splits_check"
    src.write_text(HARNESS)
    cc = os.environ.get("CXX", "g++")
    subprocess.run([cc, "-O2", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
