"""Host-side check of the scoring kernel's work partition (no GPU).

The kernel's CTAs take contiguous runs of 128-key tiles, cut either flat across the whole
tile space or aligned to the KV heads. `run_begin` (where a CTA's run starts) and
`owner_of` (which CTA holds a tile) are inline functions shared by the host plan and the
device code; a mismatch between them would make a CTA publish its partial softmax into
the wrong slot or wait for the wrong number of peers. This compiles a small C++ program
against the library's internal header and checks, for many shapes:

* the runs cover every tile exactly once, in order, and none is empty;
* owner_of(t) names the CTA whose run holds t;
* head-aligned runs never cross a head, and every head gets the same number of runs;
* the number of CTAs touching a head (the slots it needs) never exceeds the plan's count.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

PROGRAM = r"""
#include <cstdio>
#include "kvp_internal.cuh"
using namespace kvp;

static int check(long long T, long long grid, long long tph, long long cph) {
    long long prev_end = 0;
    for (long long c = 0; c < grid; ++c) {
        const long long a = run_begin(c, T, grid, tph, cph), b = run_begin(c + 1, T, grid, tph, cph);
        if (a != prev_end || b <= a) { std::printf("bad run %lld [%lld,%lld)\n", c, a, b); return 1; }
        if (cph > 0 && a / tph != (b - 1) / tph) { std::printf("run %lld crosses a head\n", c); return 1; }
        for (long long t = a; t < b; ++t)
            if (owner_of(t, T, grid, tph, cph) != (int)c) {
                std::printf("owner_of(%lld) = %d, expected %lld\n", t, owner_of(t, T, grid, tph, cph), c);
                return 1;
            }
        prev_end = b;
    }
    if (prev_end != T) { std::printf("runs end at %lld of %lld\n", prev_end, T); return 1; }
    if (cph > 0)
        for (long long h = 0; h < T / tph; ++h) {
            const int touch = owner_of(h * tph + tph - 1, T, grid, tph, cph) - owner_of(h * tph, T, grid, tph, cph) + 1;
            if (touch != (int)cph) { std::printf("head %lld touched by %d runs\n", h, touch); return 1; }
        }
    return 0;
}

int main() {
    const long long units_list[] = {1, 2, 3, 7, 8, 16, 32, 64, 148, 149, 300};
    const long long tph_list[] = {1, 2, 4, 5, 128, 129, 256, 1024};
    int bad = 0, cases = 0;
    for (long long units : units_list)
        for (long long tph : tph_list) {
            const long long T = units * tph;
            const long long flat_grid = T < kPlanGrid ? T : kPlanGrid;
            bad += check(T, flat_grid, tph, 0);
            ++cases;
            if (units <= kPlanGrid) {
                long long cph = kPlanGrid / units;
                if (cph > tph) cph = tph;
                bad += check(T, cph * units, tph, cph);
                ++cases;
            }
        }
    std::printf("%d cases, %d bad\n", cases, bad);
    return bad ? 1 : 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.isdir(CUDA_INC),
                    reason="needs g++ and the CUDA headers")
def test_run_cuts_and_owner_lookup_agree(tmp_path):
    src = tmp_path / "partition_check.cpp"
    exe = tmp_path / "partition_check"
    src.write_text(PROGRAM)
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(ROOT, "token_eviction_b200", "csrc"), "-I", CUDA_INC,
                           str(src), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "0 bad" in out.stdout
