"""Host-side check of the scoring kernel's work partition (no GPU).

The kernel's CTAs take segments of consecutive 128-key tiles: the flattened tile space cut
flat across the CTAs, or every KV head cut into parts with one or two parts (segments) per
CTA. `segment_of`, `slot_in_head` and `ctas_touching` are inline functions shared by the
host plan and the device code; a mismatch would make a CTA publish its partial softmax
into a slot another CTA also writes, or wait for the wrong number of peers. This compiles
a small C++ program against the library's internal header and checks, for many shapes:

* the segments of all CTAs cover every tile exactly once and none is empty;
* head-aligned segments never cross a head, and the two segments of a CTA lie in
  different heads;
* within every head, the CTAs touching it have distinct slots in [0, touching), and
  their number is what ctas_touching reports;
* the plan's slot count covers every head.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

PROGRAM = r"""
#include <cstdio>
#include <vector>
#include "kvp_internal.cuh"
using namespace kvp;

static int check(long long units, long long tph, long long grid, long long cph, int nseg) {
    const long long T = units * tph;
    std::vector<int> seen(T, 0);
    std::vector<std::vector<int>> slots(units);
    for (long long c = 0; c < grid; ++c) {
        long long prev_head = -1;
        for (int s = 0; s < nseg; ++s) {
            long long a, b;
            segment_of(c, s, T, grid, tph, cph, a, b);
            if (b <= a || a < 0 || b > T) { std::printf("bad segment %lld/%d [%lld,%lld)\n", c, s, a, b); return 1; }
            if (cph > 0 && a / tph != (b - 1) / tph) { std::printf("segment %lld/%d crosses a head\n", c, s); return 1; }
            if (cph > 0 && a / tph == prev_head) { std::printf("CTA %lld has two segments in one head\n", c); return 1; }
            prev_head = a / tph;
            for (long long t = a; t < b; ++t) ++seen[t];
            for (long long h = a / tph; h <= (b - 1) / tph; ++h)
                slots[h].push_back(slot_in_head(c, s, h, T, grid, tph, cph));
        }
    }
    for (long long t = 0; t < T; ++t)
        if (seen[t] != 1) { std::printf("tile %lld covered %d times\n", t, seen[t]); return 1; }
    for (long long h = 0; h < units; ++h) {
        const int touch = ctas_touching(h, T, grid, tph, cph);
        if ((int)slots[h].size() != touch) { std::printf("head %lld: %zu CTAs, ctas_touching %d\n", h, slots[h].size(), touch); return 1; }
        std::vector<int> used(touch, 0);
        for (int sl : slots[h]) {
            if (sl < 0 || sl >= touch || used[sl]++) { std::printf("head %lld: bad or repeated slot %d\n", h, sl); return 1; }
        }
    }
    return 0;
}

int main() {
    const long long units_list[] = {1, 2, 3, 6, 7, 8, 16, 32, 64, 148, 149, 296, 300};
    const long long tph_list[] = {1, 2, 4, 5, 128, 129, 256, 1024};
    int bad = 0, cases = 0;
    for (long long units : units_list)
        for (long long tph : tph_list) {
            const long long T = units * tph;
            const long long flat_grid = T < kPlanGrid ? T : kPlanGrid;
            bad += check(units, tph, flat_grid, 0, 1);
            ++cases;
            if (units <= kPlanGrid) {
                long long cph = kPlanGrid / units;
                if (cph > tph) cph = tph;
                bad += check(units, tph, cph * units, cph, 1);
                ++cases;
            }
            if (units % 2 == 0 && units <= 2 * kPlanGrid) {
                long long cph = 2 * kPlanGrid / units;
                if (cph > tph) cph = tph;
                bad += check(units, tph, cph * units / 2, cph, 2);
                ++cases;
            }
        }
    // the plans kvp_workspace_bytes uses: every head's touching CTAs fit the slot count
    const int shapes[][7] = {{1, 32, 8, 128, 32768, 32, 2048}, {1, 32, 8, 128, 131072, 32, 13107},
                             {8, 28, 4, 128, 16384, 64, 1024}, {1, 4, 2, 64, 512, 16, 128},
                             {2, 6, 3, 64, 777, 16, 100}, {1, 4, 1, 128, 129, 32, 64},
                             {64, 8, 8, 128, 4096, 16, 64}, {1, 2, 2, 128, 700, 300, 400}};
    for (const auto& v : shapes) {
        kvp_shape sh{v[0], v[1], v[2], v[3], v[4], v[5], v[6]};
        Plan pl;
        if (!plan_of(sh, &pl)) { std::printf("no plan\n"); ++bad; continue; }
        const long long units = (long long)sh.batch * sh.hkv;
        bad += check(units, pl.tiles_per_head, pl.grid, pl.cph, pl.nseg);
        for (long long h = 0; h < units; ++h)
            if (ctas_touching(h, pl.total_tiles, pl.grid, pl.tiles_per_head, pl.cph) * kSlotsPerCta > pl.maxslots) {
                std::printf("slots short\n");
                ++bad;
            }
        if (pl.grid > kPlanGrid) { std::printf("grid %d over %d\n", pl.grid, kPlanGrid); ++bad; }
        std::printf("plan b%d hkv%d L%d: grid %d cph %d nseg %d\n", sh.batch, sh.hkv, sh.seq_len, pl.grid, pl.cph, pl.nseg);
        ++cases;
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
                           str(src), "-x", "c++", os.path.join(ROOT, "token_eviction_b200", "csrc", "kvp_plan.cu"),
                           "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "0 bad" in out.stdout
    plans = dict(line.split(": ", 1) for line in out.stdout.splitlines() if line.startswith("plan "))
    # the 32K layer: two head-aligned segments per CTA (both 32 KiB query blocks stay in
    # shared memory), 37 parts per head on 148 CTAs
    assert plans["plan b1 hkv8 L32768"] == "grid 148 cph 37 nseg 2"
    # GQA-7 (G w = 448: 112 KiB query blocks, too big to keep two): one segment per CTA,
    # so that no CTA changes head and reloads its block
    assert plans["plan b8 hkv4 L16384"].endswith("nseg 1")
