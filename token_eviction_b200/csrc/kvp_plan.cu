// The work plan of a shape (host code only): which limits a shape must meet, how the
// scoring kernel's tiles are cut among its CTAs, and the workspace layout. Kept apart from
// the CUDA entry points so that host-side tests can compile it with a plain C++ compiler.
#include <algorithm>
#include <cstdint>

#include "kvp_internal.cuh"

namespace kvp {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static bool shape_ok(const kvp_shape& s) {
    if (s.batch < 1 || s.hkv < 1 || s.hq < 1 || s.hq % s.hkv != 0) return false;
    if (s.head_dim != 64 && s.head_dim != 128) return false;
    if (s.seq_len < 1 || s.window < 1 || s.window > s.seq_len) return false;
    if (s.budget < s.window || s.budget > s.seq_len) return false;
    if ((int64_t)(s.hq / s.hkv) * s.window > kMaxGroupRows) return false;
    // element offsets of k/v stay well inside int64; row counts inside int32
    if ((int64_t)s.batch * s.hkv > 65535) return false;  // grid y extent
    if ((int64_t)s.batch * s.hkv * s.seq_len > INT32_MAX) return false;
    if ((int64_t)s.batch * s.hq * s.window > INT32_MAX) return false;
    if ((int64_t)s.batch * s.hkv * s.budget * 16 > INT32_MAX / 2) return false;  // gather pieces
    return true;
}

bool plan_of(const kvp_shape& s, Plan* p) {
    if (!shape_ok(s)) return false;
    p->G = s.hq / s.hkv;
    p->rows = p->G * s.window;
    const long long units = (long long)s.batch * s.hkv;
    p->tiles_per_head = (s.seq_len + 127) / 128;
    const long long T = units * p->tiles_per_head;
    if (T > INT32_MAX) return false;
    // the device's 32-bit partition arithmetic (segment_of_u32 and friends)
    if (T * (kPlanGrid + 1) >= (1LL << 32)) return false;
    p->total_tiles = (int)T;
    const long long tph = p->tiles_per_head;
    // Candidate cuts, compared by the tiles of the longest CTA's work.
    //   flat: the flattened tiles over kPlanGrid CTAs (runs may cross heads, which costs
    //     about kHeadSwitchTiles tiles of waiting);
    //   one segment per CTA: every head cut into floor(148 / heads) parts;
    //   two segments per CTA (an even number of heads): every head cut into
    //     floor(296 / heads) parts, each CTA taking parts of two heads.
    const long long flat_grid = std::min<long long>(kPlanGrid, T);
    long long best_cost = (T + flat_grid - 1) / flat_grid + kHeadSwitchTiles;
    p->cph = 0;
    p->nseg = 1;
    p->grid = (int)flat_grid;
    if (units <= kPlanGrid) {
        const long long cph = std::min<long long>(kPlanGrid / units, tph);
        const long long cost = (tph + cph - 1) / cph;
        if (cost <= best_cost) {
            best_cost = cost;
            p->cph = (int)cph;
            p->nseg = 1;
            p->grid = (int)(cph * units);
        }
    }
    // Two segments change head twice more per CTA. The scoring kernel keeps both runs'
    // query blocks in shared memory when they fit beside four 128-key ring slots (and some
    // 24 KiB of bookkeeping); otherwise every change of head reloads a block, which costs
    // about as much as kHeadSwitchTiles tiles (GQA-7 with w = 64: 112 KiB per block).
    const long long qblock = (long long)(p->rows + 63) / 64 * 64 * s.head_dim * 2;
    const long long tile = 128LL * s.head_dim * 2;
    const bool both_blocks = 2 * qblock + 4 * tile + 24 * 1024 <= 227 * 1024;
    if (units % 2 == 0 && units <= 2 * kPlanGrid) {
        const long long cph = std::min<long long>(2 * kPlanGrid / units, tph);
        const long long cost = 2 * ((tph + cph - 1) / cph) + (both_blocks ? 0 : kHeadSwitchTiles);
        if (cost <= best_cost) {
            best_cost = cost;
            p->cph = (int)cph;
            p->nseg = 2;
            p->grid = (int)(cph * units / 2);
        }
    }
    int slots = 0;
    for (long long h = 0; h < units; ++h)
        slots = std::max(slots, ctas_touching(h, T, p->grid, tph, p->cph));
    p->maxslots = slots * kSlotsPerCta;
    // the error word sits at offset 0 of every workspace, so that a status read needs no shape
    size_t off = 0;
    p->off_err = off;
    off += 256;
    p->off_done = off;
    off += align_up((size_t)units * sizeof(uint32_t), 256);
    p->off_part = off;
    off += align_up((size_t)s.batch * s.hq * s.window * p->maxslots * sizeof(float2), 256);
    p->off_select = off;
    off += 256;
    p->bytes = off;
    return true;
}

}  // namespace kvp
