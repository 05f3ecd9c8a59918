// S1 * S2 scoring on sm_100a: one persistent, warp-specialised tcgen05 kernel.
//
// "Preserving Large Activations: The Key to KV Cache Pruning" (SlimKV), Section 3:
//   Eq. 3  S1[j] = sum over the G query heads of the KV head's group (Section 3.1) and
//                  the w window queries of softmax_j(q . k_j / sqrt(d))
//   Eq. 4  S2[j] = max_c |V[j, c]|
//   Eq. 5  S[j]  = S1[j] * S2[j]
// Window query i sits at position L - w + i and sees keys j <= L - w + i.
//
// A softmax row's denominator must be known before any key's S1 can be summed, so K is
// swept twice; both sweeps run inside one kernel. Each CTA owns a contiguous run of
// 128-key tiles of the flattened (sequence, KV head, tile) space.
//   phase 0 (log-sum-exp; one query row per thread): tcgen05 computes
//     D[row, key] = Q_group[row] . K_tile[key]  (M = 128 rows of one row block, N = keys),
//     so each epilogue thread owns one query row (a TMEM lane) and keeps its running
//     offset m and sum l = sum_j 2^(t_j - m) in registers, t = logit * log2(e) / sqrt(d).
//     At the end of each KV head in its run a CTA publishes one (m, l) slot per row to
//     the workspace and bumps the head's completion counter.
//   phase 1 (scores; one key per thread): the same tiles again (K now mostly from L2),
//     with D[key, row] = K_tile[key] . Q_group[row]  (M = 128 keys, N = query rows).
//     Before its first tile of a head a CTA waits (bounded) until every CTA touching the
//     head has published, then merges the slots into lse2 = M + log2(sum_s l_s 2^(m_s-M))
//     per row. Per tile each thread sums 2^(t - lse2) over its key's query rows: S1.
//   S2 is reduced from each V tile, staged once in shared memory, by two warps of its own,
//   so that V's arrival from HBM never stalls the exponentials.
// Warp roles: warp 0 issues TMA loads (a ring of tile slots and the group's query rows),
// warp 1 allocates TMEM and issues the MMAs from one thread, warps 2-3 reduce V tiles to
// S2, and two epilogue warpgroups (warps 4-7 and 8-11, one TMEM lane quarter per warp)
// read the accumulators. TMEM holds four accumulator stages of 128 columns; a tile's work
// is cut into units of at most 128 columns (phase 0: a run of keys over every row block;
// phase 1: a part of the query rows), unit k takes stage k % 4, and stage s belongs to
// epilogue group s % 2.
// Every wait is bounded by a timer; a wait that gives up records an error code in the
// workspace and the CTA unwinds without touching TMEM or shared memory still in use.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "kvp_internal.cuh"
#include "kvp_ptx.cuh"

namespace kvp {

namespace {

constexpr int kTile = 128;                        // keys per tile
constexpr int kGroups = 2;                        // epilogue warpgroups
constexpr int kStages = 4;                        // TMEM accumulator stages
constexpr int kStageCols = 128;                   // TMEM columns per stage
constexpr uint32_t kTmemCols = kStages * kStageCols;
constexpr int kWarpS2 = 2, kS2Warps = 2;          // warps that reduce V tiles to S2
constexpr int kWarpEpi = kWarpS2 + kS2Warps;      // first epilogue warp
constexpr int kEpiThreads = 128 * kGroups;
constexpr int kThreads = 32 * kWarpEpi + kEpiThreads;
constexpr int kMaxSlots = 8;                      // tile slots of the load ring
constexpr int kS2Bufs = 4;                        // S2 hand-off buffers (one tile each)
constexpr int kCombBufs = 2;                      // partial-S1 hand-off buffers
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s on any single wait
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMinSmem = 116 * 1024;              // forces one CTA per SM (TMEM is taken whole)
constexpr int kQBoxRows = 64;
constexpr size_t kBarBytes = 640;                 // shared memory reserved for SmemBars
constexpr float kSumLimit = 1.8446744e19f;        // 2^64: a chunk sum above it raises the offset

#ifdef KVP_TRACE
// Debug builds only: %globaltimer stamps per CTA at phase boundaries.
__device__ unsigned long long g_kvp_trace[kPlanGrid][8];
#define KVP_STAMP(i) (g_kvp_trace[blockIdx.x][(i)] = ptx::globaltimer_ns())
// per-tile events of four CTAs: [cta][tile][event]
__device__ unsigned long long g_kvp_ttrace[4][64][8];
__device__ long long g_kvp_mtrace[4][64][12];
__device__ __forceinline__ int kvp_trace_slot() {
    return blockIdx.x == 0 ? 0 : blockIdx.x == 18 ? 1 : blockIdx.x == 73 ? 2 : blockIdx.x == 143 ? 3 : -1;
}
#define KVP_TSTAMP(t, e) \
    ((kvp_trace_slot() >= 0 && (t) < 64) ? (void)(g_kvp_ttrace[kvp_trace_slot()][(t)][(e)] = ptx::globaltimer_ns()) : (void)0)
#else
#define KVP_STAMP(i) ((void)0)
#define KVP_TSTAMP(t, e) ((void)0)
#endif

// error codes recorded in the workspace (first one wins)
enum : int { kErrWaitTma = 1, kErrWaitMma = 2, kErrWaitEpi = 3, kErrWaitPeers = 4, kErrWaitS2 = 5 };

struct Params {
    int L, w, rows, hq, hkv, G;
    int nrb, nk0, u0, lg_cpb;  // phase 0: row blocks, keys per unit, units per tile, log2(nk0 / 32)
    int p1, n1, rows16;        // phase 1: parts per tile, rows per part, rows rounded up to 16
    int qrows;                 // query rows staged in shared memory (rows rounded up to 64)
    int tiles_per_head, total_tiles, grid, cph, maxslots;
    int ns, nk1, nv1;          // ring slots; phase 1 gives K slots [0, nk1), V slots [nk1, ns)
    float scale2;              // log2(e) / sqrt(d)
    uint32_t q_bytes, tile_bytes;
    uint32_t off_slots, off_lse, off_comb, off_s2, off_stage, off_wpos, off_bar;
    int extra_peers;           // fault injection (debug builds): peers that never arrive
    unsigned long long wait_limit_ns;
    float* score;
    float* s1;
    float* s2;
    float2* part;              // [b*hq*w][maxslots]: (max, sum) in log2 units
    uint32_t* done;            // [b*hkv]
    int* err;
};

struct SmemBars {
    uint64_t kfull[kMaxSlots], kempty[kMaxSlots];   // per slot, for its K loads
    uint64_t vfull[kMaxSlots], vempty[kMaxSlots];   // per phase 1 V slot (index s - nk1)
    uint64_t accfull[kStages], accempty[kStages];
    uint64_t combfull[kCombBufs], combempty[kCombBufs];
    uint64_t s2full[kS2Bufs], s2empty[kS2Bufs];
    uint64_t qfull, qempty, fin;
    uint64_t epi;        // rendezvous of all epilogue threads
    uint32_t tmem_base;
    int abort_flag;
};

// Wait for phase `parity` of `bar`; false if the CTA is unwinding or the wait timed out
// (then the first error code is recorded and the CTA told to unwind).
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, SmemBars* sb,
                                           const Params& p, int code) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*(volatile int*)&sb->abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > p.wait_limit_ns) {
            atomicCAS(p.err, 0, code);
            *(volatile int*)&sb->abort_flag = 1;
            return false;
        }
    }
}

// Wait for phase `parity` of `bar` for at most the wait limit, whatever the CTA's state:
// used before exit, so that no copy or MMA is still writing this CTA's memory.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity))
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) return;
}

// Rendezvous of all epilogue threads on an mbarrier, so that a thread that gives up a
// wait can never leave the others blocked in a hardware barrier. One arrival per warp,
// after the warp's memory writes are ordered before it.
__device__ __forceinline__ bool epi_sync(SmemBars* sb, uint32_t& phase, const Params& p) {
    __threadfence_block();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(&sb->epi);
    const bool ok = wait_phase(&sb->epi, phase, sb, p, kErrWaitEpi);
    phase ^= 1u;
    return ok;
}

__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
    __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
    __nv_bfloat162 m = __hmax2(x, y);
    return *reinterpret_cast<uint32_t*>(&m);
}

// max |v| over the D bf16 values of one row in shared memory, read in 16-byte pieces in a
// rotated order per lane (consecutive lanes hit distinct bank groups).
template <int D>
__device__ __forceinline__ float row_absmax(const uint8_t* row, int lane) {
    constexpr int kPieces = D * 2 / 16;
    const uint4* r = reinterpret_cast<const uint4*>(row);
    uint32_t mx = 0;
#pragma unroll
    for (int c = 0; c < kPieces; ++c) {
        const uint4 x = r[(c + lane) & (kPieces - 1)];
        mx = bf16x2_absmax(mx, x.x & 0x7FFF7FFFu);
        mx = bf16x2_absmax(mx, x.y & 0x7FFF7FFFu);
        mx = bf16x2_absmax(mx, x.z & 0x7FFF7FFFu);
        mx = bf16x2_absmax(mx, x.w & 0x7FFF7FFFu);
    }
    return fmaxf(__uint_as_float(mx << 16), __uint_as_float(mx & 0xFFFF0000u));
}

// Uses of ring position s among the first n uses of a ring of `period` positions.
__device__ __forceinline__ int ring_uses(int s, int period, int n) {
    return n > s ? (n - s + period - 1) / period : 0;
}
// K slot of the run's tile i in `phase`, and the number of that slot's earlier K loads.
// Phase 0 streams K through all ns slots in turn; phase 1 through slots [0, nk1).
__device__ __forceinline__ int k_slot(int phase, int i, int n, const Params& p, int& use) {
    if (phase == 0) {
        use = i / p.ns;
        return i % p.ns;
    }
    const int s = i % p.nk1;
    use = ring_uses(s, p.ns, n) + i / p.nk1;
    return s;
}

// Segments of a CTA's run: maximal stretches of tiles within one KV head.
struct RunIter {
    long long t, end;
    int tph;
    __device__ RunIter(long long b, long long e, int tiles_per_head) : t(b), end(e), tph(tiles_per_head) {}
    __device__ bool next(int& head, long long& a, long long& b) {
        if (t >= end) return false;
        head = (int)(t / tph);
        a = t;
        b = min(end, (long long)(head + 1) * tph);
        t = b;
        return true;
    }
};

// Element i of a 4-entry register array with a run-time index, without local memory.
template <typename T>
__device__ __forceinline__ T pick4(const T (&a)[4], int i) {
    return i == 0 ? a[0] : i == 1 ? a[1] : i == 2 ? a[2] : a[3];
}
template <typename T>
__device__ __forceinline__ void put4(T (&a)[4], int i, T x) {
    a[0] = i == 0 ? x : a[0];
    a[1] = i == 1 ? x : a[1];
    a[2] = i == 2 ? x : a[2];
    a[3] = i == 3 ? x : a[3];
}

// Phase 0, one chunk of 32 keys of one query row (v: raw logits, -inf where masked):
// adds sum_e 2^(v_e * scale2 - m) to l. The offset m is raised (and l rescaled) only when
// a chunk sum would exceed 2^64, which also covers the head's first chunk (m = -inf).
__device__ __forceinline__ void lse_chunk(const float (&v)[32], float scale2, float& m, float& l) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
        a0 += ptx::ex2(fmaf(v[e + 0], scale2, -m));
        a1 += ptx::ex2(fmaf(v[e + 1], scale2, -m));
        a2 += ptx::ex2(fmaf(v[e + 2], scale2, -m));
        a3 += ptx::ex2(fmaf(v[e + 3], scale2, -m));
    }
    float cs = (a0 + a1) + (a2 + a3);
    if (__any_sync(0xffffffffu, !(cs <= kSumLimit))) {
        // rare: the chunk holds logits far above this row's offset (or the offset is unset)
        float mc = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e) mc = fmaxf(mc, v[e]);
        mc *= scale2;
        if (mc > m) {
            l *= ptx::ex2(m - mc);                 // m = -inf: l is 0 and stays 0
            m = mc;
        }
        cs = 0.f;
        if (m != -INFINITY) {
            a0 = a1 = a2 = a3 = 0.f;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                a0 += ptx::ex2(fmaf(v[e + 0], scale2, -m));
                a1 += ptx::ex2(fmaf(v[e + 1], scale2, -m));
                a2 += ptx::ex2(fmaf(v[e + 2], scale2, -m));
                a3 += ptx::ex2(fmaf(v[e + 3], scale2, -m));
            }
            cs = (a0 + a1) + (a2 + a3);
        }
    }
    l += cs;
}

// Phase 1, one chunk of 32 query rows of one key: adds 2^(v_e * scale2 - lse2_e). With
// `masked`, rows from `nrem` on (past the part's last) contribute nothing, nor, for a
// window key (jw > 0), rows whose window position is before the key.
__device__ __forceinline__ float s1_chunk(const float (&v)[32], const float* lse2, const uint16_t* wp,
                                          bool masked, int jw, int nrem, float scale2) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    if (!masked) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
            const float4 l4 = *(const float4*)(lse2 + e);
            a0 += ptx::ex2(fmaf(v[e + 0], scale2, -l4.x));
            a1 += ptx::ex2(fmaf(v[e + 1], scale2, -l4.y));
            a2 += ptx::ex2(fmaf(v[e + 2], scale2, -l4.z));
            a3 += ptx::ex2(fmaf(v[e + 3], scale2, -l4.w));
        }
    } else {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
            const float4 l4 = *(const float4*)(lse2 + e);
            const bool m0 = e + 0 < nrem && jw <= (int)wp[e + 0];
            const bool m1 = e + 1 < nrem && jw <= (int)wp[e + 1];
            const bool m2 = e + 2 < nrem && jw <= (int)wp[e + 2];
            const bool m3 = e + 3 < nrem && jw <= (int)wp[e + 3];
            a0 += m0 ? ptx::ex2(fmaf(v[e + 0], scale2, -l4.x)) : 0.f;
            a1 += m1 ? ptx::ex2(fmaf(v[e + 1], scale2, -l4.y)) : 0.f;
            a2 += m2 ? ptx::ex2(fmaf(v[e + 2], scale2, -l4.z)) : 0.f;
            a3 += m3 ? ptx::ex2(fmaf(v[e + 3], scale2, -l4.w)) : 0.f;
        }
    }
    return (a0 + a1) + (a2 + a3);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
score_fused_tc(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* Qs = smem;                                  // [D / 64][qrows][64] bf16, 128B swizzle
    uint8_t* Slots = smem + p.off_slots;                 // ring slots of tile_bytes each
    float* lse2 = (float*)(smem + p.off_lse);            // [rows, padded to 4]
    float* comb = (float*)(smem + p.off_comb);           // [kCombBufs][128] partial S1 hand-off
    float* s2buf = (float*)(smem + p.off_s2);            // [kS2Bufs][128] S2 of a tile's keys
    float2* stage0 = (float2*)(smem + p.off_stage);      // [rows] phase 0 group hand-off
    uint16_t* wpos = (uint16_t*)(smem + p.off_wpos);     // window position of query row n: n % w
    SmemBars* sb = (SmemBars*)(smem + p.off_bar);

    constexpr int kHalves = D / 64;                 // 128-byte swizzle rows per operand row
    constexpr uint32_t kHalfTile = kTile * 128;     // bytes of one 64-column half of a tile
    constexpr uint32_t kSlotBytes = kTile * D * 2;
    const uint32_t qhalf = (uint32_t)p.qrows * 128;  // bytes of one 64-column half of Q

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long T = p.total_tiles;
    const long long t0 = run_begin(blockIdx.x, T, p.grid, p.tiles_per_head, p.cph);
    const long long t1 = run_begin(blockIdx.x + 1, T, p.grid, p.tiles_per_head, p.cph);
    const int n = (int)(t1 - t0);                   // tiles in this CTA's run
    const int U0 = n * p.u0;                        // phase 0 units of the run

    for (int r = threadIdx.x; r < p.rows; r += kThreads) wpos[r] = (uint16_t)(r % p.w);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxSlots; ++s) {
            ptx::mbar_init(&sb->kfull[s], 1);
            ptx::mbar_init(&sb->kempty[s], 1);
            ptx::mbar_init(&sb->vfull[s], 1);
            ptx::mbar_init(&sb->vempty[s], kS2Warps);
        }
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&sb->accfull[s], 1);
            ptx::mbar_init(&sb->accempty[s], 4);
        }
        for (int s = 0; s < kCombBufs; ++s) {
            ptx::mbar_init(&sb->combfull[s], 4);
            ptx::mbar_init(&sb->combempty[s], 4);
        }
        for (int s = 0; s < kS2Bufs; ++s) {
            ptx::mbar_init(&sb->s2full[s], kS2Warps);
            ptx::mbar_init(&sb->s2empty[s], 4);
        }
        ptx::mbar_init(&sb->qfull, 1);
        ptx::mbar_init(&sb->qempty, 1);
        ptx::mbar_init(&sb->fin, 1);
        ptx::mbar_init(&sb->epi, kEpiThreads / 32);
        sb->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tensormap(&qmap);
        ptx::prefetch_tensormap(&kmap);
        ptx::prefetch_tensormap(&vmap);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&sb->tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sb->tmem_base;
    if (threadIdx.x == 0) KVP_STAMP(0);

    auto group_row0 = [&](int bh) {
        const int b = bh / p.hkv, h = bh % p.hkv;
        return (b * p.hq + h * p.G) * p.w;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // K is read again by phase 1 (from L2 when it fits); V and phase 1's K stream
            const uint64_t pol_keep = ptx::policy_evict_normal();
            const uint64_t pol_stream = ptx::policy_evict_first();
            int qgen = 0, cur = -1;
            int kiss[kMaxSlots] = {}, viss[kMaxSlots] = {};   // loads issued per slot
            bool ok = true;
            for (int phase = 0; phase < 2 && ok; ++phase) {
                RunIter it(t0, t1, p.tiles_per_head);
                int head;
                long long a, b;
                int i = 0;                                  // tile number within the run
                while (ok && it.next(head, a, b)) {
                    if (head != cur) {
                        if (qgen > 0 && !(ok = wait_phase(&sb->qempty, (qgen - 1) & 1, sb, p, kErrWaitTma))) break;
                        ptx::mbar_arrive_expect_tx(&sb->qfull, p.q_bytes);
                        const int r0 = group_row0(head);
                        for (int rb = 0; rb < p.qrows; rb += kQBoxRows)
                            for (int c = 0; c < kHalves; ++c)
                                ptx::tma_load_2d(Qs + c * qhalf + rb * 128, &qmap, &sb->qfull,
                                                 c * 64, r0 + rb, pol_keep);
                        ++qgen;
                        cur = head;
                    }
                    for (long long t = a; t < b; ++t, ++i) {
                        const int key0 = (int)(t - (long long)head * p.tiles_per_head) * kTile;
                        int use;
                        const int s = k_slot(phase, i, n, p, use);
                        if (!(ok = wait_phase(&sb->kempty[s], (use & 1) ^ 1, sb, p, kErrWaitTma))) break;
                        KVP_TSTAMP(phase * n + i, 0);
                        ptx::mbar_arrive_expect_tx(&sb->kfull[s], p.tile_bytes);
                        for (int c = 0; c < kHalves; ++c)
                            ptx::tma_load_3d(Slots + s * kSlotBytes + c * kHalfTile, &kmap, &sb->kfull[s],
                                             c * 64, key0, head, phase == 0 ? pol_keep : pol_stream);
                        ++kiss[s];
                        if (phase == 1) {
                            const int jv = i % p.nv1, sv = p.nk1 + jv, vuse = i / p.nv1;
                            // a V slot's first load waits for its last K load of phase 0 to be consumed
                            const int u0s = vuse == 0 ? ring_uses(sv, p.ns, n) : 0;
                            if (u0s > 0 && !(ok = wait_phase(&sb->kempty[sv], (u0s - 1) & 1, sb, p, kErrWaitTma))) break;
                            if (!(ok = wait_phase(&sb->vempty[jv], (vuse & 1) ^ 1, sb, p, kErrWaitTma))) break;
                            KVP_TSTAMP(phase * n + i, 6);
                            ptx::mbar_arrive_expect_tx(&sb->vfull[jv], p.tile_bytes);
                            ptx::tma_load_3d(Slots + sv * kSlotBytes, &vmap, &sb->vfull[jv], 0, key0, head,
                                             pol_stream);
                            ++viss[jv];
                        }
                    }
                }
                KVP_STAMP(1 + phase);
            }
            // Never leave with copies in flight: wait for the last load issued to every slot
            // (these waits do not stop early when the CTA unwinds).
            for (int s = 0; s < p.ns; ++s)
                if (kiss[s] > 0) drain_wait(&sb->kfull[s], (kiss[s] - 1) & 1);
            for (int jv = 0; jv < p.nv1; ++jv)
                if (viss[jv] > 0) drain_wait(&sb->vfull[jv], (viss[jv] - 1) & 1);
            if (qgen > 0) drain_wait(&sb->qfull, (qgen - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t q_addr = ptx::smem_u32(Qs), k_addr = ptx::smem_u32(Slots);
            const uint32_t idesc0 = ptx::idesc_bf16_f32(128, p.nk0);
            int qgen = 0, cur = -1;
            bool ok = true;
            for (int phase = 0; phase < 2 && ok; ++phase) {
                RunIter it(t0, t1, p.tiles_per_head);
                int head;
                long long a, b;
                int i = 0;                                  // tile number within the run
                int unit = 0;                               // unit number within the phase
                while (ok && it.next(head, a, b)) {
                    if (head != cur) {
                        if (!(ok = wait_phase(&sb->qfull, qgen & 1, sb, p, kErrWaitMma))) break;
                        ++qgen;
                        cur = head;
                        ptx::tc_fence_after();
                    }
                    for (long long t = a; t < b && ok; ++t, ++i) {
                        int kuse;
                        const int s = k_slot(phase, i, n, p, kuse);
                        if (!(ok = wait_phase(&sb->kfull[s], kuse & 1, sb, p, kErrWaitMma))) break;
                        KVP_TSTAMP(phase * n + i, 1);
                        const uint32_t kbase = k_addr + s * kSlotBytes;
                        const int nunits = phase == 0 ? p.u0 : p.p1;
                        for (int j = 0; j < nunits; ++j, ++unit) {
                            const int st = unit & (kStages - 1);
                            const int use = (phase == 0 ? 0 : ring_uses(st, kStages, U0)) + unit / kStages;
                            if (!(ok = wait_phase(&sb->accempty[st], (use & 1) ^ 1, sb, p, kErrWaitMma))) break;
                            ptx::tc_fence_after();
                            const uint32_t d0 = tmem + (uint32_t)(st * kStageCols);
                            if (phase == 0) {
                                // D[row, key] for every row block: A = Q rows, B = the unit's keys
                                for (int rb = 0; rb < p.nrb; ++rb) {
                                    const uint64_t qd = ptx::sw128_kmajor_desc(q_addr + rb * 128 * 128);
                                    const uint64_t kd = ptx::sw128_kmajor_desc(kbase + j * p.nk0 * 128);
#pragma unroll
                                    for (int ks = 0; ks < D / 16; ++ks) {
                                        const uint32_t qo = ((ks >> 2) * qhalf + (ks & 3) * 32) >> 4;
                                        const uint32_t ko = ((ks >> 2) * kHalfTile + (ks & 3) * 32) >> 4;
                                        ptx::mma_bf16_ss(d0 + rb * p.nk0, qd + qo, kd + ko, idesc0, ks > 0);
                                    }
                                }
                            } else {
                                // D[key, row] for one part of the query rows: A = keys, B = Q rows
                                const int np = j == p.p1 - 1 ? p.rows16 - j * p.n1 : p.n1;
                                const uint32_t idesc1 = ptx::idesc_bf16_f32(128, np);
                                const uint64_t qd = ptx::sw128_kmajor_desc(q_addr + j * p.n1 * 128);
                                const uint64_t kd = ptx::sw128_kmajor_desc(kbase);
#pragma unroll
                                for (int ks = 0; ks < D / 16; ++ks) {
                                    const uint32_t qo = ((ks >> 2) * qhalf + (ks & 3) * 32) >> 4;
                                    const uint32_t ko = ((ks >> 2) * kHalfTile + (ks & 3) * 32) >> 4;
                                    ptx::mma_bf16_ss(d0, kd + ko, qd + qo, idesc1, ks > 0);
                                }
                            }
                            ptx::mma_commit(&sb->accfull[st]);
                        }
                        if (!ok) break;
                        ptx::mma_commit(&sb->kempty[s]);
                        KVP_TSTAMP(phase * n + i, 3);
                    }
                    if (!ok) break;
                    // release the query rows when the next segment loads another head's
                    {
                        RunIter peek = it;
                        int nh = -1;
                        long long na, nb;
                        bool more = peek.next(nh, na, nb);
                        if (!more && phase == 0) {
                            RunIter again(t0, t1, p.tiles_per_head);
                            more = again.next(nh, na, nb);
                        }
                        if (more && nh != cur) ptx::mma_commit(&sb->qempty);
                    }
                }
                KVP_STAMP(3 + phase);
            }
            // every MMA issued by this thread completes before TMEM is released, also when
            // the CTA unwinds
            ptx::mma_commit(&sb->fin);
            drain_wait(&sb->fin, 0);
        }
    } else if (warp < kWarpEpi) {
        // ------------------------------------------------------------ S2: max |V| per key
        const int k2 = threadIdx.x - 32 * kWarpS2;          // 0 .. 63: keys k2 and k2 + 64
        bool ok = true;
        for (int i = 0; i < n && ok; ++i) {
            const int jv = i % p.nv1, vuse = i / p.nv1;
            if (!(ok = wait_phase(&sb->vfull[jv], vuse & 1, sb, p, kErrWaitS2))) break;
            const uint8_t* vt = Slots + (p.nk1 + jv) * kSlotBytes;
            const float ra = row_absmax<D>(vt + k2 * (D * 2), lane);
            const float rb = row_absmax<D>(vt + (k2 + 64) * (D * 2), lane);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sb->vempty[jv]);
            const int e = i & (kS2Bufs - 1), use = i / kS2Bufs;
            if (!(ok = wait_phase(&sb->s2empty[e], (use & 1) ^ 1, sb, p, kErrWaitS2))) break;
            s2buf[e * kTile + k2] = ra;
            s2buf[e * kTile + k2 + 64] = rb;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sb->s2full[e]);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 32 * kWarpEpi;      // 0 .. kEpiThreads-1
        const int eg = et >> 7;                           // epilogue group
        const int quarter = warp & 3;                     // TMEM lane quarter of this warp
        const int lq = quarter * 32 + lane;               // lane: query row (phase 0) / key (phase 1)
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);
        const int window0 = p.L - p.w;                    // first window position
        uint32_t epi_phase = 0;
        bool ok = true;
        // ---- phase 0: per query row, the running offset and sum of 2^(t - m) over the keys
        //      of this group's units (thread = row, TMEM columns = keys)
        {
            // last visible key of this thread's row in each row block
            int lim[4];
#pragma unroll
            for (int rb = 0; rb < 4; ++rb) lim[rb] = window0 + (rb * 128 + lq) % p.w;
            // chunks of a unit that hold rows of this warp: all rows of a row block
            // are live or none, and live chunks are a prefix of the unit's four
            const int rbl = p.rows > quarter * 32 ? min(p.nrb, (p.rows - quarter * 32 + 127) / 128) : 0;
            const int nl = min(4, rbl << p.lg_cpb);
            const int cmask = (1 << p.lg_cpb) - 1;
            RunIter it(t0, t1, p.tiles_per_head);
            int head;
            long long a, b;
            int unit = 0, i = 0;
            while (ok && it.next(head, a, b)) {
                float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                float l[4] = {0.f, 0.f, 0.f, 0.f};
                for (long long t = a; t < b && ok; ++t, ++i) {
                    const int key_t = (int)(t - (long long)head * p.tiles_per_head) * kTile;
                    for (int j = 0; j < p.u0; ++j, ++unit) {
                        if ((unit & 1) != eg) continue;      // the other group's unit
                        const int st = unit & (kStages - 1);
                        if (!(ok = wait_phase(&sb->accfull[st], (unit / kStages) & 1, sb, p, kErrWaitEpi))) break;
                        if (lq == 0) KVP_TSTAMP(i, 4);
                        ptx::tc_fence_after();
                        const int kbase = key_t + j * p.nk0;
                        const uint32_t tst = tlane + (uint32_t)(st * kStageCols);
                        // chunk c: TMEM columns [32c, 32c + 32) of the stage, row block c >> lg_cpb,
                        // keys kbase + 32 (c & cmask) + e
                        auto proc = [&](float (&v)[32], int c) {
                            const int rb = c >> p.lg_cpb;
                            const int j0 = kbase + ((c & cmask) << 5);
                            if (j0 + 31 > window0) {         // window or ragged keys: mask per row
                                const int rel = pick4(lim, rb) - j0;
#pragma unroll
                                for (int e = 0; e < 32; ++e)
                                    if (e > rel) v[e] = -INFINITY;
                            }
                            float mr = pick4(m, rb), lr = pick4(l, rb);
                            lse_chunk(v, p.scale2, mr, lr);
                            put4(m, rb, mr);
                            put4(l, rb, lr);
                        };
                        if (nl > 0) {
                            float x[32], y[32];
                            __syncwarp();
                            ptx::tmem_ld_32x32b_x32(tst, x);
                            ptx::tmem_ld_wait(x);
#pragma unroll 1
                            for (int c = 0; c < nl; c += 2) {
                                const bool h1 = c + 1 < nl, h2 = c + 2 < nl;
                                if (h1) {
                                    __syncwarp();
                                    ptx::tmem_ld_32x32b_x32(tst + (c + 1) * 32, y);
                                }
                                proc(x, c);
                                if (h1) {
                                    ptx::tmem_ld_wait(y);
                                    if (h2) {
                                        __syncwarp();
                                        ptx::tmem_ld_32x32b_x32(tst + (c + 2) * 32, x);
                                    }
                                    proc(y, c + 1);
                                    if (h2) ptx::tmem_ld_wait(x);
                                }
                            }
                        }
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&sb->accempty[st]);
                        if (lq == 0) KVP_TSTAMP(i, 5);
                    }
                }
                if (!ok) break;
                // Combine the two groups' (m, l) of every row, then publish one slot per row.
                if (!(ok = epi_sync(sb, epi_phase, p))) break;   // stage0 free again
                if (eg == 1) {
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const int r = rb * 128 + lq;
                        if (rb < p.nrb && r < p.rows) stage0[r] = make_float2(m[rb], l[rb]);
                    }
                }
                if (!(ok = epi_sync(sb, epi_phase, p))) break;
                if (eg == 0) {
                    const long long first = (long long)head * p.tiles_per_head;
                    const int slot = (int)blockIdx.x - owner_of(first, T, p.grid, p.tiles_per_head, p.cph);
                    const int r0 = group_row0(head);
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) {
                        const int r = rb * 128 + lq;
                        if (rb < p.nrb && r < p.rows) {
                            const float2 o = stage0[r];
                            const float M = fmaxf(m[rb], o.x);
                            float S = 0.f;
                            if (M != -INFINITY) S = l[rb] * ptx::ex2(m[rb] - M) + o.y * ptx::ex2(o.x - M);
                            if (KVP_CHECK(slot >= 0 && slot < p.maxslots, 202, slot, head))
                                p.part[(size_t)(r0 + r) * p.maxslots + slot] = make_float2(M, S);
                        }
                    }
                    __threadfence();
                }
                if (!(ok = epi_sync(sb, epi_phase, p))) break;
                if (et == 0) {
                    __threadfence();
                    atomicAdd(p.done + head, 1u);
                }
            }
        }
        if (et == 0) KVP_STAMP(5);
        // ---- phase 1: scores (thread = key, TMEM columns = query rows)
        {
            bool first_seg = true;
            RunIter it(t0, t1, p.tiles_per_head);
            int head;
            long long a, b;
            int unit = 0, i = 0;
            while (ok && it.next(head, a, b)) {
                const long long first = (long long)head * p.tiles_per_head;
                const int touch = owner_of(first + p.tiles_per_head - 1, T, p.grid, p.tiles_per_head, p.cph) -
                                  owner_of(first, T, p.grid, p.tiles_per_head, p.cph) + 1 + p.extra_peers;
                // the previous head's lse2 is no longer in use
                if (!(ok = epi_sync(sb, epi_phase, p))) break;
                if (et == 0) {
                    const uint64_t ts = ptx::globaltimer_ns();
                    while (ptx::ld_acquire_u32(p.done + head) < (uint32_t)touch) {
                        if (*(volatile int*)&sb->abort_flag) break;
                        if (ptx::globaltimer_ns() - ts > p.wait_limit_ns) {
                            atomicCAS(p.err, 0, kErrWaitPeers);
                            *(volatile int*)&sb->abort_flag = 1;
                            break;
                        }
                        __nanosleep(128);
                    }
                }
                if (!(ok = epi_sync(sb, epi_phase, p))) break;
                if (et == 0 && first_seg) KVP_STAMP(6);
                first_seg = false;
                if (*(volatile int*)&sb->abort_flag) {
                    ok = false;
                    break;
                }
                const int r0 = group_row0(head);
                const int nslots = (touch - p.extra_peers) * kSlotsPerCta;
                // Two threads per row, each over every other slot: first the row's
                // maximum, then the sum of l 2^(m - max); every load and term independent.
                for (int base = 0; base < 2 * p.rows; base += kEpiThreads) {
                    const int r2 = base + et, r = r2 >> 1;
                    const float2* pr = p.part + (size_t)(r0 + (r < p.rows ? r : 0)) * p.maxslots;
                    float M = -INFINITY;
                    if (r < p.rows) {
#pragma unroll 4
                        for (int sl = r2 & 1; sl < nslots; sl += 2) {
                            const float2 ml = __ldcg(pr + sl);
                            if (ml.y != 0.f) M = fmaxf(M, ml.x);
                        }
                    }
                    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 1));
                    float S = 0.f;
                    if (r < p.rows && M != -INFINITY) {
#pragma unroll 4
                        for (int sl = r2 & 1; sl < nslots; sl += 2) {
                            const float2 ml = __ldcg(pr + sl);
                            if (ml.y != 0.f) S += ml.y * ptx::ex2(ml.x - M);
                        }
                    }
                    S += __shfl_xor_sync(0xffffffffu, S, 1);
                    if (r < p.rows && (r2 & 1) == 0) lse2[r] = M + __log2f(S);
                }
                if (!(ok = epi_sync(sb, epi_phase, p))) break;
                for (long long t = a; t < b && ok; ++t, ++i) {
                    const int j = (int)(t - first) * kTile + lq;     // this thread's key
                    const int jw = j - window0;                      // > 0 only inside the window
                    // masks (window keys) are decided per warp: TMEM loads are warp-collective,
                    // so every lane takes the same path
                    const bool win = __any_sync(0xffffffffu, jw > 0);
                    float acc = 0.f;
                    bool mine = false;
                    for (int pp = 0; pp < p.p1; ++pp, ++unit) {
                        if ((unit & 1) != eg) continue;
                        mine = true;
                        const int st = unit & (kStages - 1);
                        const int use = ring_uses(st, kStages, U0) + unit / kStages;
                        if (!(ok = wait_phase(&sb->accfull[st], use & 1, sb, p, kErrWaitEpi))) break;
                        if (lq == 0) KVP_TSTAMP(n + i, 4);
                        ptx::tc_fence_after();
                        const uint32_t tst = tlane + (uint32_t)(st * kStageCols);
                        const int col0 = pp * p.n1;
                        const int ncols = min(p.n1, p.rows - col0);
                        const int nch = (ncols + 31) >> 5;
                        auto proc = [&](const float (&v)[32], int c) {
                            const int nrem = ncols - c * 32;
                            acc += s1_chunk(v, lse2 + col0 + c * 32, wpos + col0 + c * 32,
                                            win || nrem < 32, jw, nrem, p.scale2);
                        };
                        float x[32], y[32];
                        __syncwarp();
                        ptx::tmem_ld_32x32b_x32(tst, x);
                        ptx::tmem_ld_wait(x);
#pragma unroll 1
                        for (int c = 0; c < nch; c += 2) {
                            const bool h1 = c + 1 < nch, h2 = c + 2 < nch;
                            if (h1) {
                                __syncwarp();
                                ptx::tmem_ld_32x32b_x32(tst + (c + 1) * 32, y);
                            }
                            proc(x, c);
                            if (h1) {
                                ptx::tmem_ld_wait(y);
                                if (h2) {
                                    __syncwarp();
                                    ptx::tmem_ld_32x32b_x32(tst + (c + 2) * 32, x);
                                }
                                proc(y, c + 1);
                                if (h2) ptx::tmem_ld_wait(x);
                            }
                        }
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&sb->accempty[st]);
                        if (lq == 0) KVP_TSTAMP(n + i, 5);
                    }
                    if (!ok || !mine) continue;
                    if (p.p1 > 1) {
                        // the tile's rows are split over both groups: the group of the last part
                        // finishes the tile, the other hands over its partial S1
                        const int fin = (i * p.p1 + p.p1 - 1) & 1;
                        const int cb = i & (kCombBufs - 1), cuse = i / kCombBufs;
                        if (eg != fin) {
                            if (!(ok = wait_phase(&sb->combempty[cb], (cuse & 1) ^ 1, sb, p, kErrWaitEpi))) break;
                            comb[cb * kTile + lq] = acc;
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(&sb->combfull[cb]);
                            continue;
                        }
                        if (!(ok = wait_phase(&sb->combfull[cb], cuse & 1, sb, p, kErrWaitEpi))) break;
                        acc += comb[cb * kTile + lq];
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&sb->combempty[cb]);
                    }
                    const int e = i & (kS2Bufs - 1), suse = i / kS2Bufs;
                    if (!(ok = wait_phase(&sb->s2full[e], suse & 1, sb, p, kErrWaitEpi))) break;
                    const float s2v = s2buf[e * kTile + lq];
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sb->s2empty[e]);
                    if (j < p.L) {
                        const size_t o = (size_t)head * p.L + j;
                        p.score[o] = acc * s2v;
                        if (p.s1) p.s1[o] = acc;
                        if (p.s2) p.s2[o] = s2v;
                    }
                }
            }
        }
    }

    if (threadIdx.x == 32 * kWarpEpi) KVP_STAMP(7);
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace
}  // namespace kvp

namespace kvp {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// bf16 tensor map of `rank` dims (innermost first), tile box `box`.
bool make_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides_bytes, const cuuint32_t* box, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                    strides_bytes, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct Launch {
    Params p;
    int grid;
    size_t smem;
};

// Fault injection for the tests of a debug build: peers a head waits for that never
// arrive, and the limit of every wait. Release builds keep the defaults.
int g_extra_peers = 0;
unsigned long long g_wait_limit_ns = kWaitLimitNs;

bool build_launch(const kvp_shape& s, const Plan& plan, int sms, Launch* L) {
    Params& p = L->p;
    const int D = s.head_dim;
    p.L = s.seq_len;
    p.w = s.window;
    p.G = plan.G;
    p.rows = plan.rows;
    p.hq = s.hq;
    p.hkv = s.hkv;
    // phase 0: row blocks of 128 query rows; a unit covers nk0 keys of every row block in
    // 128 TMEM columns (4 chunks of 32 per thread)
    p.nrb = (plan.rows + 127) / 128;
    p.nk0 = p.nrb == 1 ? 128 : p.nrb == 2 ? 64 : 32;
    p.u0 = kTile / p.nk0;
    p.lg_cpb = p.nk0 == 128 ? 2 : p.nk0 == 64 ? 1 : 0;
    // phase 1: the query rows in p1 parts of n1 (a multiple of 16, at most 128) rows
    p.rows16 = (plan.rows + 15) / 16 * 16;
    p.p1 = (p.rows16 + kStageCols - 1) / kStageCols;
    p.n1 = ((p.rows16 + p.p1 - 1) / p.p1 + 15) / 16 * 16;
    p.tiles_per_head = plan.tiles_per_head;
    p.total_tiles = plan.total_tiles;
    // the planned cut, or a flat cut over the SMs of a smaller device
    p.cph = plan.grid <= sms ? plan.cph : 0;
    p.grid = plan.grid <= sms ? plan.grid : sms;
    // slots each head needs with this grid must fit the workspace's
    {
        const long long T = p.total_tiles;
        int need = 0;
        for (int h = 0; h < s.batch * s.hkv; ++h) {
            const long long f = (long long)h * p.tiles_per_head;
            need = std::max(need, owner_of(f + p.tiles_per_head - 1, T, p.grid, p.tiles_per_head, p.cph) -
                                      owner_of(f, T, p.grid, p.tiles_per_head, p.cph) + 1);
        }
        if (need * kSlotsPerCta > plan.maxslots) return false;
    }
    p.maxslots = plan.maxslots;
    p.scale2 = 1.4426950408889634f / sqrtf((float)D);
    p.qrows = (plan.rows + kQBoxRows - 1) / kQBoxRows * kQBoxRows;
    p.q_bytes = (uint32_t)p.qrows * D * 2;
    p.tile_bytes = (uint32_t)kTile * D * 2;
    p.extra_peers = g_extra_peers;
    p.wait_limit_ns = g_wait_limit_ns;
    // shared memory: Q | ring slots | lse2 | comb | s2buf | stage0 | wpos | barriers
    // (+1 KB to align the base)
    const size_t lse_bytes = (size_t)((plan.rows + 3) / 4 * 4) * sizeof(float);
    const size_t comb_bytes = (size_t)kCombBufs * kTile * sizeof(float);
    const size_t s2_bytes = (size_t)kS2Bufs * kTile * sizeof(float);
    const size_t stage_bytes = (size_t)plan.rows * sizeof(float2);
    const size_t wpos_bytes = (size_t)((plan.rows + 7) / 8 * 8) * sizeof(uint16_t);
    const size_t fixed = lse_bytes + comb_bytes + s2_bytes + stage_bytes + wpos_bytes + kBarBytes + 1024;
    if (p.q_bytes + fixed > (size_t)kSmemLimit) return false;
    p.ns = (int)std::min<size_t>(kMaxSlots, ((size_t)kSmemLimit - p.q_bytes - fixed) / p.tile_bytes);
    if (p.ns < 2) return false;
    // phase 1: K comes again (mostly from L2), V from HBM gets the deeper share; a tile
    // split into several parts holds its K slot longer, so one K slot can do
    p.nk1 = (p.p1 > 1 && p.ns <= 3) ? 1 : 2;
    p.nv1 = p.ns - p.nk1;
    if (p.nv1 < 1) return false;
    p.off_slots = p.q_bytes;
    uint32_t off = p.off_slots + (uint32_t)p.ns * p.tile_bytes;
    p.off_lse = off;
    off += (uint32_t)lse_bytes;
    p.off_comb = off;
    off += (uint32_t)comb_bytes;
    p.off_s2 = off;
    off += (uint32_t)s2_bytes;
    p.off_stage = off;
    off += (uint32_t)stage_bytes;
    p.off_wpos = off;
    off += (uint32_t)wpos_bytes;
    off = (off + 15) & ~15u;
    p.off_bar = off;
    off += (uint32_t)kBarBytes;
    static_assert(sizeof(SmemBars) <= kBarBytes, "barrier block");
    L->grid = p.grid;
    L->smem = std::max<size_t>((size_t)off + 1024, (size_t)kMinSmem);
    return L->smem <= (size_t)kSmemLimit;
}

}  // namespace

cudaError_t launch_score(const kvp_shape& s, const Plan& plan, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, void* workspace, float* score, float* s1, float* s2,
                         cudaStream_t st) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    Launch Lc;
    if (!build_launch(s, plan, sms, &Lc)) return cudaErrorInvalidConfiguration;
    Params& p = Lc.p;
    char* ws = (char*)workspace;
    p.done = (uint32_t*)(ws + plan.off_done);
    p.err = (int*)(ws + plan.off_err);
    p.part = (float2*)(ws + plan.off_part);
    p.score = score;
    p.s1 = s1;
    p.s2 = s2;

    const int D = s.head_dim;
    const cuuint64_t bh = (cuuint64_t)s.batch * s.hkv;
    CUtensorMap qmap, kmap, vmap;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)s.batch * s.hq * s.window};
        const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
        const cuuint32_t box[2] = {64, kQBoxRows};
        if (!make_map(&qmap, q, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)s.seq_len, bh};
        const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)s.seq_len * D * 2};
        const cuuint32_t kbox[3] = {64, kTile, 1};
        const cuuint32_t vbox[3] = {(cuuint32_t)D, kTile, 1};
        if (!make_map(&kmap, k, 3, dims, strides, kbox, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        if (!make_map(&vmap, v, 3, dims, strides, vbox, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    // the error word, then the completion counters, start at zero on every call
    if ((e = cudaMemsetAsync(ws + plan.off_err, 0, plan.off_part - plan.off_err, st)) != cudaSuccess)
        return e;

    void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const Params) =
        D == 128 ? score_fused_tc<128> : score_fused_tc<64>;
    if ((e = allow_dynamic_smem((const void*)kern, Lc.smem)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(Lc.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Lc.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: peers can be awaited
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, qmap, kmap, vmap, p);
}

#ifdef KVP_CHECKS
KVP_DEFINE_CHECK_READER(take_check_score)
// Debug builds only: make every later scoring call wait for `extra_peers` completions per
// head that never come, and give up any wait after `wait_limit_ns`.
void set_fault(int extra_peers, unsigned long long wait_limit_ns) {
    g_extra_peers = extra_peers;
    g_wait_limit_ns = wait_limit_ns ? wait_limit_ns : kWaitLimitNs;
}
#endif
#ifdef KVP_TRACE
int take_trace(unsigned long long* out) {
    if (cudaMemcpyFromSymbol(out, g_kvp_trace, sizeof(g_kvp_trace)) != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(out + 148 * 8, g_kvp_ttrace, sizeof(g_kvp_ttrace)) != cudaSuccess) return -1;
    return cudaMemcpyFromSymbol(out + 148 * 8 + 4 * 64 * 8, g_kvp_mtrace, sizeof(g_kvp_mtrace)) == cudaSuccess ? 0 : -1;
}
#endif

}  // namespace kvp
