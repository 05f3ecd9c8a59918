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
// swept twice; both sweeps run inside one kernel. Each CTA owns one or two segments of
// consecutive 128-key tiles (of different KV heads, when two), and sweeps phase 0 over all
// of them before phase 1, so that the wait for one head's other CTAs overlaps the next
// head's phase 0.
//   phase 0 (log-sum-exp; one query row per thread): tcgen05 computes
//     D[row, key] = Q_group[row] . K_tile[key]  (M = 128 rows of one row block, N = keys),
//     so each epilogue thread owns one query row (a TMEM lane) and keeps its running
//     offset m and sum l = sum_j 2^(t_j - m) in registers, t = logit * log2(e) / sqrt(d).
//     At the end of each segment a CTA publishes one (m, l) slot per row to the workspace
//     and bumps the head's completion counter.
//   phase 1 (scores; one key per thread): the same tiles again (K now mostly from L2),
//     with D[key, row] = K_tile[key] . Q_group[row]  (M = 128 keys, N = query rows).
//     Before its first tile of a head a CTA waits (bounded) until every CTA touching the
//     head has published, then merges the slots into lse2 = M + log2(sum_s l_s 2^(m_s-M))
//     per row. Per tile each thread sums 2^(t - lse2) over its key's query rows: S1.
//   S2 comes from phase 1's V tiles (V streams from HBM beside phase 1's K, which comes
//     mostly from L2: phase 0 streams K alone, so that K stays in L2). Each V tile is cut
//     into 4 pieces of 32 keys; warps 2 and 3 claim the next piece (in order, through a
//     shared counter) and reduce it into a ring of per-tile S2 rows in shared memory, which
//     the tile's finishing warps read. No busy warp holds up the V stream.
// Query rows: a CTA has at most a few runs of one head each (two with the head-aligned
// cut); when shared memory allows, every run's query block stays resident (two blocks), so
// that neither a change of head nor the phase boundary waits for query rows to load again.
// Warp roles: warp 0 issues the TMA loads (a ring of tile slots in shared memory, and the
// group's query rows); warp 1 allocates TMEM and issues the MMAs from one thread; warp 2
// combines the epilogue groups' phase 0 sums and publishes them (so that no epilogue thread
// waits on a global fence), then reduces V pieces like warp 3; four epilogue warpgroups (warps
// 4-19, one TMEM lane quarter per warp) read the accumulators. TMEM holds four accumulator
// stages of 128 columns, stage s belonging to epilogue group s. A tile's work is cut into
// units of at most 128 columns (phase 0: a run of keys over every row block; phase 1: a
// part of the query rows), and unit k takes stage k % 4, so four units are in flight and
// each group has four units' time for one.
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
constexpr int kStages = 4;                        // TMEM accumulator stages
constexpr int kGroups = kStages;                  // epilogue warpgroups, one per stage
constexpr int kStageCols = 128;                   // TMEM columns per stage
constexpr uint32_t kTmemCols = kStages * kStageCols;
constexpr int kWarpPub = 2;                       // the warp that publishes phase 0 sums
constexpr int kWarpV = 3;                         // a warp that only reduces V pieces (and warp 2,
                                                  // once it has published phase 0)
constexpr int kWarpEpi = 4;                       // first epilogue warp
constexpr int kEpiThreads = 128 * kGroups;
constexpr int kThreads = 32 * kWarpEpi + kEpiThreads;
constexpr int kMaxSlots = 8;                      // tile slots of the load ring
constexpr int kCombBufs = 4;                      // partial-S1 hand-off buffers (one tile each)
constexpr int kS2Ring = 8;                        // per-tile S2 rows in shared memory
constexpr int kVPieces = 4;                       // pieces of 32 keys per V tile
constexpr int kMaxParts = 4;                      // phase 1 parts per tile (512 rows / 128)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s on any single wait
#ifdef KVP_TRACE
constexpr int kSmemLimit = 227 * 1024 - 10240;   // the trace's static shared arrays take 10 KB
#else
constexpr int kSmemLimit = 227 * 1024;
#endif
constexpr int kMinSmem = 116 * 1024;              // forces one CTA per SM (TMEM is taken whole)
constexpr int kQBoxRows = 64;
constexpr size_t kBarBytes = 704;                 // shared memory reserved for SmemBars
#ifndef KVP_MAX_QBUFS
#define KVP_MAX_QBUFS 2
#endif
constexpr int kMaxQBufs = KVP_MAX_QBUFS;          // resident query blocks (one per run of a head)
constexpr float kSumLimit = 1.8446744e19f;        // 2^64: a chunk sum above it raises the offset

#ifdef KVP_TRACE
// Debug builds only: %globaltimer stamps per CTA at phase boundaries.
// [cta][0..7]: phase boundaries; [8]: SM id
__device__ unsigned long long g_kvp_trace[kPlanGrid][12];
#define KVP_STAMP(i) (g_kvp_trace[blockIdx.x][(i)] = ptx::globaltimer_ns())
// per-tile events of four CTAs, [cta][tile][event]: kept in shared memory while the kernel
// runs (no global stores or fences in the traced roles) and copied out at the end
__device__ unsigned long long g_kvp_ttrace[4][64][8];
__device__ unsigned long long g_kvp_mtrace[4][64][12];
__shared__ unsigned long long s_kvp_ttrace[64][8];
__shared__ unsigned long long s_kvp_mtrace[64][12];
#define KVP_MSTAMP(t, e) ((t) < 64 ? (void)(s_kvp_mtrace[(t)][(e)] = ptx::globaltimer_ns()) : (void)0)
__device__ __forceinline__ int kvp_trace_slot() {
    return blockIdx.x == 0 ? 0 : blockIdx.x == 18 ? 1 : blockIdx.x == 73 ? 2 : blockIdx.x == 143 ? 3 : -1;
}
#define KVP_TSTAMP(t, e) ((t) < 64 ? (void)(s_kvp_ttrace[(t)][(e)] = ptx::globaltimer_ns()) : (void)0)
#else
#define KVP_STAMP(i) ((void)0)
#define KVP_TSTAMP(t, e) ((void)0)
#define KVP_MSTAMP(t, e) ((void)0)
#endif

// error codes recorded in the workspace (first one wins)
enum : int { kErrWaitTma = 1, kErrWaitMma = 2, kErrWaitEpi = 3, kErrWaitPeers = 4, kErrWaitS2 = 5 };

struct Params {
    int L, w, rows, hq, hkv, G;
    int nrb, u0;               // phase 0: row blocks of 128 query rows; units per tile (one per block)
    int p1, n1, rows16;        // phase 1: parts per tile, rows per part, rows rounded up to 16
    int qrows;                 // query rows staged in shared memory (rows rounded up to 64)
    int nqb;                   // query blocks resident in shared memory (1 or 2)
    int qreuse;                // every CTA has at most nqb runs: phase 1 reuses phase 0's blocks
    int tiles_per_head, total_tiles, grid, cph, nseg, maxslots;
    int ns, nk, nv;            // ring slots; phase 1 gives K slots [0, nk), V slots [nk, ns)
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
    uint64_t vfull[kMaxSlots], vempty[kMaxSlots];   // per phase 1 V slot (index s - nk)
    uint64_t accfull[kStages], accempty[kStages];
    uint64_t combfull[kCombBufs], combempty[kCombBufs];
    uint64_t s2full[kS2Ring], s2empty[kS2Ring];     // per S2 ring row: its pieces, its readers
    uint64_t pubfull[2], pubempty[2];               // phase 0 sums of a segment, per buffer
    uint64_t lsefull[2], lseempty[2];               // phase 1 lse2 of a segment, per buffer
    uint64_t qfull[2], qempty[2];                   // per query block
    uint64_t fin;
    uint32_t tmem_base;
    int abort_flag;
};

// Wait for phase `parity` of `bar`; false if the CTA is unwinding or the wait timed out
// (then the first error code is recorded and the CTA told to unwind). After the first
// test the thread sleeps in the barrier (woken by the phase's completion, or after at most
// 20 us to look at the clock), so that waiting warps do not flood shared memory with
// polls while the TMA, the tensor cores and the working warps use it.
// The sleeping part is out of line (bounded_wait_slow): it is entered only when the first
// test fails, and one copy of it keeps the kernel's code small.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, SmemBars* sb,
                                           const Params& p, int code) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    return ptx::bounded_wait_slow(bar, parity, &sb->abort_flag, p.wait_limit_ns, p.err, code);
}

// wait_phase with the slow part inline, for the MMA thread: it keeps many values live
// across its waits, which a call would make it save to local memory.
__device__ __forceinline__ bool wait_inline(uint64_t* bar, uint32_t parity, SmemBars* sb,
                                            const Params& p, int code) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
        if (ptx::mbar_try_wait_sleep(bar, parity, 20000)) return true;
        if (*(volatile int*)&sb->abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > p.wait_limit_ns) {
            atomicCAS(p.err, 0, code);
            *(volatile int*)&sb->abort_flag = 1;
            return false;
        }
    }
}

// wait_phase for the roles whose warps work as a whole (S2, epilogue): the warp takes one
// decision for all its lanes, so that an abort seen by some lanes only can never split
// the warp in front of a warp barrier or a warp-collective TMEM load.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, SmemBars* sb,
                                          const Params& p, int code) {
    return __all_sync(0xffffffffu, wait_phase(bar, parity, sb, p, code));
}

// Wait for phase `parity` of `bar` for at most the wait limit, whatever the CTA's state:
// used before exit, so that no copy or MMA is still writing this CTA's memory.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait_sleep(bar, parity, 20000))
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) return;
}

// Per 16-bit half: a value whose magnitude is max(|a|, |b|) (its sign is the xor of the
// inputs' signs, which the caller masks off at the end).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// max |v| over the D bf16 values of one row in shared memory, read in 16-byte pieces in a
// rotated order per lane (consecutive lanes hit distinct bank groups), eight loads in flight
// at a time, each piece folded into its own running maximum.
template <int D>
__device__ __forceinline__ float row_absmax(const uint8_t* row, int lane) {
    constexpr int kPieces = D * 2 / 16;
    constexpr int kBatch = 8;
    const uint4* r = reinterpret_cast<const uint4*>(row);
    uint32_t m[kBatch];
#pragma unroll
    for (int c = 0; c < kBatch; ++c) m[c] = 0u;
#pragma unroll
    for (int c0 = 0; c0 < kPieces; c0 += kBatch) {
        uint4 x[kBatch];
#pragma unroll
        for (int c = 0; c < kBatch; ++c) x[c] = r[(c0 + c + lane) & (kPieces - 1)];
#pragma unroll
        for (int c = 0; c < kBatch; ++c)
            m[c] = bf16x2_absmax(m[c], bf16x2_absmax(bf16x2_absmax(x[c].x, x[c].y),
                                                     bf16x2_absmax(x[c].z, x[c].w)));
    }
#pragma unroll
    for (int h = kBatch / 2; h >= 1; h >>= 1)
#pragma unroll
        for (int c = 0; c < h; ++c) m[c] = bf16x2_absmax(m[c], m[c + h]);
    const uint32_t mx = m[0] & 0x7FFF7FFFu;
    return fmaxf(__uint_as_float(mx << 16), __uint_as_float(mx & 0xFFFF0000u));
}

// Uses of ring position s among the first n uses of a ring of `period` positions.
__device__ __forceinline__ int ring_uses(int s, int period, int n) {
    return n > s ? (n - s + period - 1) / period : 0;
}
// The CTA's work in one phase: its segments in order, each split where it crosses a KV
// head (only flat runs do), with the slot of the CTA's partial in that head.
// Tile numbers fit in 32 bits (the plan checks it).
struct CtaRun {
    const Params* p;
    int s, t, end;
    __device__ explicit CtaRun(const Params& prm) : p(&prm), s(-1), t(0), end(0) {}
    __device__ bool next(int& head, int& a, int& b, int& slot) {
        while (t >= end) {
            if (++s >= p->nseg) return false;
            uint32_t tb, te;
            segment_of_u32(blockIdx.x, s, p->total_tiles, p->grid, p->tiles_per_head, p->cph, tb, te);
            t = (int)tb;
            end = (int)te;
        }
        head = t / p->tiles_per_head;
        a = t;
        b = min(end, (head + 1) * p->tiles_per_head);
        t = b;
        slot = (int)slot_in_head_u32(blockIdx.x, s, head, p->total_tiles, p->grid, p->tiles_per_head, p->cph);
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

// Phase 1's V stream, for warps of their own (two share it): take the next piece
// (32 keys of a tile) by ticket, wait until its tile has landed and its S2 ring row is
// free, reduce each key to S2 = max |V| (one key per lane) into the ring, and release the
// piece's share of the V slot and of the ring row. A worker only ever waits on the barriers
// of a piece it holds, whose phases cannot move on before it is done. Every wait sleeps in
// the barrier and is bounded.
template <int D>
__device__ __forceinline__ void v_worker(uint8_t* smem, const Params& p, int n, SmemBars* sb) {
    constexpr uint32_t kSlotBytes = kTile * D * 2;
    constexpr int kKeys = kTile / kVPieces;               // keys per piece: one per lane
    static_assert(kKeys == 32, "one key per lane");
    const int lane = threadIdx.x & 31;
    const uint8_t* Slots = smem + p.off_slots;
    float* s2ring = (float*)(smem + p.off_s2);
    uint32_t* vclaim = (uint32_t*)(s2ring + kS2Ring * kTile);
    const uint32_t npieces = (uint32_t)(kVPieces * n);
    while (true) {
        uint32_t c = 0;
        if (lane == 0) c = atomicAdd(vclaim, 1u);
        c = __shfl_sync(0xffffffffu, c, 0);
        if (c >= npieces) break;
        const int vi = (int)(c / kVPieces), rs = vi & (kS2Ring - 1);
        if (vi >= kS2Ring && !wait_warp(&sb->s2empty[rs], (vi / kS2Ring - 1) & 1, sb, p, kErrWaitS2)) break;
        if (!wait_warp(&sb->vfull[vi % p.nv], (vi / p.nv) & 1, sb, p, kErrWaitS2)) break;
        if (lane == 0 && c % kVPieces == 0) KVP_MSTAMP(vi, 0);
        if (lane == 0) KVP_MSTAMP(vi, 3 + (int)(c % kVPieces));
        const int key = (int)(c % kVPieces) * kKeys + lane;
        const float s2 = row_absmax<D>(Slots + (p.nk + vi % p.nv) * kSlotBytes + key * (D * 2), lane);
        __syncwarp();                                     // every lane is done with the V slot
        if (lane == 0) ptx::mbar_arrive(&sb->vempty[vi % p.nv]);
        s2ring[rs * kTile + key] = s2;
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            ptx::mbar_arrive(&sb->s2full[rs]);
            if (c % kVPieces == kVPieces - 1) KVP_MSTAMP(vi, 1);
            KVP_MSTAMP(vi, 7 + (int)(c % kVPieces));
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
score_fused_tc(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* Qs = smem;                                  // [nqb][D / 64][qrows][64] bf16, 128B swizzle
    uint8_t* Slots = smem + p.off_slots;                 // ring slots of tile_bytes each
    float* lse2 = (float*)(smem + p.off_lse);            // [2][rows4]: a segment's lse2 per buffer
    float* comb = (float*)(smem + p.off_comb);           // [kCombBufs][kMaxParts - 1][128]
    float2* pub = (float2*)(smem + p.off_stage);         // [2][kGroups][rows] phase 0 (m, l)
    float* s2ring = (float*)(smem + p.off_s2);           // [kS2Ring][128] S2 of a tile's keys
    uint32_t* vclaim = (uint32_t*)(s2ring + kS2Ring * kTile);  // V piece tickets taken
    uint16_t* wpos = (uint16_t*)(smem + p.off_wpos);     // window position of query row n: n % w
    SmemBars* sb = (SmemBars*)(smem + p.off_bar);

    constexpr int kHalves = D / 64;                 // 128-byte swizzle rows per operand row
    constexpr uint32_t kHalfTile = kTile * 128;     // bytes of one 64-column half of a tile
    constexpr uint32_t kSlotBytes = kTile * D * 2;
    const uint32_t qhalf = (uint32_t)p.qrows * 128;  // bytes of one 64-column half of Q
    const int rows4 = (p.rows + 3) & ~3;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int n = 0;                                      // tiles in this CTA's run
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        if (s < p.nseg) {
            uint32_t b, e;
            segment_of_u32(blockIdx.x, s, p.total_tiles, p.grid, p.tiles_per_head, p.cph, b, e);
            n += (int)(e - b);
        }
    }
    const int U0 = n * p.u0;                        // phase 0 units of the run

    for (int r = threadIdx.x; r < p.rows; r += kThreads) wpos[r] = (uint16_t)(r % p.w);
    if (threadIdx.x == 0) *vclaim = 0u;
#ifdef KVP_TRACE
    for (int i = threadIdx.x; i < 64 * 8; i += kThreads) s_kvp_ttrace[i / 8][i % 8] = 0;
    for (int i = threadIdx.x; i < 64 * 12; i += kThreads) s_kvp_mtrace[i / 12][i % 12] = 0;
#endif
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxSlots; ++s) {
            ptx::mbar_init(&sb->kfull[s], 1);
            ptx::mbar_init(&sb->kempty[s], 1);
            ptx::mbar_init(&sb->vfull[s], 1);
            ptx::mbar_init(&sb->vempty[s], kVPieces);
        }
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&sb->accfull[s], 1);
            ptx::mbar_init(&sb->accempty[s], 4);
        }
        for (int s = 0; s < kS2Ring; ++s) {
            ptx::mbar_init(&sb->s2full[s], kVPieces);
            ptx::mbar_init(&sb->s2empty[s], 4);        // the finishing group's four warps
        }
        for (int s = 0; s < kCombBufs; ++s) {
            ptx::mbar_init(&sb->combfull[s], 4 * (p.p1 - 1 > 0 ? p.p1 - 1 : 1));
            ptx::mbar_init(&sb->combempty[s], 4);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&sb->pubfull[s], kEpiThreads / 32);
            ptx::mbar_init(&sb->pubempty[s], 1);
            ptx::mbar_init(&sb->lsefull[s], kEpiThreads / 32);
            ptx::mbar_init(&sb->lseempty[s], kEpiThreads / 32);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&sb->qfull[s], 1);
            ptx::mbar_init(&sb->qempty[s], 1);
        }
        ptx::mbar_init(&sb->fin, 1);
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
#ifdef KVP_TRACE
    if (threadIdx.x == 0) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        g_kvp_trace[blockIdx.x][8] = smid;
    }
#endif

    auto group_row0 = [&](int bh) {
        const int b = bh / p.hkv, h = bh % p.hkv;
        return (b * p.hq + h * p.G) * p.w;
    };


    // Roles are dispatched on whole warps: every lane of a warp takes the same branch, and a
    // single-lane role sits inside its warp's branch, so no lane can fall into another role.
    if (warp == 0) {
      if (lane == 0) {
        // ------------------------------------------------------------ TMA producer
        // K is read again by phase 1 (from L2 when it fits); V and phase 1's K stream
        const uint64_t pol_keep = ptx::policy_evict_normal();
        const uint64_t pol_stream = ptx::policy_evict_first();
        // Run r of a phase uses query block r % nqb; when every CTA has at most nqb runs, the
        // blocks loaded in phase 0 stay for phase 1, else every run loads its block again.
        int qgen0 = 0, qgen1 = 0;                           // loads into each query block
        // per slot, in registers: bit s = parity of the loads issued to it, and whether any was
        uint32_t kpar = 0, kused = 0, vpar = 0, vused = 0;
        int vs = 0;                                         // next V slot (index s - nk)
        bool ok = true;
        for (int phase = 0; phase < 2 && ok; ++phase) {
            // K goes round slots [0, ns) in phase 0 and [0, nk) in phase 1; the parity of a
            // slot's loads so far gives the phase of its barriers
            const int kring = phase == 0 ? p.ns : p.nk;
            int ks = 0;
            CtaRun it(p);
            int head, slot, a, b;
            int i = 0;                                      // tile number within the run
            int qb = p.nqb - 1;                             // query block of the run
            while (ok && it.next(head, a, b, slot)) {
                qb ^= p.nqb - 1;
                if (phase == 0 || !p.qreuse) {
                    const int qg = qb ? qgen1 : qgen0;
                    if (qg > 0 && !(ok = wait_phase(&sb->qempty[qb], (qg - 1) & 1, sb, p, kErrWaitTma))) break;
                    ptx::mbar_arrive_expect_tx(&sb->qfull[qb], p.q_bytes);
                    const int r0 = group_row0(head);
                    uint8_t* qdst = Qs + (size_t)qb * p.q_bytes;
                    for (int rb = 0; rb < p.qrows; rb += kQBoxRows)
                        for (int c = 0; c < kHalves; ++c)
                            ptx::tma_load_2d(qdst + c * qhalf + rb * 128, &qmap, &sb->qfull[qb],
                                             c * 64, r0 + rb, pol_keep);
                    if (qb) ++qgen1;
                    else ++qgen0;
                }
                for (int t = a; t < b; ++t, ++i) {
                    const int key0 = (t - head * p.tiles_per_head) * kTile;
                    const int s = ks;
                    ks = ks + 1 == kring ? 0 : ks + 1;
                    if (!(ok = wait_phase(&sb->kempty[s], ((kpar >> s) & 1) ^ 1, sb, p, kErrWaitTma))) break;
                    KVP_TSTAMP(phase * n + i, 0);
                    ptx::mbar_arrive_expect_tx(&sb->kfull[s], p.tile_bytes);
                    for (int c = 0; c < kHalves; ++c)
                        ptx::tma_load_3d(Slots + s * kSlotBytes + c * kHalfTile, &kmap, &sb->kfull[s],
                                         c * 64, key0, head, phase == 0 ? pol_keep : pol_stream);
                    kpar ^= 1u << s;
                    kused |= 1u << s;
                    if (phase == 1) {
                        const int jv = vs, sv = p.nk + jv;
                        vs = vs + 1 == p.nv ? 0 : vs + 1;
                        // a V slot's first load waits for its last K load of phase 0 to be consumed
                        if (!((vused >> jv) & 1) && ((kused >> sv) & 1) &&
                            !(ok = wait_phase(&sb->kempty[sv], ((kpar >> sv) & 1) ^ 1, sb, p, kErrWaitTma)))
                            break;
                        if (!(ok = wait_phase(&sb->vempty[jv], ((vpar >> jv) & 1) ^ 1, sb, p, kErrWaitTma))) break;
                        KVP_TSTAMP(n + i, 6);
                        ptx::mbar_arrive_expect_tx(&sb->vfull[jv], p.tile_bytes);
                        ptx::tma_load_3d(Slots + sv * kSlotBytes, &vmap, &sb->vfull[jv], 0, key0, head,
                                         pol_stream);
                        vpar ^= 1u << jv;
                        vused |= 1u << jv;
                    }
                }
            }
            KVP_STAMP(1 + phase);
        }
        // Never leave with copies in flight: wait for the last load issued to every slot
        // (these waits do not stop early when the CTA unwinds).
        for (int s = 0; s < p.ns; ++s)
            if ((kused >> s) & 1) drain_wait(&sb->kfull[s], ((kpar >> s) & 1) ^ 1);
        for (int jv = 0; jv < p.nv; ++jv)
            if ((vused >> jv) & 1) drain_wait(&sb->vfull[jv], ((vpar >> jv) & 1) ^ 1);
        if (qgen0 > 0) drain_wait(&sb->qfull[0], (qgen0 - 1) & 1);
        if (qgen1 > 0) drain_wait(&sb->qfull[1], (qgen1 - 1) & 1);
      }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t q_base = ptx::smem_u32(Qs), k_addr = ptx::smem_u32(Slots);
            const uint32_t idesc0 = ptx::idesc_bf16_f32(128, kTile);
            uint32_t qpar = 0;                              // bit b: parity of block b's loads waited for
            uint32_t kpar = 0;                              // bit s: parity of slot s's loads consumed
            uint32_t apar = 0;                              // bit st: parity of stage st's units
            bool ok = true;
            for (int phase = 0; phase < 2 && ok; ++phase) {
                const int kring = phase == 0 ? p.ns : p.nk;   // the producer's slot order
                int ks = 0;
                CtaRun it(p);
                int head, slot, a, b;
                int i = 0;                                  // tile number within the run
                int unit = 0;                               // unit number within the phase
                int qb = p.nqb - 1;                         // query block of the run
                while (ok && it.next(head, a, b, slot)) {
                    qb ^= p.nqb - 1;
                    if (phase == 0 || !p.qreuse) {
                        if (!(ok = wait_inline(&sb->qfull[qb], (qpar >> qb) & 1, sb, p, kErrWaitMma))) break;
                        qpar ^= 1u << qb;
                        ptx::tc_fence_after();
                    }
                    const uint32_t q_addr = q_base + (uint32_t)qb * p.q_bytes;
                    for (int t = a; t < b && ok; ++t, ++i) {
                        const int s = ks;
                        ks = ks + 1 == kring ? 0 : ks + 1;
                        if (!(ok = wait_inline(&sb->kfull[s], (kpar >> s) & 1, sb, p, kErrWaitMma))) break;
                        KVP_TSTAMP(phase * n + i, 1);
                        const uint32_t kbase = k_addr + s * kSlotBytes;
                        const int nunits = phase == 0 ? p.u0 : p.p1;
                        for (int j = 0; j < nunits; ++j, ++unit) {
                            const int st = unit & (kStages - 1);
                            if (!(ok = wait_inline(&sb->accempty[st], ((apar >> st) & 1) ^ 1, sb, p, kErrWaitMma))) break;
                            apar ^= 1u << st;
                            if (j == 0) KVP_TSTAMP(phase * n + i, 2);
                            ptx::tc_fence_after();
                            const uint32_t d0 = tmem + (uint32_t)(st * kStageCols);
                            if (phase == 0) {
                                // D[row, key] for row block j and the tile's 128 keys: A = Q rows,
                                // B = the K tile (each operand read once per unit)
                                const uint64_t qd = ptx::sw128_kmajor_desc(q_addr + j * 128 * 128);
                                const uint64_t kd = ptx::sw128_kmajor_desc(kbase);
#pragma unroll
                                for (int ks = 0; ks < D / 16; ++ks) {
                                    const uint32_t qo = ((ks >> 2) * qhalf + (ks & 3) * 32) >> 4;
                                    const uint32_t ko = ((ks >> 2) * kHalfTile + (ks & 3) * 32) >> 4;
                                    ptx::mma_bf16_ss(d0, qd + qo, kd + ko, idesc0, ks > 0);
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
                        kpar ^= 1u << s;
                        KVP_TSTAMP(phase * n + i, 3);
                    }
                    if (!ok) break;
                    // release the query block once its last MMA of this load has completed
                    if (phase == 1 || !p.qreuse) ptx::mma_commit(&sb->qempty[qb]);
                }
                KVP_STAMP(3 + phase);
            }
            // every MMA issued by this thread completes before TMEM is released, also when
            // the CTA unwinds
            ptx::mma_commit(&sb->fin);
            drain_wait(&sb->fin, 0);
        }
    } else if (warp == kWarpPub || warp == kWarpV) {
      bool ok = true;
      if (warp == kWarpPub) {
        // ------------------------------------------------------------ phase 0 publisher
        // Per segment: combine the epilogue groups' (m, l) of every row, write the CTA's
        // slot, then bump the head's completion counter (so that no epilogue thread waits on
        // a global fence).
        CtaRun it(p);
        int head, slot, a, b;
        int k = 0;
        while (ok && it.next(head, a, b, slot)) {
            const int buf = k & 1, use = k >> 1;
            if (!(ok = wait_warp(&sb->pubfull[buf], use & 1, sb, p, kErrWaitEpi))) break;
            const int r0 = group_row0(head);
            const float2* pbuf = pub + (size_t)buf * kGroups * p.rows;
            for (int r = lane; r < p.rows; r += 32) {
                float2 o[kGroups];
                float M = -INFINITY;
#pragma unroll
                for (int g = 0; g < kGroups; ++g) {
                    o[g] = pbuf[g * p.rows + r];
                    M = fmaxf(M, o[g].x);
                }
                float S = 0.f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int g = 0; g < kGroups; ++g) S += o[g].y * ptx::ex2(o[g].x - M);
                }
                if (KVP_CHECK(slot >= 0 && slot < p.maxslots, 202, slot, head))
                    p.part[(size_t)(r0 + r) * p.maxslots + slot] = make_float2(M, S);
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sb->pubempty[buf]);
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(p.done + head, 1u);
            ++k;
        }
        if (lane == 0) KVP_STAMP(5);
      }
      // ------------------------------------------------------------ V pieces (warps 2 and 3)
      if (ok) v_worker<D>(smem, p, n, sb);
    } else if (warp >= kWarpEpi) {
        // ------------------------------------------------------------ epilogue (warps 4-19)
        const int et = threadIdx.x - 32 * kWarpEpi;      // 0 .. kEpiThreads-1
        const int eg = et >> 7;                           // epilogue group = its TMEM stage
        const int quarter = warp & 3;                     // TMEM lane quarter of this warp
        const int lq = quarter * 32 + lane;               // lane: query row (phase 0) / key (phase 1)
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);
        const uint32_t tst = tlane + (uint32_t)(eg * kStageCols);
        const int window0 = p.L - p.w;                    // first window position
        bool ok = true;
        // ---- phase 0: per query row, the running offset and sum of 2^(t - m) over the keys
        //      of this group's units (thread = row, TMEM columns = keys)
        {
            CtaRun it(p);
            int head, slot, a, b;
            int unit = 0, i = 0, k = 0;
            while (ok && it.next(head, a, b, slot)) {
                float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                float l[4] = {0.f, 0.f, 0.f, 0.f};
                for (int t = a; t < b && ok; ++t, ++i) {
                    const int key_t = (t - head * p.tiles_per_head) * kTile;
                    for (int j = 0; j < p.u0; ++j, ++unit) {
                        if ((unit & (kStages - 1)) != eg) continue;   // another group's unit
                        if (!(ok = wait_warp(&sb->accfull[eg], (unit / kStages) & 1, sb, p, kErrWaitEpi))) break;
                        if (lq == 0) KVP_TSTAMP(i, 4);
                        ptx::tc_fence_after();
                        // unit j is row block j; chunk c: TMEM columns [32c, 32c + 32) of the
                        // stage, keys key_t + 32 c + e. A warp whose rows of the block all lie
                        // beyond the group's rows skips it (rows past the last are not published)
                        const int rb = j;
                        const int nl = rb * 128 + quarter * 32 < p.rows ? 4 : 0;
#pragma unroll 1
                        for (int c = 0; c < nl; ++c) {
                            float v[32];
                            __syncwarp();
                            ptx::tmem_ld_32x32b_x32(tst + c * 32, v);
                            ptx::tmem_ld_wait(v);
                            const int j0 = key_t + (c << 5);
                            if (j0 + 31 > window0) {         // window or ragged keys: mask per row
                                // the row's last visible key is window0 + its window position
                                const int rel = window0 + (rb * 128 + lq) % p.w - j0;
#pragma unroll
                                for (int e = 0; e < 32; ++e)
                                    if (e > rel) v[e] = -INFINITY;
                            }
                            float mr = pick4(m, rb), lr = pick4(l, rb);
                            lse_chunk(v, p.scale2, mr, lr);
                            put4(m, rb, mr);
                            put4(l, rb, lr);
                        }
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&sb->accempty[eg]);
                        if (lq == 0) KVP_TSTAMP(i, 5);
                    }
                }
                if (!ok) break;
                // hand this group's (m, l) of every row to the publisher and go on
                const int buf = k & 1, use = k >> 1;
                if (!(ok = wait_warp(&sb->pubempty[buf], (use & 1) ^ 1, sb, p, kErrWaitEpi))) break;
                float2* pb = pub + ((size_t)buf * kGroups + eg) * p.rows;
#pragma unroll
                for (int rb = 0; rb < 4; ++rb) {
                    const int r = rb * 128 + lq;
                    if (rb < p.nrb && r < p.rows) pb[r] = make_float2(m[rb], l[rb]);
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sb->pubfull[buf]);
                ++k;
            }
        }
        // Wait for `cond` (a warp-uniform test of memory that no barrier guards), polling;
        // bounded.
        auto pwait = [&](auto&& cond, int code) -> bool {
            if (cond()) return true;
            // the low 32 bits of the ns timer: they wrap every 4.29 s, above any wait limit
            const uint32_t t0 = (uint32_t)ptx::globaltimer_ns();
            while (true) {
                __nanosleep(256);
                if (cond()) return true;
                if (__any_sync(0xffffffffu, *(volatile int*)&sb->abort_flag != 0)) return false;
                // one decision for the warp: its lanes read the clock at slightly different times
                if (__any_sync(0xffffffffu, (uint32_t)ptx::globaltimer_ns() - t0 > (uint32_t)p.wait_limit_ns)) {
                    if (lane == 0) {
                        atomicCAS(p.err, 0, code);
                        *(volatile int*)&sb->abort_flag = 1;
                    }
                    return false;
                }
            }
        };
        auto bwait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return wait_warp(bar, parity, sb, p, kErrWaitEpi);
        };
        // ---- phase 1: scores (thread = key, TMEM columns = query rows)
        {
            bool first_seg = true;
            CtaRun it(p);
            int head, slot, a, b;
            int i = 0, k = 0;
            while (ok && it.next(head, a, b, slot)) {
                const int first = head * p.tiles_per_head;
                const int buf = k & 1, use = k >> 1;
                float* ls = lse2 + buf * rows4;
                // This group merges the head's slots into lse2 for its share of the rows (the
                // 32-row blocks b with b % 4 == eg), once the buffer is free and every CTA
                // touching the head has published.
                if (!(ok = bwait(&sb->lseempty[buf], (use & 1) ^ 1))) break;
                const int touch = (int)ctas_touching_u32(head, p.total_tiles, p.grid, p.tiles_per_head, p.cph);
                const uint32_t want = (uint32_t)(touch + p.extra_peers);
                if (!(ok = pwait([&]() {
                          uint32_t d = 0;
                          if (lane == 0) d = ptx::ld_acquire_u32(p.done + head);
                          return __shfl_sync(0xffffffffu, d, 0) >= want;
                      }, kErrWaitPeers)))
                    break;
                (void)ptx::ld_acquire_u32(p.done + head);     // every lane acquires the slots
                if (et == 0 && first_seg) KVP_STAMP(6);
                first_seg = false;
                const int r0 = group_row0(head);
                const int nslots = touch * kSlotsPerCta;
                // four threads per row, each over every fourth slot, in batches of kMergeBatch
                // loads issued before any is used (the slots come from L2, whose latency would
                // otherwise be paid once per slot); per batch, the offset is raised to the
                // batch's maximum first and the sum rescaled once
                constexpr int kMergeBatch = 12;
                for (int rr = (et & 127) >> 2; ; rr += 32) {
                    const int r = ((rr >> 5) * kGroups + eg) * 32 + (rr & 31);
                    if (__all_sync(0xffffffffu, r >= p.rows)) break;
                    const int q = et & 3;
                    float M = -INFINITY, S = 0.f;
                    if (r < p.rows) {
                        const float2* pr = p.part + (size_t)(r0 + r) * p.maxslots;
                        for (int s0 = q; s0 < nslots; s0 += 4 * kMergeBatch) {
                            float2 ml[kMergeBatch];
#pragma unroll
                            for (int u = 0; u < kMergeBatch; ++u)
                                ml[u] = s0 + 4 * u < nslots ? __ldcg(pr + s0 + 4 * u) : make_float2(0.f, 0.f);
                            float Mb = M;
#pragma unroll
                            for (int u = 0; u < kMergeBatch; ++u)
                                if (ml[u].y != 0.f) Mb = fmaxf(Mb, ml[u].x);
                            if (Mb > M) {
                                S *= ptx::ex2(M - Mb);             // M = -inf: S is 0 and stays 0
                                M = Mb;
                            }
#pragma unroll
                            for (int u = 0; u < kMergeBatch; ++u)
                                if (ml[u].y != 0.f) S += ml[u].y * ptx::ex2(ml[u].x - M);
                        }
                    }
#pragma unroll
                    for (int o = 1; o <= 2; o <<= 1) {
                        const float Mo = __shfl_xor_sync(0xffffffffu, M, o);
                        const float So = __shfl_xor_sync(0xffffffffu, S, o);
                        const float Mn = fmaxf(M, Mo);
                        S = (Mn == -INFINITY) ? 0.f : S * ptx::ex2(M - Mn) + So * ptx::ex2(Mo - Mn);
                        M = Mn;
                    }
                    if (r < p.rows && q == 0) ls[r] = M + __log2f(S);
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sb->lsefull[buf]);
                if (!(ok = bwait(&sb->lsefull[buf], use & 1))) break;
                for (int t = a; t < b && ok; ++t, ++i) {
                    const int j = (t - first) * kTile + lq;          // this thread's key
                    const int jw = j - window0;                      // > 0 only inside the window
                    // units of this tile: i * p1 + part, in stages (and groups) (i * p1 + part) % 4
                    const int u_first = i * p.p1;
                    const int pp = (eg - u_first) & (kStages - 1);   // this group's part, if any
                    if (pp >= p.p1) continue;                        // not this group's tile
                    const int myunit = u_first + pp;
                    // masks (window keys) are decided per warp: TMEM loads are warp-collective,
                    // so every lane takes the same path
                    const bool win = __any_sync(0xffffffffu, jw > 0);
                    const int ause = ring_uses(eg, kStages, U0) + myunit / kStages;
                    if (!(ok = bwait(&sb->accfull[eg], ause & 1))) break;
                    if (lq == 0) KVP_TSTAMP(n + i, 4);
                    ptx::tc_fence_after();
                    const int col0 = pp * p.n1;
                    const int ncols = min(p.n1, p.rows - col0);
                    const int nch = (ncols + 31) >> 5;
                    float acc = 0.f;
#pragma unroll 1
                    for (int c = 0; c < nch; ++c) {
                        float v[32];
                        __syncwarp();
                        ptx::tmem_ld_32x32b_x32(tst + c * 32, v);
                        ptx::tmem_ld_wait(v);
                        const int nrem = ncols - c * 32;
                        acc += s1_chunk(v, ls + col0 + c * 32, wpos + col0 + c * 32, win || nrem < 32,
                                        jw, nrem, p.scale2);
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sb->accempty[eg]);
                    if (lq == 0) KVP_TSTAMP(n + i, 5);
                    const int cb = i & (kCombBufs - 1), cuse = i / kCombBufs;
                    if (p.p1 > 1) {
                        // the tile's rows are split over p1 groups: the group of the last part
                        // finishes the tile, the others hand over their partial S1
                        if (pp != p.p1 - 1) {
                            if (!(ok = bwait(&sb->combempty[cb], (cuse & 1) ^ 1))) break;
                            comb[(cb * (kMaxParts - 1) + pp) * kTile + lq] = acc;
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(&sb->combfull[cb]);
                            continue;
                        }
                        // a plain wait: the part groups wait for their accumulators in waits
                        // that take V pieces, so the V stream goes on meanwhile
                        if (!(ok = wait_warp(&sb->combfull[cb], cuse & 1, sb, p, kErrWaitEpi))) break;
                        float others = 0.f;
                        for (int q = 0; q < p.p1 - 1; ++q) others += comb[(cb * (kMaxParts - 1) + q) * kTile + lq];
                        acc += others;
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&sb->combempty[cb]);
                    }
                    // the tile's S2, once its V pieces are in the ring; then the ring row is
                    // released (four warps of this group read it)
                    const int rs = i & (kS2Ring - 1);
                    if (!(ok = bwait(&sb->s2full[rs], (i / kS2Ring) & 1))) break;
                    if (lq == 0) KVP_MSTAMP(i, 2);
                    const float s2v = s2ring[rs * kTile + lq];
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sb->s2empty[rs]);
                    if (j < p.L) {
                        const size_t o = (size_t)head * p.L + j;
                        p.score[o] = acc * s2v;
                        if (p.s1) p.s1[o] = acc;
                        if (p.s2) p.s2[o] = s2v;
                    }
                }
                if (!ok) break;
                // this segment's lse2 is no longer read by this warp
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sb->lseempty[buf]);
                ++k;
            }
        }
    }

    if (threadIdx.x == 32 * kWarpEpi) KVP_STAMP(7);
    ptx::tc_fence_before();
    __syncthreads();
#ifdef KVP_TRACE
    if (kvp_trace_slot() >= 0) {
        for (int i = threadIdx.x; i < 64 * 8; i += kThreads)
            g_kvp_ttrace[kvp_trace_slot()][i / 8][i % 8] = s_kvp_ttrace[i / 8][i % 8];
        for (int i = threadIdx.x; i < 64 * 12; i += kThreads)
            g_kvp_mtrace[kvp_trace_slot()][i / 12][i % 12] = s_kvp_mtrace[i / 12][i % 12];
    }
#endif
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
    // phase 0: row blocks of 128 query rows; unit j of a tile covers row block j and the
    // tile's 128 keys in 128 TMEM columns (4 chunks of 32 per thread)
    p.nrb = (plan.rows + 127) / 128;
    p.u0 = p.nrb;
    // phase 1: the query rows in p1 parts of n1 (a multiple of 16, at most 128) rows
    p.rows16 = (plan.rows + 15) / 16 * 16;
    p.p1 = (p.rows16 + kStageCols - 1) / kStageCols;
    p.n1 = ((p.rows16 + p.p1 - 1) / p.p1 + 15) / 16 * 16;
    p.tiles_per_head = plan.tiles_per_head;
    p.total_tiles = plan.total_tiles;
    // the planned cut, or a flat cut over the SMs of a smaller device
    if (plan.grid <= sms) {
        p.grid = plan.grid;
        p.cph = plan.cph;
        p.nseg = plan.nseg;
    } else {
        p.grid = sms;
        p.cph = 0;
        p.nseg = 1;
        // slots each head needs with this grid must fit the workspace's
        int need = 0;
        for (int h = 0; h < s.batch * s.hkv; ++h)
            need = std::max(need, ctas_touching(h, p.total_tiles, p.grid, p.tiles_per_head, 0));
        if (need * kSlotsPerCta > plan.maxslots) return false;
    }
    p.maxslots = plan.maxslots;
    p.scale2 = 1.4426950408889634f / sqrtf((float)D);
    p.qrows = (plan.rows + kQBoxRows - 1) / kQBoxRows * kQBoxRows;
    p.q_bytes = (uint32_t)p.qrows * D * 2;
    p.tile_bytes = (uint32_t)kTile * D * 2;
    p.extra_peers = g_extra_peers;
    p.wait_limit_ns = g_wait_limit_ns;
    // shared memory: Q | ring slots | lse2 [2] | comb | S2 ring | phase 0 hand-off [2] | wpos | barriers
    // (+1 KB to align the base)
    const size_t lse_bytes = 2 * (size_t)((plan.rows + 3) / 4 * 4) * sizeof(float);
    const size_t comb_bytes = p.p1 > 1 ? (size_t)kCombBufs * (kMaxParts - 1) * kTile * sizeof(float) : 0;
    const size_t stage_bytes = 2 * (size_t)kGroups * plan.rows * sizeof(float2);
    const size_t s2_bytes = (size_t)kS2Ring * kTile * sizeof(float) + 16;
    const size_t wpos_bytes = (size_t)((plan.rows + 7) / 8 * 8) * sizeof(uint16_t);
    const size_t fixed = lse_bytes + comb_bytes + s2_bytes + stage_bytes + wpos_bytes + kBarBytes + 1024;
    // two query blocks (no reload when a CTA changes head) while the ring keeps four slots
    p.nqb = kMaxQBufs;
    while (p.nqb > 1 && (size_t)p.nqb * p.q_bytes + fixed + 4 * (size_t)p.tile_bytes > (size_t)kSmemLimit)
        --p.nqb;
    // the most runs any CTA has (a run: consecutive tiles of one head); one block is enough
    // when no CTA changes head
    int max_runs = 0;
    for (int c = 0; c < p.grid; ++c) {
        int runs = 0;
        for (int sg = 0; sg < p.nseg; ++sg) {
            long long b, e;
            segment_of(c, sg, p.total_tiles, p.grid, p.tiles_per_head, p.cph, b, e);
            if (e > b) runs += (int)((e - 1) / p.tiles_per_head - b / p.tiles_per_head + 1);
        }
        max_runs = std::max(max_runs, runs);
    }
    if (max_runs <= 1) p.nqb = 1;
    const size_t qall = (size_t)p.nqb * p.q_bytes;
    // phase 1 reuses phase 0's blocks when every CTA has at most nqb runs
    p.qreuse = max_runs <= p.nqb ? 1 : 0;
    if (qall + fixed > (size_t)kSmemLimit) return false;
    p.ns = (int)std::min<size_t>(kMaxSlots, ((size_t)kSmemLimit - qall - fixed) / p.tile_bytes);
    if (p.ns < 2) return false;
    // phase 0 streams K through every slot; phase 1 gives V (from HBM) the deeper share and
    // K (mostly from L2) two slots, or one when the ring is short
    p.nk = p.ns >= 4 ? 2 : 1;
    p.nv = p.ns - p.nk;
    if (p.nv < 1) return false;
    p.off_slots = (uint32_t)qall;
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

}  // namespace

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
    if (cudaMemcpyFromSymbol(out + 148 * 12, g_kvp_ttrace, sizeof(g_kvp_ttrace)) != cudaSuccess) return -1;
    return cudaMemcpyFromSymbol(out + 148 * 12 + 4 * 64 * 8, g_kvp_mtrace, sizeof(g_kvp_mtrace)) == cudaSuccess ? 0 : -1;
}
#endif

}  // namespace kvp
