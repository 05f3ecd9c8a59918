// S1 * S2 scoring on sm_100a: one persistent, warp-specialised tcgen05 kernel.
//
// "Preserving Large Activations: The Key to KV Cache Pruning" (SlimKV), Section 3:
//   Eq. 3  S1[j] = sum over the G query heads of the KV head's group (Section 3.1) and
//                  the w window queries of softmax_j(q . k_j / sqrt(d))
//   Eq. 4  S2[j] = max_c |V[j, c]|
//   Eq. 5  S[j]  = S1[j] * S2[j]
// Window query i sits at position L - w + i and sees keys j <= L - w + i.
//
// The softmax denominators must be known before any key's S1 can be summed, so K is
// swept twice; both sweeps run inside one kernel. In both, tcgen05 computes the tile's
// logits transposed, D[key, row] = K_tile[key] . Q_group[row] (M = 128 keys, N = G w
// query rows), so every epilogue thread owns one key and each TMEM column is a query row.
//   phase 0 (log-sum-exp): each CTA owns a contiguous run of 128-key tiles of the
//     flattened (sequence, KV head, tile) space. Per query row, each warp keeps a running
//     offset and sum of 2^(t - offset) over its 32 keys, t = logit * log2(e) / sqrt(d);
//     a butterfly reduce-scatter turns a 32 x 32 chunk of exponentials into per-row sums.
//     At the end of each KV head in its run, a CTA combines its warps' (offset, sum)
//     pairs, publishes one slot per row and bumps the head's completion counter.
//   phase 1 (scores): the same CTA sweeps the same tiles again (K now mostly from L2).
//     Before its first tile of a head it waits (bounded) until every CTA touching that
//     head has published, then merges the slots into lse2 = M + log2(sum_s l_s 2^(m_s - M))
//     per row. Per tile each thread sums 2^(t - lse2) over its key's row columns, reads
//     the key's V row once from shared memory for S2, and writes S (and S1, S2 if asked).
// Loads go through a ring of tile slots in shared memory: phase 0 streams K through all
// of them; phase 1 gives V (from HBM) the larger share and K (mostly L2) the rest.
// Warp roles: warp 0 issues TMA loads (the ring and the group's query rows), warp 1
// allocates TMEM and issues the MMAs from one thread, and two epilogue warpgroups
// (warps 2-5 and 6-9, one TMEM lane quarter per warp) each own TMEM accumulator
// stages. When a tile's accumulator fits one stage (G w <= 256) the groups take
// alternate tiles; otherwise every tile is split across both stages (query-row halves in
// phase 0, column halves in phase 1) and the second group hands its partial S1 to the
// first through shared memory.
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
constexpr int kEpiGroups = 2;                     // epilogue warpgroups
constexpr int kEpiThreads = 128 * kEpiGroups;
constexpr int kThreads = 64 + kEpiThreads;        // + TMA warp + MMA warp
constexpr int kMaxSlots = 8;                     // tile slots of the load ring
constexpr size_t kRingBytes = 128 * 1024;        // at most this much of it in flight (see build_launch)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kMaxStageCols = 256;           // widest accumulator stage
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s on any single wait
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMinSmem = 116 * 1024;              // forces one CTA per SM (TMEM is taken whole)
constexpr int kQBoxRows = 64;
constexpr size_t kBarBytes = 512;                 // shared memory reserved for SmemBars

#ifdef KVP_TRACE
// Debug builds only: %globaltimer stamps per CTA at phase boundaries.
__device__ unsigned long long g_kvp_trace[kPlanGrid][8];
#define KVP_STAMP(i) (g_kvp_trace[blockIdx.x][(i)] = ptx::globaltimer_ns())
// per-tile events of the first 4 CTAs: [cta][tile][event]
__device__ unsigned long long g_kvp_ttrace[4][64][8];
// MMA-thread steps of the first 4 CTAs (clock64): [cta][tile][step]
__device__ long long g_kvp_mtrace[4][64][12];
#define KVP_MSTAMP(t, e) ((blockIdx.x < 4 && (t) < 64) ? (void)(g_kvp_mtrace[blockIdx.x][(t)][(e)] = clock64()) : (void)0)
__device__ __forceinline__ int kvp_trace_slot() {
    return blockIdx.x == 0 ? 0 : blockIdx.x == 18 ? 1 : blockIdx.x == 73 ? 2 : blockIdx.x == 147 ? 3 : -1;
}
#define KVP_TSTAMP(t, e) \
    ((kvp_trace_slot() >= 0 && (t) < 64) ? (void)(g_kvp_ttrace[kvp_trace_slot()][(t)][(e)] = ptx::globaltimer_ns()) : (void)0)
#else
#define KVP_STAMP(i) ((void)0)
#define KVP_TSTAMP(t, e) ((void)0)
#define KVP_MSTAMP(t, e) ((void)0)
#endif

// error codes recorded in the workspace (first one wins)
enum : int { kErrWaitTma = 1, kErrWaitMma = 2, kErrWaitEpi = 3, kErrWaitPeers = 4 };

struct Params {
    int L, w, G, rows, hq, hkv, D;
    int qrows;           // query rows staged in shared memory (rows rounded up to 64)
    int n1, n2;          // phase 1 MMA N of the two column chunks (n2 = 0: one chunk)
    int split;           // 0: groups alternate tiles; 1: every tile split over both stages
    int stage_cols;      // TMEM columns per accumulator stage (128 or 256)
    int spg;             // accumulator stages per epilogue group (2 when a stage is 128 wide)
    int tiles_per_head, total_tiles, grid, cph, maxslots;
    int ns, nk1, nv1;    // ring slots; phase 1 gives K slots [0, nk1), V slots [nk1, ns)
    float scale2;        // log2(e) / sqrt(d)
    uint32_t q_bytes, k_bytes, v_bytes;
    uint32_t off_q, off_slots, off_lse, off_cw, off_wpos, off_bar;
    int cw_stride;       // floats per epilogue warp of phase 0 row offsets
    float* score;
    float* s1;
    float* s2;
    float2* part;        // [b*hq*w][maxslots]: (max, sum) in log2 units
    uint32_t* done;      // [b*hkv]
    int* err;
};

struct SmemBars {
    uint64_t kfull[kMaxSlots], kempty[kMaxSlots];   // per slot, for its K loads
    uint64_t vfull[kMaxSlots], vempty[kMaxSlots];   // per phase 1 V slot (index s - nk1)
    uint64_t accfull[4], accempty[4];
    uint64_t combfull[2], combempty[2];
    uint64_t qfull, qempty, fin;
    uint64_t epi;        // rendezvous of all epilogue threads
    uint32_t tmem_base;
    int abort_flag;
};

// Wait for phase `parity` of `bar`; false if the CTA is unwinding or the wait timed out
// (then the first error code is recorded and the CTA told to unwind).
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, SmemBars* sb,
                                           int* err, int code) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*(volatile int*)&sb->abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicCAS(err, 0, code);
            *(volatile int*)&sb->abort_flag = 1;
            return false;
        }
    }
}

// Wait for phase `parity` of `bar` for at most the wait limit, whatever the CTA's state:
// used before exit, so that no copy is still writing this CTA's shared memory.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity))
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) return;
}

// Rendezvous of all epilogue threads on an mbarrier, so that a thread that gives up a
// wait can never leave the others blocked in a hardware barrier. One arrival per warp,
// after the warp's shared-memory writes are ordered before it.
__device__ __forceinline__ bool epi_sync(SmemBars* sb, uint32_t& phase, int* err) {
    __threadfence_block();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(&sb->epi);
    const bool ok = wait_phase(&sb->epi, phase, sb, err, kErrWaitEpi);
    phase ^= 1u;
    return ok;
}

__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
    __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
    __nv_bfloat162 m = __hmax2(x, y);
    return *reinterpret_cast<uint32_t*>(&m);
}

// Accumulator stage that epilogue group g uses for the CTA's tile number i, and the
// parity of that use. Alternate-tile mode: group i & 1 takes tile i, cycling through its
// spg stages (stages g, g + 2); split mode: group g takes stage g of every tile.
__device__ __forceinline__ int acc_stage(int split, int spg, int i, int g, uint32_t& parity) {
    if (split) {
        parity = (uint32_t)i & 1u;
        return g;
    }
    const int u = i >> 1;
    parity = (uint32_t)(u / spg) & 1u;
    return g + 2 * (u % spg);
}

// The load ring. Phase 0 streams only K, through all ns slots in turn; phase 1 streams K
// through slots [0, nk1) and V through slots [nk1, ns). Each slot's K loads are counted
// across both phases, so the parity of a slot's barriers follows from the tile number.
__device__ __forceinline__ int ring_uses(int s, int period, int n) {   // uses of slot s
    return n > s ? (n - s + period - 1) / period : 0;                   // among n tiles
}
// K slot of the run's tile i in `phase`, and the number of that slot's earlier K loads.
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

// Butterfly reduce-scatter across the 32 lanes of a warp: v[i] holds this lane's value of
// column i; on return lane L's v[0] holds the maximum (kMax) or sum over all 32 lanes of
// column L. Five rounds, 31 shuffles.
template <bool kMax>
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
        const bool upper = (lane & k) != 0;
#pragma unroll
        for (int i = 0; i < k; ++i) {
            const float send = upper ? v[i] : v[i + k];
            const float keep = upper ? v[i + k] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, k);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
    return v[0];
}

// The one rare path of the epilogue (phase 0: logits far above their row's offset) is an
// out-of-line function that takes only scalars and loads its chunk from TMEM itself, so
// that the steady-state loops stay small (the instruction cache holds them) and carry
// none of its registers. Masks (window keys, a ragged last chunk) stay in the steady-state
// loops behind a warp-uniform flag: a separate masked path made the tile holding a head's
// window keys the last of the whole launch to finish.

// 32 TMEM columns of this warp's lanes at taddr: v[e] is the thread's key against local
// column cbase + e, masked to -inf past the group's ncols columns and, inside the window
// (key offset jw > 0), for query rows before the key.
__device__ __forceinline__ void load_masked(uint32_t taddr, float (&v)[32], int cbase, int ncols,
                                            int col0, int jw, const uint16_t* wpos) {
    __syncwarp();
    ptx::tmem_ld_32x32b_x32(taddr, v);
    ptx::tmem_ld_wait(v);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int n = cbase + e;
        if (n >= ncols || (jw > 0 && jw > (int)wpos[col0 + n])) v[e] = -INFINITY;
    }
}

// Phase 0, one chunk on the rare path. cw[0..31]: the warp's offsets (log2 units) of the
// chunk's rows; `first` sets them to each row's maximum over the warp's keys. Returns
// (lane L's sum of 2^(t - cw) over the warp's keys for row L of the chunk, lsum rescaled
// if the offsets had to be raised to keep the exponentials finite).
__device__ __noinline__ float2 lse_chunk_slow(uint32_t taddr, int cbase, int ncols, int col0,
                                              int jw, bool first, float* cw,
                                              const uint16_t* wpos, float scale2, float lsum) {
    const int lane = threadIdx.x & 31;
    float v[32];
    load_masked(taddr, v, cbase, ncols, col0, jw, wpos);
    if (first) {
        const float cmax = warp_reduce_scatter32<true>(v);
        __syncwarp();
        cw[lane] = cmax == -INFINITY ? -1e30f : cmax * scale2;
        __syncwarp();
        load_masked(taddr, v, cbase, ncols, col0, jw, wpos);
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = ptx::ex2(fmaf(v[i], scale2, -cw[i]));
    float sum = warp_reduce_scatter32<false>(v);
    if (__any_sync(0xffffffffu, !(sum < INFINITY))) {
        load_masked(taddr, v, cbase, ncols, col0, jw, wpos);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = fmaf(v[i], scale2, -cw[i]);
        float d = warp_reduce_scatter32<true>(v);
        d = d > 0.f ? d : 0.f;                    // also maps NaN (all masked) to 0
        lsum *= ptx::ex2(-d);
        __syncwarp();
        cw[lane] += d;
        __syncwarp();
        load_masked(taddr, v, cbase, ncols, col0, jw, wpos);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = ptx::ex2(fmaf(v[i], scale2, -cw[i]));
        sum = warp_reduce_scatter32<false>(v);
    }
    return make_float2(sum, lsum);
}

// Phase 0 hot path, two chunks at once (row offsets cwx, cwy): each element becomes
// 2^(t - cw) in place, the two chunks interleaved for independent work in flight.
__device__ __forceinline__ void lse_pair_fast(float (&x)[32], float (&y)[32], const float* cwx,
                                              const float* cwy, float scale2) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        const float4 c4 = *(const float4*)(cwx + i);
        const float4 d4 = *(const float4*)(cwy + i);
        x[i + 0] = ptx::ex2(fmaf(x[i + 0], scale2, -c4.x));
        x[i + 1] = ptx::ex2(fmaf(x[i + 1], scale2, -c4.y));
        x[i + 2] = ptx::ex2(fmaf(x[i + 2], scale2, -c4.z));
        x[i + 3] = ptx::ex2(fmaf(x[i + 3], scale2, -c4.w));
        y[i + 0] = ptx::ex2(fmaf(y[i + 0], scale2, -d4.x));
        y[i + 1] = ptx::ex2(fmaf(y[i + 1], scale2, -d4.y));
        y[i + 2] = ptx::ex2(fmaf(y[i + 2], scale2, -d4.z));
        y[i + 3] = ptx::ex2(fmaf(y[i + 3], scale2, -d4.w));
    }
}

// Phase 1 hot path, one full chunk: add 2^(t - lse2[n0 + e]) over its 32 query rows.
__device__ __forceinline__ void s1_chunk_fast(const float (&v)[32], const float* lse2, float scale2,
                                              float& a0, float& a1, float& a2, float& a3) {
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
        const float4 l4 = *(const float4*)(lse2 + e);
        a0 += ptx::ex2(fmaf(v[e + 0], scale2, -l4.x));
        a1 += ptx::ex2(fmaf(v[e + 1], scale2, -l4.y));
        a2 += ptx::ex2(fmaf(v[e + 2], scale2, -l4.z));
        a3 += ptx::ex2(fmaf(v[e + 3], scale2, -l4.w));
    }
}

// Phase 1, one chunk with masks: columns from `nrem` on (past the group's last) and, for a
// window key (jw > 0), query rows before the key contribute nothing.
__device__ __forceinline__ void s1_chunk_masked(const float (&v)[32], const float* lse2, const uint16_t* wp,
                                                int jw, int nrem, float scale2, float& a0, float& a1,
                                                float& a2, float& a3) {
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

}  // namespace
}  // namespace kvp

namespace kvp {
namespace {

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
score_fused_tc(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* Qs = smem + p.off_q;
    uint8_t* Slots = smem + p.off_slots;               // ring slots of tile_bytes each
    float* lse2 = (float*)(smem + p.off_lse);          // [rows, padded to 4]
    float* comb = lse2 + ((p.rows + 3) & ~3);           // [2][128] partial S1 handoff (split mode)
    // phase 0: [8 warps][cw_stride] row offsets; at the end of a head the same bytes stage
    // the warps' (offset, sum) pairs as float2 [8][cw_stride]
    float* cw_all = (float*)(smem + p.off_cw);
    // window position i of query row n (row n = g * w + i), so no division in the loops
    uint16_t* wpos = (uint16_t*)(smem + p.off_wpos);
    SmemBars* sb = (SmemBars*)(smem + p.off_bar);

    constexpr int kHalves = D / 64;                 // 128-byte swizzle rows per operand row
    constexpr uint32_t kHalfTile = kTile * 128;     // bytes of one 64-column half of a tile
    constexpr uint32_t kSlotBytes = kTile * D * 2;
    const uint32_t qhalf = (uint32_t)p.qrows * 128;  // bytes of one 64-column half of Q

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long T = p.total_tiles;
    const long long t0 = run_begin(blockIdx.x, T, p.grid, p.tiles_per_head, p.cph);
    const long long t1 = run_begin(blockIdx.x + 1, T, p.grid, p.tiles_per_head, p.cph);

    for (int n = threadIdx.x; n < p.rows; n += kThreads) wpos[n] = (uint16_t)(n % p.w);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxSlots; ++s) {
            ptx::mbar_init(&sb->kfull[s], 1);
            ptx::mbar_init(&sb->kempty[s], 1);
            ptx::mbar_init(&sb->vfull[s], 1);
            ptx::mbar_init(&sb->vempty[s], 4);
        }
        for (int s = 0; s < 4; ++s) {
            ptx::mbar_init(&sb->accfull[s], 1);
            ptx::mbar_init(&sb->accempty[s], 4);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&sb->combfull[s], 4);
            ptx::mbar_init(&sb->combempty[s], 4);
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
#ifdef KVP_TRACE
    if (threadIdx.x == 0 && blockIdx.x < 4) {
        g_kvp_ttrace[blockIdx.x][63][0] = clock64();
        g_kvp_ttrace[blockIdx.x][63][1] = ptx::globaltimer_ns();
    }
#endif

    auto group_row0 = [&](int bh) {
        const int b = bh / p.hkv, h = bh % p.hkv;
        return (b * p.hq + h * p.G) * p.w;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // K is read again by phase 1; plain L2 eviction measured a little faster than
            // marking it evict-last (K alone fits in L2 at 32K, K and V do not)
            const uint64_t pol_keep = ptx::policy_evict_normal();
            const uint64_t pol_stream = ptx::policy_evict_first();
            const int n = (int)(t1 - t0);
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
                        if (qgen > 0 && !(ok = wait_phase(&sb->qempty, (qgen - 1) & 1, sb, p.err, kErrWaitTma))) break;
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
                        if (!(ok = wait_phase(&sb->kempty[s], (use & 1) ^ 1, sb, p.err, kErrWaitTma))) break;
                        KVP_TSTAMP(phase * n + i, 0);
                        ptx::mbar_arrive_expect_tx(&sb->kfull[s], p.k_bytes);
                        for (int c = 0; c < kHalves; ++c)
                            ptx::tma_load_3d(Slots + s * kSlotBytes + c * kHalfTile, &kmap, &sb->kfull[s],
                                             c * 64, key0, head, phase == 0 ? pol_keep : pol_stream);
                        ++kiss[s];
                        if (phase == 1) {
                            const int jv = i % p.nv1, sv = p.nk1 + jv, vuse = i / p.nv1;
                            // a V slot's first load waits for its last K load of phase 0 to be consumed
                            const int u0 = vuse == 0 ? ring_uses(sv, p.ns, n) : 0;
                            if (u0 > 0 && !(ok = wait_phase(&sb->kempty[sv], (u0 - 1) & 1, sb, p.err, kErrWaitTma))) break;
                            if (!(ok = wait_phase(&sb->vempty[jv], (vuse & 1) ^ 1, sb, p.err, kErrWaitTma))) break;
                            KVP_TSTAMP(phase * n + i, 6);
                            ptx::mbar_arrive_expect_tx(&sb->vfull[jv], p.v_bytes);
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
            for (int s2 = 0; s2 < p.ns; ++s2)
                if (kiss[s2] > 0) drain_wait(&sb->kfull[s2], (kiss[s2] - 1) & 1);
            for (int jv = 0; jv < p.nv1; ++jv)
                if (viss[jv] > 0) drain_wait(&sb->vfull[jv], (viss[jv] - 1) & 1);
            if (qgen > 0) drain_wait(&sb->qfull, (qgen - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc1a = ptx::idesc_bf16_f32(128, p.n1);
            const uint32_t idesc1b = ptx::idesc_bf16_f32(128, p.n2 > 0 ? p.n2 : 16);
            const uint32_t q_addr = ptx::smem_u32(Qs), k_addr = ptx::smem_u32(Slots);
            const int n = (int)(t1 - t0);
            int ait = 0, qgen = 0, cur = -1;
            bool ok = true;
            for (int phase = 0; phase < 2 && ok; ++phase) {
                RunIter it(t0, t1, p.tiles_per_head);
                int head;
                long long a, b;
                int i = 0;                                  // tile number within the run
                while (ok && it.next(head, a, b)) {
                    if (head != cur) {
                        if (!(ok = wait_phase(&sb->qfull, qgen & 1, sb, p.err, kErrWaitMma))) break;
                        ++qgen;
                        cur = head;
                        ptx::tc_fence_after();
                    }
                    for (long long t = a; t < b; ++t, ++i) {
                        const int kit = phase * n + i;              // trace index
                        (void)kit;
                        int use;
                        const int s = k_slot(phase, i, n, p, use);
                        if (!(ok = wait_phase(&sb->kfull[s], use & 1, sb, p.err, kErrWaitMma))) break;
                        KVP_TSTAMP(kit, 1);
                        KVP_MSTAMP(kit, 0);
                        const uint32_t kbase = k_addr + s * kSlotBytes;
                        // stages written for this tile: one (alternating) or both (split)
                        const int g_lo = p.split ? 0 : (ait & 1);
                        const int g_hi = p.split ? 1 : (ait & 1);
                        for (int g = g_lo; g <= g_hi && ok; ++g) {
                            uint32_t use_parity;
                            const int st = acc_stage(p.split, p.spg, ait, g, use_parity);
                            if (!(ok = wait_phase(&sb->accempty[st], use_parity ^ 1, sb, p.err, kErrWaitMma))) break;
                            KVP_TSTAMP(kit, 2);
                            KVP_MSTAMP(kit, 1);
                            ptx::tc_fence_after();
                            KVP_MSTAMP(kit, 2);
                            const uint32_t d0 = tmem + (uint32_t)(st * p.stage_cols);
                            // descriptors of the first k-step; later k-steps add byte
                            // offsets (in 16-byte units) to the start-address field
                            const uint64_t kdesc0 = ptx::sw128_kmajor_desc(kbase);
                            const uint64_t qdesc0 = ptx::sw128_kmajor_desc(q_addr);
                            const bool first_chunk = !p.split || g == 0;
                            const bool second_chunk = p.n2 > 0 && (!p.split || g == 1);
                            const uint32_t n2_col = p.split ? 0u : (uint32_t)p.n1;
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t koff = (uint32_t)((ks >> 2) * kHalfTile + (ks & 3) * 32) >> 4;
                                const uint32_t qoff = ((ks >> 2) * qhalf + (ks & 3) * 32) >> 4;
                                const uint64_t kd = kdesc0 + koff;
                                if (first_chunk)
                                    ptx::mma_bf16_ss(d0, kd, qdesc0 + qoff, idesc1a, ks > 0);
                                if (second_chunk)
                                    ptx::mma_bf16_ss(d0 + n2_col, kd, qdesc0 + qoff + (uint32_t)(p.n1 * 128 >> 4),
                                                     idesc1b, ks > 0);
                                KVP_MSTAMP(kit, 3 + (ks & 7));
                            }
                            ptx::mma_commit(&sb->accfull[st]);
                        }
                        if (!ok) break;
                        ptx::mma_commit(&sb->kempty[s]);
                        KVP_TSTAMP(kit, 3);
                        KVP_MSTAMP(kit, 11);
                        ++ait;
                    }
                    if (!ok) break;
                    // release the query tile when the next segment loads another head's
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
            // all MMAs issued by this thread have completed before TMEM is released
            ptx::mma_commit(&sb->fin);
            wait_phase(&sb->fin, 0, sb, p.err, kErrWaitMma);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;                  // 0 .. kEpiThreads-1
        const int wg = et >> 7;                           // epilogue group = TMEM stage
        const int quarter = warp & 3;                     // TMEM lane quarter of this warp
        const int lrow = quarter * 32 + lane;             // lane: query row (phase 0) / key (phase 1)
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16);   // this warp's lanes
        const int window0 = p.L - p.w;                    // first window position
        // columns (query rows) this group's TMEM stage holds: all rows when the groups
        // alternate tiles, one half each when every tile is split across both stages
        const int col0 = (p.split && wg == 1) ? p.n1 : 0;
        const int ncols = p.split ? (wg == 0 ? p.n1 : p.rows - p.n1) : p.rows;
        const int nch = (ncols + 31) >> 5;
        const int warp8 = et >> 5;                        // epilogue warp 0..7
        float* cwp = cw_all + warp8 * p.cw_stride;        // this warp's row offsets
        int ait = 0;
        uint32_t epi_phase = 0;
        bool ok = true;
        // ---- phase 0: per query row, each warp's running offset and sum of 2^(t - offset)
        //      over its keys (thread = key, TMEM columns = query rows)
        {
            RunIter it(t0, t1, p.tiles_per_head);
            int head;
            long long a, b;
            while (ok && it.next(head, a, b)) {
                float lw[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                bool first_tile = true;
                for (long long t = a; t < b && ok; ++t, ++ait) {
                    if (!p.split && (ait & 1) != wg) continue;       // the other group's tile
                    uint32_t parity;
                    const int st = acc_stage(p.split, p.spg, ait, wg, parity);
                    const uint32_t tstage = tlane + (uint32_t)(st * p.stage_cols);
                    if (!(ok = wait_phase(&sb->accfull[st], parity, sb, p.err, kErrWaitEpi))) break;
                    if (lrow == 0) KVP_TSTAMP(ait, 4);
                    ptx::tc_fence_after();
                    const int key0 = (int)(t - (long long)head * p.tiles_per_head) * kTile;
                    const int j = key0 + lrow;                       // this thread's key
                    const int jw = j - window0;                      // > 0 only inside the window
                    // masks, needed only by warps holding window keys and by a ragged last chunk
                    // masks: window keys (query rows before the key) and columns past the
                    // group's last; only warps holding window keys or a ragged last chunk
                    // need them, which the warp decides as a whole
                    const bool masked = __any_sync(0xffffffffu, jw > 0) || (ncols & 31);
                    auto mask_chunk = [&](float (&v)[32], int c) {
                        if (jw > 0) {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (jw > (int)wpos[col0 + c * 32 + e]) v[e] = -INFINITY;
                        }
                        if ((c + 1) * 32 > ncols) {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (c * 32 + e >= ncols) v[e] = -INFINITY;
                        }
                    };
                    // A head's first tile takes each row's offset from the warp's first key
                    // (any offset within ~100 of a row's maximum keeps every exponential
                    // finite; farther ones are caught by the overflow path).
                    auto set_offsets = [&](const float (&v)[32], int c) {
                        if (lane == 0) {
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                cwp[c * 32 + e] = v[e] == -INFINITY ? -1e30f : v[e] * p.scale2;
                        }
                    };
                    // Two chunks at a time so that their exponentials and shuffles interleave;
                    // an odd last chunk is paired with an empty one.
                    float x[32], y[32];
                    __syncwarp();
                    ptx::tmem_ld_32x32b_x32(tstage, x);
                    ptx::tmem_ld_wait(x);
#pragma unroll 1
                    for (int c = 0; c < nch; c += 2) {
                        const bool pair = c + 1 < nch;
                        if (pair) {
                            __syncwarp();
                            ptx::tmem_ld_32x32b_x32(tstage + (c + 1) * 32, y);
                            ptx::tmem_ld_wait(y);
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) y[e] = -INFINITY;
                        }
                        if (masked) {
                            mask_chunk(x, c);
                            if (pair) mask_chunk(y, c + 1);
                        }
                        if (first_tile) {
                            __syncwarp();
                            set_offsets(x, c);
                            if (pair) set_offsets(y, c + 1);
                            __syncwarp();
                        }
                        lse_pair_fast(x, y, cwp + c * 32, pair ? cwp + c * 32 + 32 : cwp + c * 32, p.scale2);
                        float s0 = warp_reduce_scatter32<false>(x);
                        float s1 = warp_reduce_scatter32<false>(y);
                        float l0 = 0.f, l1 = 0.f;
#pragma unroll
                        for (int cc = 0; cc < 8; cc += 2)
                            if (cc == c) {
                                l0 = lw[cc];
                                l1 = lw[cc + 1];
                            }
                        if (__any_sync(0xffffffffu, !(s0 < INFINITY) || !(s1 < INFINITY))) {
                            // rare: a logit far above its row's offset; raise, redo
                            float2 r = lse_chunk_slow(tstage + c * 32, c * 32, ncols, col0, jw, false,
                                                      cwp + c * 32, wpos, p.scale2, l0);
                            s0 = r.x;
                            l0 = r.y;
                            if (pair) {
                                r = lse_chunk_slow(tstage + (c + 1) * 32, (c + 1) * 32, ncols, col0, jw,
                                                   false, cwp + (c + 1) * 32, wpos, p.scale2, l1);
                                s1 = r.x;
                                l1 = r.y;
                            }
                        }
#pragma unroll
                        for (int cc = 0; cc < 8; cc += 2)
                            if (cc == c) {
                                lw[cc] = l0 + s0;
                                if (pair) lw[cc + 1] = l1 + s1;
                            }
                        if (c + 2 < nch) {
                            __syncwarp();
                            ptx::tmem_ld_32x32b_x32(tstage + (c + 2) * 32, x);
                            ptx::tmem_ld_wait(x);
                        }
                    }
                    first_tile = false;
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sb->accempty[st]);
                    if (lrow == 0) KVP_TSTAMP(ait, 5);
                }
                if (!ok) break;
                // Combine the warps' (offset, sum) of every row inside the CTA, then publish
                // one slot per row. The staging buffer aliases the offsets, so each lane
                // first takes its own offsets into registers.
                float cwr[8];
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const int n = cc * 32 + lane;
                    cwr[cc] = (n < ncols) ? cwp[n] : 0.f;
                }
                if (!(ok = epi_sync(sb, epi_phase, p.err))) break;
                float2* stage = reinterpret_cast<float2*>(cw_all) + warp8 * p.cw_stride;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    const int n = cc * 32 + lane;
                    if (n < ncols)
                        stage[n] = first_tile ? make_float2(-INFINITY, 0.f) : make_float2(cwr[cc], lw[cc]);
                }
                if (!(ok = epi_sync(sb, epi_phase, p.err))) break;
                const long long first = (long long)head * p.tiles_per_head;
                const int slot = (int)blockIdx.x - owner_of(first, T, p.grid, p.tiles_per_head, p.cph);
                const int r0 = group_row0(head);
                for (int r = et; r < p.rows; r += kEpiThreads) {
                    // warps holding row r: all eight, or the four of the group owning it
                    const int g = (p.split && r >= p.n1) ? 1 : 0;
                    const int n = r - (g ? p.n1 : 0);
                    const int w_lo = p.split ? 4 * g : 0, w_hi = p.split ? 4 * g + 4 : 8;
                    float M = -INFINITY, S = 0.f;
                    for (int w = w_lo; w < w_hi; ++w) {
                        const float2 ml = reinterpret_cast<const float2*>(cw_all)[w * p.cw_stride + n];
                        if (ml.y == 0.f) continue;
                        if (ml.x > M) {
                            S = S * ptx::ex2(M - ml.x) + ml.y;
                            M = ml.x;
                        } else {
                            S += ml.y * ptx::ex2(ml.x - M);
                        }
                    }
                    if (KVP_CHECK(slot >= 0 && slot < p.maxslots, 202, slot, head))
                        p.part[(size_t)(r0 + r) * p.maxslots + slot] = make_float2(M, S);
                }
                if (!(ok = epi_sync(sb, epi_phase, p.err))) break;
                if (et == 0) {
                    __threadfence();
                    atomicAdd(p.done + head, 1u);
                }
            }
        }
        if (et == 0) KVP_STAMP(5);
        // ---- phase 1: scores
        {
            bool first_seg = true;
            RunIter it(t0, t1, p.tiles_per_head);
            int head;
            long long a, b;
            int pt = 0;                                   // phase 1 tile counter (V ring, handoff)
            while (ok && it.next(head, a, b)) {
                const long long first = (long long)head * p.tiles_per_head;
                const int touch = owner_of(first + p.tiles_per_head - 1, T, p.grid, p.tiles_per_head, p.cph) -
                                  owner_of(first, T, p.grid, p.tiles_per_head, p.cph) + 1;
                // the previous head's lse2 is no longer in use
                if (!(ok = epi_sync(sb, epi_phase, p.err))) break;
                if (et == 0) {
                    const uint64_t ts = ptx::globaltimer_ns();
                    while (ptx::ld_acquire_u32(p.done + head) < (uint32_t)touch) {
                        if (*(volatile int*)&sb->abort_flag) break;
                        if (ptx::globaltimer_ns() - ts > kWaitLimitNs) {
                            atomicCAS(p.err, 0, kErrWaitPeers);
                            *(volatile int*)&sb->abort_flag = 1;
                            break;
                        }
                        __nanosleep(128);
                    }
                }
                if (!(ok = epi_sync(sb, epi_phase, p.err))) break;
                if (et == 0 && first_seg) KVP_STAMP(6);
                first_seg = false;
                if (*(volatile int*)&sb->abort_flag) {
                    ok = false;
                    break;
                }
                const int r0 = group_row0(head);
                const int nslots = touch * kSlotsPerCta;
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
                if (!(ok = epi_sync(sb, epi_phase, p.err))) break;
                for (long long t = a; t < b && ok; ++t, ++ait, ++pt) {
                    const bool mine = p.split || (ait & 1) == wg;
                    if (!mine) continue;
                    const bool reads_v = !p.split || wg == 0;
                    const int key0 = (int)(t - first) * kTile;
                    const int j = key0 + lrow;
                    float s2v = 0.f;
                    if (reads_v) {
                        // S2: max |V[j, :]| from the staged tile, 16-byte pieces in a
                        // rotated order per lane (conflict-free shared-memory reads)
                        const int jv = pt % p.nv1;
                        if (!(ok = wait_phase(&sb->vfull[jv], (pt / p.nv1) & 1, sb, p.err, kErrWaitEpi))) break;
                        if (lrow == 0) KVP_TSTAMP(ait, 7);
                        const uint4* vrow = (const uint4*)(Slots + (p.nk1 + jv) * kSlotBytes + lrow * (D * 2));
                        constexpr int kPieces = D * 2 / 16;
                        uint32_t mx = 0;
#pragma unroll
                        for (int c = 0; c < kPieces; ++c) {
                            const uint4 x = vrow[(c + lane) & (kPieces - 1)];
                            mx = bf16x2_absmax(mx, x.x & 0x7FFF7FFFu);
                            mx = bf16x2_absmax(mx, x.y & 0x7FFF7FFFu);
                            mx = bf16x2_absmax(mx, x.z & 0x7FFF7FFFu);
                            mx = bf16x2_absmax(mx, x.w & 0x7FFF7FFFu);
                        }
                        s2v = fmaxf(__uint_as_float(mx << 16), __uint_as_float(mx & 0xFFFF0000u));
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&sb->vempty[jv]);
                    }
                    // S1 over this group's columns
                    uint32_t parity;
                    const int st = acc_stage(p.split, p.spg, ait, wg, parity);
                    const uint32_t tstage = tlane + (uint32_t)(st * p.stage_cols);
                    if (!(ok = wait_phase(&sb->accfull[st], parity, sb, p.err, kErrWaitEpi))) break;
                    if (lrow == 0) KVP_TSTAMP(ait, 4);
                    ptx::tc_fence_after();
                    const int jw = j - window0;                     // > 0 only inside the window
                    const int col0 = (p.split && wg == 1) ? p.n1 : 0;        // first query row
                    const int ncols = p.split ? (wg == 0 ? p.n1 : p.rows - p.n1) : p.rows;
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                    // masks (window keys, a ragged last chunk) are decided per warp: TMEM loads
                    // are warp-collective, so every lane takes the same loop
                    const bool masked = __any_sync(0xffffffffu, jw > 0) || (ncols & 31);
                    auto s1_chunk = [&](const float (&v)[32], int c) {
                        if (masked)
                            s1_chunk_masked(v, lse2 + col0 + c * 32, wpos + col0 + c * 32, jw, ncols - c * 32,
                                            p.scale2, a0, a1, a2, a3);
                        else
                            s1_chunk_fast(v, lse2 + col0 + c * 32, p.scale2, a0, a1, a2, a3);
                    };
                    float x[32], y[32];
                    __syncwarp();
                    ptx::tmem_ld_32x32b_x32(tstage, x);
                    ptx::tmem_ld_wait(x);
                    for (int c = 0; c < nch; c += 2) {
                        const bool has1 = c + 1 < nch, has2 = c + 2 < nch;
                        if (has1) {
                            __syncwarp();
                            ptx::tmem_ld_32x32b_x32(tstage + (c + 1) * 32, y);
                        }
                        s1_chunk(x, c);
                        if (has1) {
                            ptx::tmem_ld_wait(y);
                            if (has2) {
                                __syncwarp();
                                ptx::tmem_ld_32x32b_x32(tstage + (c + 2) * 32, x);
                            }
                            s1_chunk(y, c + 1);
                            if (has2) ptx::tmem_ld_wait(x);
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sb->accempty[st]);
                    if (lrow == 0) KVP_TSTAMP(ait, 5);
                    float s1v = (a0 + a1) + (a2 + a3);
                    if (p.split) {
                        // hand the second group's partial to the first
                        const int cb = pt & 1;
                        const uint32_t cpar = (pt >> 1) & 1;
                        if (wg == 1) {
                            if (!(ok = wait_phase(&sb->combempty[cb], cpar ^ 1, sb, p.err, kErrWaitEpi))) break;
                            comb[cb * kTile + lrow] = s1v;
                            __syncwarp();
                            if (lane == 0) ptx::mbar_arrive(&sb->combfull[cb]);
                            continue;
                        }
                        if (!(ok = wait_phase(&sb->combfull[cb], cpar, sb, p.err, kErrWaitEpi))) break;
                        s1v += comb[cb * kTile + lrow];
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(&sb->combempty[cb]);
                    }
                    if (j < p.L && KVP_CHECK(head < p.total_tiles / p.tiles_per_head, 201, head, j)) {
                        const size_t o = (size_t)head * p.L + j;
                        p.score[o] = s1v * s2v;
                        if (p.s1) p.s1[o] = s1v;
                        if (p.s2) p.s2[o] = s2v;
                    }
                }
            }
        }
    }

    if (threadIdx.x == 64) KVP_STAMP(7);
#ifdef KVP_TRACE
    if (threadIdx.x == 64 && blockIdx.x < 4) {
        g_kvp_ttrace[blockIdx.x][63][2] = clock64();
        g_kvp_ttrace[blockIdx.x][63][3] = ptx::globaltimer_ns();
    }
#endif
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

bool build_launch(const kvp_shape& s, const Plan& plan, int sms, Launch* L) {
    Params& p = L->p;
    const int D = s.head_dim;
    p.L = s.seq_len;
    p.w = s.window;
    p.G = plan.G;
    p.rows = plan.rows;
    p.hq = s.hq;
    p.hkv = s.hkv;
    p.D = D;
    const int npad = (plan.rows + 15) / 16 * 16;
    if (npad <= 256) {
        p.n1 = npad;
        p.n2 = 0;
    } else {
        p.n1 = (npad / 2 + 15) / 16 * 16;
        p.n2 = npad - p.n1;
    }
    p.split = plan.rows > (int)kMaxStageCols ? 1 : 0;
    // two 128-column stages per group when a tile's accumulator fits 128 columns
    p.stage_cols = (!p.split && (plan.rows + 31) / 32 * 32 <= 128) ? 128 : 256;
    p.spg = p.stage_cols == 128 ? 2 : 1;
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
    const int qrows = (plan.rows + kQBoxRows - 1) / kQBoxRows * kQBoxRows;
    p.qrows = qrows;
    const uint32_t qbytes = (uint32_t)qrows * D * 2;
    const uint32_t tile_bytes = (uint32_t)kTile * D * 2;
    p.q_bytes = qbytes;
    p.k_bytes = tile_bytes;
    p.v_bytes = tile_bytes;
    // shared memory: Q | K ring | V ring | lse2 + handoff | phase 0 row offsets | barriers
    // (+1 KB to align the base)
    const int group_cols = p.split ? std::max(p.n1, plan.rows - p.n1) : plan.rows;
    p.cw_stride = (group_cols + 31) / 32 * 32;
    const size_t cw_bytes = (size_t)(kEpiThreads / 32) * p.cw_stride * sizeof(float2);
    // lse2[rows] (16-byte padded), then the split-mode handoff comb[2][128]
    const size_t lse_floats = (size_t)((plan.rows + 3) / 4 * 4);
    const size_t lse_bytes = (lse_floats + (p.split ? 2 * kTile : 0)) * sizeof(float);
    const size_t wpos_bytes = (size_t)((plan.rows + 7) / 8 * 8) * sizeof(uint16_t);
    const size_t fixed = std::max(lse_bytes, cw_bytes) + wpos_bytes + kBarBytes + 1024;
    // As many ring slots as fit. Phase 1 splits them between K (read again, mostly from
    // L2) and V (from HBM, so it gets the deeper share). Alternate-tile mode: both epilogue
    // groups read V slots, each its own tiles; with an even number of V slots a group only
    // ever waits on its own slots, one phase ahead at most (an odd count would make a group
    // wait two phases ahead on a shared slot, where the parity test cannot tell the phases
    // apart). Split mode: group 0 alone reads V.
    if (qbytes + fixed > (size_t)kSmemLimit) return false;
    // (a deeper ring measured slower on the 32K layer: 5 slots of 32 KiB gave a 1.5 us
    // longer launch than 4)
    p.ns = (int)std::min<size_t>(std::min<size_t>(kMaxSlots, kRingBytes / tile_bytes),
                                 ((size_t)kSmemLimit - qbytes - fixed) / tile_bytes);
    if (p.split) {
        if (p.ns < 2) return false;
        p.nv1 = p.ns / 2;
    } else {
        if (p.ns < 3) return false;
        p.nv1 = p.ns >= 6 ? 4 : 2;
    }
    p.nk1 = p.ns - p.nv1;
    const size_t total = qbytes + (size_t)p.ns * tile_bytes + fixed;
    p.off_q = 0;
    p.off_slots = qbytes;
    // phase 0's row offsets / staging and phase 1's lse2 + handoff are never live at the
    // same time (all epilogue threads pass a rendezvous between the phases): one region
    p.off_cw = p.off_slots + p.ns * tile_bytes;
    p.off_lse = p.off_cw;
    p.off_wpos = p.off_cw + (uint32_t)std::max(lse_bytes, cw_bytes);
    p.off_bar = p.off_wpos + (uint32_t)wpos_bytes;
    static_assert(sizeof(SmemBars) <= kBarBytes, "barrier block");
    L->grid = p.grid;
    L->smem = std::max(total, (size_t)kMinSmem);
    return true;
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
    if ((e = cudaMemsetAsync(ws + plan.off_done, 0, plan.off_part - plan.off_done, st)) != cudaSuccess)
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
#endif
#ifdef KVP_TRACE
int take_trace(unsigned long long* out) {
    if (cudaMemcpyFromSymbol(out, g_kvp_trace, sizeof(g_kvp_trace)) != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(out + 148 * 8, g_kvp_ttrace, sizeof(g_kvp_ttrace)) != cudaSuccess) return -1;
    return cudaMemcpyFromSymbol(out + 148 * 8 + 4 * 64 * 8, g_kvp_mtrace, sizeof(g_kvp_mtrace)) == cudaSuccess ? 0 : -1;
}
#endif

}  // namespace kvp
