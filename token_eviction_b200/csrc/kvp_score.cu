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
// swept twice; both sweeps run inside one kernel:
//   phase 0 (log-sum-exp): each CTA owns a contiguous run of 128-key tiles of the
//     flattened (sequence, KV head, tile) space. Per tile, tcgen05 computes the logits
//     D[row, key] = Q_group[row] . K_tile[key] (M = query rows, N = 128 keys) into TMEM;
//     the epilogue keeps, per query row, a running max m and sum l of 2^(t - m),
//     t = logit * log2(e) / sqrt(d). At the end of each KV head in its run, a CTA
//     publishes (m, l) per row into its slot and bumps the head's completion counter.
//   phase 1 (scores): the same CTA sweeps the same tiles again. Before its first tile of
//     a head it waits (bounded) until every CTA touching that head has published, then
//     merges the slots into lse2 = M + log2(sum_s l_s 2^(m_s - M)) per row. Per tile,
//     tcgen05 computes the transposed logits D[key, row] (M = 128 keys, N = G w rows), so
//     each epilogue thread owns one key and sums 2^(t - lse2) over its row in TMEM
//     columns with no cross-thread reduction; it reads the key's V row once from shared
//     memory for S2 and writes S (and S1, S2 if asked).
// Warp roles: warp 0 issues TMA loads (K ring, V ring, the group's query rows), warp 1
// allocates TMEM and issues MMAs from one thread, warps 2-5 run the epilogue (one TMEM
// lane quarter each). Every wait is bounded by a timer; a wait that gives up records an
// error code in the workspace and the whole CTA unwinds without touching TMEM or
// shared memory that may still be in use.
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

constexpr int kTile = 128;                    // keys per tile
constexpr int kThreads = 192;                 // 6 warps
constexpr int kEpiThreads = 128;              // warps 2..5
constexpr int kMaxStages = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s on any single wait
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMinSmem = 116 * 1024;          // forces one CTA per SM (TMEM is taken whole)

// error codes recorded in the workspace (first one wins)
enum : int { kErrWaitTma = 1, kErrWaitMma = 2, kErrWaitEpi = 3, kErrWaitPeers = 4 };

struct Params {
    int L, w, G, rows, hq, hkv, D;
    int mt;              // 128-row tiles covering the query group (phase 0 M tiles)
    int qrows;           // query rows staged in shared memory (rows rounded up to 64)
    int n1, n2;          // phase 1 MMA N split of the group rows (n2 = 0: one MMA)
    int tiles_per_head, total_tiles, grid, maxslots;
    int nk, nv;          // K and V ring depths
    int acc_stages, acc_stride;
    float scale2;        // log2(e) / sqrt(d)
    uint32_t q_bytes, k_bytes, v_bytes;
    uint32_t off_q, off_k, off_v, off_lse, off_bar;
    float* score;
    float* s1;
    float* s2;
    float2* part;        // [b*hq*w][maxslots]
    uint32_t* done;      // [b*hkv]
    int* err;
};

struct SmemBars {
    uint64_t kfull[kMaxStages], kempty[kMaxStages];
    uint64_t vfull[kMaxStages], vempty[kMaxStages];
    uint64_t accfull[2], accempty[2];
    uint64_t qfull, qempty, fin;
    uint64_t epi;        // epilogue-group rendezvous (128 arrivals per phase)
    uint32_t tmem_base;
    int abort_flag;
};

}  // namespace
}  // namespace kvp

namespace kvp {
namespace {

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

__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
    __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
    __nv_bfloat162 m = __hmax2(x, y);
    return *reinterpret_cast<uint32_t*>(&m);
}

// Rendezvous of the 128 epilogue threads on an mbarrier, so that a thread that gives up
// a wait can never leave the others blocked in a hardware barrier.
__device__ __forceinline__ bool epi_sync(SmemBars* sb, uint32_t& phase, int* err) {
    ptx::mbar_arrive(&sb->epi);
    const bool ok = wait_phase(&sb->epi, phase, sb, err, kErrWaitEpi);
    phase ^= 1u;
    return ok;
}

// Segments of a CTA's run: maximal stretches of tiles within one KV head.
struct RunIter {
    long long t, end;
    int tph;
    __device__ RunIter(long long b, long long e, int tiles_per_head) : t(b), end(e), tph(tiles_per_head) {}
    // head of the next segment and its tile range [a, b)
    __device__ bool next(int& head, long long& a, long long& b) {
        if (t >= end) return false;
        head = (int)(t / tph);
        a = t;
        b = min(end, (long long)(head + 1) * tph);
        t = b;
        return true;
    }
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
score_fused_tc(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* Qs = smem + p.off_q;
    uint8_t* Ks = smem + p.off_k;
    uint8_t* Vs = smem + p.off_v;
    float* lse2 = (float*)(smem + p.off_lse);
    SmemBars* sb = (SmemBars*)(smem + p.off_bar);

    constexpr int kHalves = D / 64;                 // 128-byte swizzle rows per operand row
    constexpr uint32_t kHalfTile = kTile * 128;     // bytes of one 64-column half of a tile
    const uint32_t kstage = kTile * D * 2, vstage = kTile * D * 2;
    const uint32_t qhalf = (uint32_t)p.qrows * 128;  // bytes of one 64-column half of Q

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long T = p.total_tiles;
    const long long t0 = run_begin(blockIdx.x, T, p.grid), t1 = run_begin(blockIdx.x + 1, T, p.grid);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxStages; ++s) {
            ptx::mbar_init(&sb->kfull[s], 1);
            ptx::mbar_init(&sb->kempty[s], 1);
            ptx::mbar_init(&sb->vfull[s], 1);
            ptx::mbar_init(&sb->vempty[s], kEpiThreads / 32);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(&sb->accfull[s], 1);
            ptx::mbar_init(&sb->accempty[s], kEpiThreads / 32);
        }
        ptx::mbar_init(&sb->qfull, 1);
        ptx::mbar_init(&sb->qempty, 1);
        ptx::mbar_init(&sb->fin, 1);
        ptx::mbar_init(&sb->epi, kEpiThreads);
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

    auto group_row0 = [&](int bh) {
        const int b = bh / p.hkv, h = bh % p.hkv;
        return (b * p.hq + h * p.G) * p.w;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_keep = ptx::policy_evict_last();
            const uint64_t pol_stream = ptx::policy_evict_first();
            int kit = 0, vit = 0, qgen = 0, cur = -1;
            bool ok = true;
            for (int phase = 0; phase < 2 && ok; ++phase) {
                RunIter it(t0, t1, p.tiles_per_head);
                int head;
                long long a, b;
                while (ok && it.next(head, a, b)) {
                    if (head != cur) {
                        if (qgen > 0 && !(ok = wait_phase(&sb->qempty, (qgen - 1) & 1, sb, p.err, kErrWaitTma))) break;
                        ptx::mbar_arrive_expect_tx(&sb->qfull, p.q_bytes);
                        const int r0 = group_row0(head);
                        for (int rb = 0; rb < p.qrows; rb += 64)
                            for (int c = 0; c < kHalves; ++c)
                                ptx::tma_load_2d(Qs + c * qhalf + rb * 128, &qmap, &sb->qfull,
                                                 c * 64, r0 + rb, pol_keep);
                        ++qgen;
                        cur = head;
                    }
                    for (long long t = a; t < b; ++t) {
                        const int key0 = (int)(t - (long long)head * p.tiles_per_head) * kTile;
                        const int s = kit % p.nk;
                        if (!(ok = wait_phase(&sb->kempty[s], ((kit / p.nk) & 1) ^ 1, sb, p.err, kErrWaitTma))) break;
                        ptx::mbar_arrive_expect_tx(&sb->kfull[s], p.k_bytes);
                        for (int c = 0; c < kHalves; ++c)
                            ptx::tma_load_3d(Ks + s * kstage + c * kHalfTile, &kmap, &sb->kfull[s],
                                             c * 64, key0, head, phase == 0 ? pol_keep : pol_stream);
                        ++kit;
                        if (phase == 1) {
                            const int sv = vit % p.nv;
                            if (!(ok = wait_phase(&sb->vempty[sv], ((vit / p.nv) & 1) ^ 1, sb, p.err, kErrWaitTma))) break;
                            ptx::mbar_arrive_expect_tx(&sb->vfull[sv], p.v_bytes);
                            ptx::tma_load_3d(Vs + sv * vstage, &vmap, &sb->vfull[sv], 0, key0, head,
                                             pol_stream);
                            ++vit;
                        }
                    }
                }
            }
            // Never leave with copies in flight: wait for the last load of every stage.
            for (int i = max(0, kit - p.nk); i < kit; ++i)
                wait_phase(&sb->kfull[i % p.nk], (i / p.nk) & 1, sb, p.err, kErrWaitTma);
            for (int i = max(0, vit - p.nv); i < vit; ++i)
                wait_phase(&sb->vfull[i % p.nv], (i / p.nv) & 1, sb, p.err, kErrWaitTma);
            if (qgen > 0) wait_phase(&sb->qfull, (qgen - 1) & 1, sb, p.err, kErrWaitTma);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc0 = ptx::idesc_bf16_f32(128, kTile);
            const uint32_t idesc1a = ptx::idesc_bf16_f32(128, p.n1);
            const uint32_t idesc1b = ptx::idesc_bf16_f32(128, p.n2 > 0 ? p.n2 : 16);
            const uint32_t q_addr = ptx::smem_u32(Qs), k_addr = ptx::smem_u32(Ks);
            int kit = 0, ait = 0, qgen = 0, cur = -1;
            bool ok = true;
            for (int phase = 0; phase < 2 && ok; ++phase) {
                RunIter it(t0, t1, p.tiles_per_head);
                int head;
                long long a, b;
                while (ok && it.next(head, a, b)) {
                    if (head != cur) {
                        if (!(ok = wait_phase(&sb->qfull, qgen & 1, sb, p.err, kErrWaitMma))) break;
                        ++qgen;
                        cur = head;
                        ptx::tc_fence_after();
                    }
                    for (long long t = a; t < b; ++t) {
                        const int s = kit % p.nk;
                        const int sa = ait % p.acc_stages;
                        if (!(ok = wait_phase(&sb->kfull[s], (kit / p.nk) & 1, sb, p.err, kErrWaitMma))) break;
                        if (!(ok = wait_phase(&sb->accempty[sa], ((ait / p.acc_stages) & 1) ^ 1, sb, p.err, kErrWaitMma))) break;
                        ptx::tc_fence_after();
                        const uint32_t d0 = tmem + (uint32_t)(sa * p.acc_stride);
                        const uint32_t kbase = k_addr + s * kstage;
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const int c = ks >> 2, kk = ks & 3;
                            const uint32_t koff = kbase + c * kHalfTile + kk * 32;
                            const uint32_t qoff = q_addr + c * qhalf + kk * 32;
                            if (phase == 0) {
                                for (int m = 0; m < p.mt; ++m)
                                    ptx::mma_bf16_ss(d0 + m * kTile,
                                                     ptx::sw128_kmajor_desc(qoff + m * kHalfTile),
                                                     ptx::sw128_kmajor_desc(koff), idesc0, ks > 0);
                            } else {
                                const uint64_t adesc = ptx::sw128_kmajor_desc(koff);
                                ptx::mma_bf16_ss(d0, adesc, ptx::sw128_kmajor_desc(qoff), idesc1a, ks > 0);
                                if (p.n2 > 0)
                                    ptx::mma_bf16_ss(d0 + p.n1, adesc,
                                                     ptx::sw128_kmajor_desc(qoff + p.n1 * 128), idesc1b,
                                                     ks > 0);
                            }
                        }
                        ptx::mma_commit(&sb->kempty[s]);
                        ptx::mma_commit(&sb->accfull[sa]);
                        ++kit;
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
            }
            // all MMAs issued by this thread have completed before TMEM is released
            ptx::mma_commit(&sb->fin);
            wait_phase(&sb->fin, 0, sb, p.err, kErrWaitMma);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;                  // 0..127
        const int quarter = warp & 3;                     // TMEM lane quarter of this warp
        const int lrow = quarter * 32 + lane;             // lane owned: row (phase 0) or key (phase 1)
        const uint32_t lane_bits = (uint32_t)(quarter * 32) << 16;
        const int window0 = p.L - p.w;                    // first window position
        int ait = 0, vit = 0;
        uint32_t epi_phase = 0;
        bool ok = true;
        // ---- phase 0: per-row running max and sum over this CTA's keys of each head
        {
            RunIter it(t0, t1, p.tiles_per_head);
            int head;
            long long a, b;
            while (ok && it.next(head, a, b)) {
                float mrun[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                float lrun[4] = {0.f, 0.f, 0.f, 0.f};
                for (long long t = a; t < b && ok; ++t) {
                    const int key0 = (int)(t - (long long)head * p.tiles_per_head) * kTile;
                    const int sa = ait % p.acc_stages;
                    if (!(ok = wait_phase(&sb->accfull[sa], (ait / p.acc_stages) & 1, sb, p.err, kErrWaitEpi))) break;
                    ptx::tc_fence_after();
                    const bool full = key0 + kTile - 1 <= window0;   // every row sees every key
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        if (m >= p.mt) break;                        // uniform across the CTA
                        const int r = m * kTile + lrow;
                        const int last = window0 + (r % p.w);        // last key row r sees
#pragma unroll 1
                        for (int ch = 0; ch < kTile / 32; ++ch) {
                            float v[32];
                            __syncwarp();
                            ptx::tmem_ld_32x32b_x32(tmem + lane_bits + sa * p.acc_stride + m * kTile + ch * 32, v);
                            ptx::tmem_ld_wait();
                            if (!full) {
#pragma unroll
                                for (int e = 0; e < 32; ++e)
                                    if (key0 + ch * 32 + e > last) v[e] = -INFINITY;
                            }
                            float cm = v[0];
#pragma unroll
                            for (int e = 1; e < 32; ++e) cm = fmaxf(cm, v[e]);
                            if (cm != -INFINITY) {
                                const float mn = fmaxf(mrun[m], cm * p.scale2);
                                float acc = lrun[m] * ptx::ex2(mrun[m] - mn);
#pragma unroll
                                for (int e = 0; e < 32; ++e) acc += ptx::ex2(fmaf(v[e], p.scale2, -mn));
                                lrun[m] = acc;
                                mrun[m] = mn;
                            }
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sb->accempty[sa]);
                    ++ait;
                }
                if (!ok) break;
                // publish this CTA's partials for `head`
                const long long first = (long long)head * p.tiles_per_head;
                const int slot = (int)blockIdx.x - owner_of(first, T, p.grid);
                const int r0 = group_row0(head);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int r = m * kTile + lrow;
                    if (m < p.mt && r < p.rows)
                        p.part[(size_t)(r0 + r) * p.maxslots + slot] = make_float2(mrun[m], lrun[m]);
                }
                if (!(ok = epi_sync(sb, epi_phase, p.err))) break;
                if (et == 0) {
                    __threadfence();
                    atomicAdd(p.done + head, 1u);
                }
            }
        }
        // ---- phase 1: scores
        {
            RunIter it(t0, t1, p.tiles_per_head);
            int head;
            long long a, b;
            while (ok && it.next(head, a, b)) {
                const long long first = (long long)head * p.tiles_per_head;
                const int touch = owner_of(first + p.tiles_per_head - 1, T, p.grid) - owner_of(first, T, p.grid) + 1;
                // previous head's lse2 no longer in use
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
                if (*(volatile int*)&sb->abort_flag) {
                    ok = false;
                    break;
                }
                const int r0 = group_row0(head);
                for (int r = et; r < p.rows; r += kEpiThreads) {
                    const float2* pr = p.part + (size_t)(r0 + r) * p.maxslots;
                    float M = -INFINITY;
                    for (int s = 0; s < touch; ++s) M = fmaxf(M, __ldcg(&pr[s].x));
                    float sum = 0.f;
                    for (int s = 0; s < touch; ++s) {
                        const float2 ml = __ldcg(pr + s);
                        if (ml.x != -INFINITY) sum += ml.y * ptx::ex2(ml.x - M);
                    }
                    lse2[r] = M + __log2f(sum);
                }
                if (!(ok = epi_sync(sb, epi_phase, p.err))) break;
                for (long long t = a; t < b && ok; ++t) {
                    const int key0 = (int)(t - first) * kTile;
                    const int j = key0 + lrow;
                    // S2: max |V[j, :]| from the staged tile (16-byte pieces in a rotated
                    // order per lane, which keeps the shared-memory reads conflict-free)
                    const int sv = vit % p.nv;
                    if (!(ok = wait_phase(&sb->vfull[sv], (vit / p.nv) & 1, sb, p.err, kErrWaitEpi))) break;
                    const uint4* vrow = (const uint4*)(Vs + sv * vstage + lrow * (D * 2));
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
                    const float s2v = fmaxf(__uint_as_float(mx << 16), __uint_as_float(mx & 0xFFFF0000u));
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sb->vempty[sv]);
                    ++vit;
                    // S1: sum over the group's window queries of 2^(t - lse2)
                    const int sa = ait % p.acc_stages;
                    if (!(ok = wait_phase(&sb->accfull[sa], (ait / p.acc_stages) & 1, sb, p.err, kErrWaitEpi))) break;
                    ptx::tc_fence_after();
                    const bool full = key0 + kTile - 1 <= window0;
                    const int jw = j - window0;       // > 0 only inside the window
                    float acc = 0.f;
                    for (int n0 = 0; n0 < p.rows; n0 += 32) {
                        float v[32];
                        __syncwarp();
                        ptx::tmem_ld_32x32b_x32(tmem + lane_bits + sa * p.acc_stride + n0, v);
                        ptx::tmem_ld_wait();
                        if (full && n0 + 32 <= p.rows) {
#pragma unroll
                            for (int e = 0; e < 32; e += 4) {
                                const float4 l4 = *(const float4*)(lse2 + n0 + e);
                                acc += ptx::ex2(fmaf(v[e + 0], p.scale2, -l4.x));
                                acc += ptx::ex2(fmaf(v[e + 1], p.scale2, -l4.y));
                                acc += ptx::ex2(fmaf(v[e + 2], p.scale2, -l4.z));
                                acc += ptx::ex2(fmaf(v[e + 3], p.scale2, -l4.w));
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const int n = n0 + e;
                                if (n < p.rows && jw <= n % p.w)
                                    acc += ptx::ex2(fmaf(v[e], p.scale2, -lse2[n]));
                            }
                        }
                    }
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sb->accempty[sa]);
                    ++ait;
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

constexpr int kQBoxRows = 64;

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
    p.mt = (plan.rows + kTile - 1) / kTile;
    const int npad = (plan.rows + 15) / 16 * 16;
    if (npad <= 256) {
        p.n1 = npad;
        p.n2 = 0;
    } else {
        p.n1 = (npad / 2 + 15) / 16 * 16;
        p.n2 = npad - p.n1;
    }
    p.tiles_per_head = plan.tiles_per_head;
    p.total_tiles = plan.total_tiles;
    p.grid = std::min(plan.grid, sms);
    // slots each head needs with this grid must fit the workspace's
    {
        const long long T = p.total_tiles;
        int need = 0;
        for (int h = 0; h < s.batch * s.hkv; ++h) {
            const long long f = (long long)h * p.tiles_per_head;
            need = std::max(need, owner_of(f + p.tiles_per_head - 1, T, p.grid) - owner_of(f, T, p.grid) + 1);
        }
        if (need > plan.maxslots) return false;
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
    // TMEM: two accumulator stages of 256 columns when both phases fit, else one of 512
    const int cols0 = p.mt * kTile, cols1 = (npad + 31) / 32 * 32;
    if (cols0 <= 256 && cols1 <= 256) {
        p.acc_stages = 2;
        p.acc_stride = 256;
    } else {
        p.acc_stages = 1;
        p.acc_stride = 512;
    }
    // shared memory: Q | K ring | V ring | lse2 | barriers (+1 KB to align the base)
    const int choices[5][2] = {{4, 2}, {3, 2}, {2, 2}, {3, 1}, {2, 1}};
    const size_t fixed = 2048 + 256 + 1024;
    size_t total = 0;
    bool fit = false;
    for (auto& c : choices) {
        total = qbytes + (size_t)(c[0] + c[1]) * tile_bytes + fixed;
        if (total <= (size_t)kSmemLimit) {
            p.nk = c[0];
            p.nv = c[1];
            fit = true;
            break;
        }
    }
    if (!fit) return false;
    p.off_q = 0;
    p.off_k = qbytes;
    p.off_v = p.off_k + p.nk * tile_bytes;
    p.off_lse = p.off_v + p.nv * tile_bytes;
    p.off_bar = p.off_lse + 2048;
    static_assert(sizeof(SmemBars) <= 256, "barrier block");
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
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lc.smem)) !=
        cudaSuccess)
        return e;
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

}  // namespace kvp
