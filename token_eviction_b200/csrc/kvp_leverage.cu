// CurDKV leverage scores on sm_100a: a streaming tcgen05 kernel and a normalisation pass.
//
// CurDKV rebuttal page (paperhub.cn/paper/klmc4fwPLd), "A clearer description of
// Algorithm 1", steps 1-4: the keys and values K, V (L x d per KV head) are projected by a
// Gaussian G (d x r, r = 20 on the page); a position's leverage score is the row norm of
// its projected key, resp. value; the two are combined and normalised. Readings: the row
// norm is squared (leverage scores are squared row norms), "combined" is the product
// lk_j * lv_j, and the normalisation divides by the sum over the head's L positions.
//
// The projection is a dense contraction (2 * L * d * r multiply-adds per KV head), so it
// runs on the tensor cores: per 128-key tile, D_K = K_tile * G and D_V = V_tile * G with
// M = 128 keys, N = 32 (G's r columns, zero-padded), K = d. The kernel is bound by reading
// K and V once from HBM: each CTA streams its flat run of tiles through a ring of (K, V)
// slot pairs by TMA, one thread issues the MMAs into four TMEM stages of 64 columns, and
// four epilogue warps (one TMEM lane quarter each, a key per thread) square and sum the
// 32 columns of each, multiply, write the combined score and keep per-warp partial sums
// of every KV head they touch in the workspace. A second small kernel (a programmatic
// dependent launch) sums a head's partials in a fixed order and divides its scores by the
// total: the result does not depend on timing.
// Warp roles: warp 0 issues the TMA loads, warp 1 allocates TMEM and issues the MMAs,
// warps 2-5 are the epilogue. Every wait is bounded; one that gives up records an error
// in the workspace's error word (kvp_workspace_status reads it).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "kvp_internal.cuh"
#include "kvp_ptx.cuh"

namespace kvp {
namespace {

constexpr int kTile = 128;                        // keys per tile
constexpr int kRPad = 32;                         // G's columns in the MMA (N)
constexpr int kStages = 4;                        // TMEM stages of 2 * kRPad columns
constexpr uint32_t kTmemCols = kStages * 2 * kRPad;
constexpr int kMaxPairs = 6;                      // (K, V) slot pairs of the load ring
constexpr int kWarpEpi = 2;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (kWarpEpi + kEpiWarps);
constexpr int kSmemLimit = 227 * 1024;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
enum : int { kErrWaitTma = 11, kErrWaitMma = 12, kErrWaitEpi = 13 };

struct LevParams {
    int L, tph, total_tiles, grid, r, npairs, maxparts;
    uint32_t tile_bytes, off_pairs, off_bar;
    const uint16_t* g;           // [d][r]
    float* score;                // [b * hkv][L]
    float* part;                 // [b * hkv][maxparts]: per epilogue warp partial sums
    int* err;
    unsigned long long wait_limit_ns;
};

struct LevBars {
    uint64_t full[kMaxPairs], empty[kMaxPairs];
    uint64_t accfull[kStages], accempty[kStages];
    uint64_t fin;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ bool lwait(uint64_t* bar, uint32_t parity, LevBars* sb, const LevParams& p,
                                      int code) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    return ptx::bounded_wait_slow(bar, parity, &sb->abort_flag, p.wait_limit_ns, p.err, code);
}
__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait_sleep(bar, parity, 20000))
        if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) return;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
leverage_tc(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
            const __grid_constant__ LevParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int kHalves = D / 64;                       // 128-byte rows per operand row
    constexpr uint32_t kHalfTile = kTile * 128;           // bytes of a tile's 64-column half
    constexpr uint32_t kGHalf = kRPad * 128;              // bytes of G^T's 64-column half
    uint8_t* Gs = smem;                                   // G^T [kHalves][32 rows][128 B], swizzled
    uint8_t* Pairs = smem + p.off_pairs;                  // [npairs][K, V][tile]
    LevBars* sb = (LevBars*)(smem + p.off_bar);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // G^T as the MMA's B operand (N = 32 rows of d bf16, K-major, 128-byte swizzle): row c
    // holds column c of G (zero for c >= r); the 16-byte chunk q of a 128-byte row sits at
    // chunk q ^ (row % 8).
    for (int idx = threadIdx.x; idx < kRPad * D; idx += kThreads) {
        const int c = idx / D, t = idx - (idx / D) * D;
        const uint16_t val = c < p.r ? p.g[t * p.r + c] : (uint16_t)0;
        const int half = t >> 6, byte = (t & 63) * 2;
        const int chunk = (byte >> 4) ^ (c & 7);
        *(uint16_t*)(Gs + half * kGHalf + c * 128 + chunk * 16 + (byte & 15)) = val;
    }
    ptx::fence_proxy_async_smem();                        // visible to the tensor cores
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMaxPairs; ++s) {
            ptx::mbar_init(&sb->full[s], 1);
            ptx::mbar_init(&sb->empty[s], 1);
        }
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&sb->accfull[s], 1);
            ptx::mbar_init(&sb->accempty[s], kEpiWarps);
        }
        ptx::mbar_init(&sb->fin, 1);
        sb->abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
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

    // this CTA's flat run of tiles [t0, t1) of the (sequence, KV head, tile) space
    const uint32_t T = (uint32_t)p.total_tiles, grid = (uint32_t)p.grid;
    const int t0 = (int)(blockIdx.x * T / grid), t1 = (int)((blockIdx.x + 1) * T / grid);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            const uint64_t pol = ptx::policy_evict_first();
            uint32_t epar = 0, used = 0;                  // per pair: load parity, any load
            int s = 0;
            bool ok = true;
            for (int t = t0; t < t1 && ok; ++t) {
                const int head = t / p.tph, key0 = (t - head * p.tph) * kTile;
                if (!(ok = lwait(&sb->empty[s], ((epar >> s) & 1) ^ 1, sb, p, kErrWaitTma))) break;
                ptx::mbar_arrive_expect_tx(&sb->full[s], 2 * p.tile_bytes);
                uint8_t* kd = Pairs + (2 * s) * p.tile_bytes;
                uint8_t* vd = kd + p.tile_bytes;
#pragma unroll
                for (int c = 0; c < kHalves; ++c) {
                    ptx::tma_load_3d(kd + c * kHalfTile, &kmap, &sb->full[s], c * 64, key0, head, pol);
                    ptx::tma_load_3d(vd + c * kHalfTile, &vmap, &sb->full[s], c * 64, key0, head, pol);
                }
                epar ^= 1u << s;
                used |= 1u << s;
                s = s + 1 == p.npairs ? 0 : s + 1;
            }
            // no copy may still be landing when the CTA exits
            for (int q = 0; q < p.npairs; ++q)
                if ((used >> q) & 1) drain(&sb->full[q], ((epar >> q) & 1) ^ 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            const uint32_t idesc = ptx::idesc_bf16_f32(kTile, kRPad);
            const uint64_t gdesc = ptx::sw128_kmajor_desc(ptx::smem_u32(Gs));
            uint32_t fpar = 0, apar = 0;
            int s = 0, i = 0;
            bool ok = true;
            for (int t = t0; t < t1 && ok; ++t, ++i) {
                const int st = i & (kStages - 1);
                if (!(ok = lwait(&sb->full[s], (fpar >> s) & 1, sb, p, kErrWaitMma))) break;
                fpar ^= 1u << s;
                if (!(ok = lwait(&sb->accempty[st], ((apar >> st) & 1) ^ 1, sb, p, kErrWaitMma))) break;
                apar ^= 1u << st;
                ptx::tc_fence_after();
                const uint32_t kaddr = ptx::smem_u32(Pairs + (2 * s) * p.tile_bytes);
                const uint64_t kdesc = ptx::sw128_kmajor_desc(kaddr);
                const uint64_t vdesc = ptx::sw128_kmajor_desc(kaddr + p.tile_bytes);
                const uint32_t d0 = tmem + (uint32_t)(st * 2 * kRPad);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t ao = ((ks >> 2) * kHalfTile + (ks & 3) * 32) >> 4;
                    const uint32_t bo = ((ks >> 2) * kGHalf + (ks & 3) * 32) >> 4;
                    ptx::mma_bf16_ss(d0, kdesc + ao, gdesc + bo, idesc, ks > 0);
                    ptx::mma_bf16_ss(d0 + kRPad, vdesc + ao, gdesc + bo, idesc, ks > 0);
                }
                ptx::mma_commit(&sb->accfull[st]);
                ptx::mma_commit(&sb->empty[s]);
                s = s + 1 == p.npairs ? 0 : s + 1;
            }
            ptx::mma_commit(&sb->fin);
            drain(&sb->fin, 0);
        }
    } else {
        // ---------------------------------------------------- epilogue (warps 2-5)
        const int quarter = warp & 3;                     // TMEM lane quarter
        const int key = quarter * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
        const int ew = warp - kWarpEpi;                   // 0 .. 3
        // partial sums: slot of this warp within the head = (CTA's index among the head's
        // CTAs) * 4 + ew
        float part = 0.f;
        int cur = -1;
        auto flush = [&](int head) {
            float x = part;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
            const uint32_t first = (uint32_t)head * (uint32_t)p.tph;
            const int slot = (int)(blockIdx.x - owner_of_u32(first, T, grid)) * kEpiWarps + ew;
            if (lane == 0 && KVP_CHECK(slot < p.maxparts, 301, head, slot))
                p.part[(size_t)head * p.maxparts + slot] = x;
        };
        uint32_t apar = 0;
        int i = 0;
        for (int t = t0; t < t1; ++t, ++i) {
            const int head = t / p.tph, key0 = (t - head * p.tph) * kTile;
            if (head != cur) {
                if (cur >= 0) flush(cur);
                cur = head;
                part = 0.f;
            }
            const int st = i & (kStages - 1);
            if (!__all_sync(0xffffffffu, lwait(&sb->accfull[st], (apar >> st) & 1, sb, p, kErrWaitEpi))) {
                cur = -1;                                 // unwinding: nothing more is written
                break;
            }
            apar ^= 1u << st;
            ptx::tc_fence_after();
            float a[32], b[32];
            __syncwarp();
            ptx::tmem_ld_32x32b_x32(tl + (uint32_t)(st * 2 * kRPad), a);
            ptx::tmem_ld_32x32b_x32(tl + (uint32_t)(st * 2 * kRPad + kRPad), b);
            ptx::tmem_ld_wait(a);
            ptx::tmem_ld_wait(b);
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sb->accempty[st]);
            // columns past r are exact zeros (G^T's padding rows), so all 32 may be summed
            float lk0 = 0.f, lk1 = 0.f, lv0 = 0.f, lv1 = 0.f;
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                lk0 = fmaf(a[c], a[c], lk0);
                lk1 = fmaf(a[c + 1], a[c + 1], lk1);
                lv0 = fmaf(b[c], b[c], lv0);
                lv1 = fmaf(b[c + 1], b[c + 1], lv1);
            }
            const float prod = (lk0 + lk1) * (lv0 + lv1);
            const int j = key0 + key;
            if (j < p.L) {
                p.score[(size_t)head * p.L + j] = prod;
                part += prod;
            }
        }
        if (cur >= 0) flush(cur);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// Divides every score of a head by the sum of its partials. Block (x, y): head y,
// positions of chunk x. The head's partial slots (its CTAs' epilogue warps, all written)
// are summed by every block in one fixed order: per thread over slots q, q + 256, ...,
// then a fixed shuffle tree and the warps in order, so every block and every call agree.
// Launched as a programmatic dependent of the scoring grid: everything before the
// dependency wait overlaps that grid's tail.
__global__ void __launch_bounds__(256)
leverage_normalise(float* __restrict__ score, const float* __restrict__ part, int L, int maxparts,
                   uint32_t T, uint32_t grid, uint32_t tph, const int* __restrict__ err) {
    __shared__ float warp_sum[8];
    const int head = blockIdx.y;
    const uint32_t first = (uint32_t)head * tph;
    const int nparts = (int)(owner_of_u32(first + tph - 1, T, grid) - owner_of_u32(first, T, grid) + 1) * kEpiWarps;
    asm volatile("griddepcontrol.wait;" ::: "memory");   // the scoring grid has completed
    if (*(volatile const int*)err != 0) return;           // the scores were not all written
    float x = 0.f;
    for (int q = threadIdx.x; q < nparts && q < maxparts; q += 256) x += part[(size_t)head * maxparts + q];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = x;
    __syncthreads();
    float total = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) total += warp_sum[w];
    const float inv = total > 0.f ? 1.f / total : 0.f;
    float* row = score + (size_t)head * L;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < L; j += gridDim.x * blockDim.x)
        row[j] = total > 0.f ? row[j] * inv : 0.f;
}

}  // namespace

size_t leverage_part_bytes(const kvp_shape& s, const Plan& plan, int grid, int* maxparts) {
    const long long units = (long long)s.batch * s.hkv;
    int need = 0;
    for (long long h = 0; h < units; ++h)
        need = std::max(need, ctas_touching(h, plan.total_tiles, grid, plan.tiles_per_head, 0));
    *maxparts = need * kEpiWarps;
    return (size_t)units * (size_t)(*maxparts) * sizeof(float);
}

cudaError_t launch_leverage(const kvp_shape& s, const Plan& plan, const uint16_t* k, const uint16_t* v,
                            const uint16_t* g, int r, float* score, void* workspace, cudaStream_t st) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int D = s.head_dim;
    LevParams p = {};
    p.L = s.seq_len;
    p.tph = plan.tiles_per_head;
    p.total_tiles = plan.total_tiles;
    // a flat cut over the SMs (kPlanGrid on a B200); the partial slots are counted for it
    p.grid = std::min(std::min(kPlanGrid, sms), plan.total_tiles);
    p.r = r;
    p.tile_bytes = (uint32_t)kTile * D * 2;
    const uint32_t gbytes = (uint32_t)kRPad * D * 2;
    p.off_pairs = gbytes;
    const size_t fixed = gbytes + sizeof(LevBars) + 1024 + 64;
    p.npairs = (int)std::min<size_t>(kMaxPairs, ((size_t)kSmemLimit - fixed) / (2 * p.tile_bytes));
    if (p.npairs < 2) return cudaErrorInvalidConfiguration;
    p.off_bar = p.off_pairs + (uint32_t)p.npairs * 2 * p.tile_bytes;
    const size_t smem = (size_t)p.off_bar + sizeof(LevBars) + 1024;
    if (plan.off_part + leverage_part_bytes(s, plan, p.grid, &p.maxparts) > plan.off_select)
        return cudaErrorInvalidConfiguration;
    char* ws = (char*)workspace;
    p.g = g;
    p.score = score;
    p.part = (float*)(ws + plan.off_part);
    p.err = (int*)(ws + plan.off_err);
    p.wait_limit_ns = kWaitLimitNs;

    CUtensorMap kmap, vmap;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)s.seq_len, (cuuint64_t)s.batch * s.hkv};
        const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)s.seq_len * D * 2};
        const cuuint32_t box[3] = {64, kTile, 1};
        if (!make_map(&kmap, k, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_map(&vmap, v, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    // the error word starts at zero (every partial slot a head has is written)
    if ((e = cudaMemsetAsync(ws + plan.off_err, 0, sizeof(int), st)) != cudaSuccess) return e;
    void (*kern)(const CUtensorMap, const CUtensorMap, const LevParams) =
        D == 128 ? leverage_tc<128> : leverage_tc<64>;
    if ((e = allow_dynamic_smem((const void*)kern, smem)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    if ((e = cudaLaunchKernelEx(&cfg, kern, kmap, vmap, p)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg2 = {};
    const int chunks = std::max(1, std::min(64, (s.seq_len + 4095) / 4096));
    cfg2.gridDim = dim3(chunks, s.batch * s.hkv);
    cfg2.blockDim = dim3(256);
    cfg2.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg2.attrs = attr;
    cfg2.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg2, leverage_normalise, score, (const float*)p.part, s.seq_len,
                              p.maxparts, (uint32_t)p.total_tiles, (uint32_t)p.grid,
                              (uint32_t)p.tph, (const int*)p.err);
}

#ifdef KVP_CHECKS
KVP_DEFINE_CHECK_READER(take_check_leverage)
#endif

}  // namespace kvp
