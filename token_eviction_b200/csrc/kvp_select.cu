// Per-(sequence, KV head) top-(B - w) selection with the window always kept.
//
// "Preserving Large Activations: The Key to KV Cache Pruning" (SlimKV), Listing 1:
// window_size (w) and max_capacity_prompt (B). Kept: the w window positions
// [L - w, L) and the B - w highest scores among [0, L - w); equal scores go to the
// lower position; the list is written in ascending position order.
//
// The policy variant (kvp_select_policy) keeps the first s positions (attention sinks) and
// ranks the candidates [s, L - w) by a key formed from S1 and S2 (see SelSource).
//
// One thread-block cluster of kCl CTAs per row. Each CTA holds a contiguous slice of
// the row's candidates in shared memory as order-preserving 32-bit keys (the fp32 bit
// pattern with the sign handled so that unsigned order equals numeric order).
// A radix select over the keys finds the exact threshold T (the (B - w)-th largest key)
// in three passes of 11, 11 and 10 bits: every CTA histograms its slice (only keys that
// match the prefix found so far), adds its histogram into the leader CTA's through
// distributed shared memory, and the leader picks the digit where the count from the top
// reaches the number still needed. The emission then writes, in position order, every key
// above T and the first keys equal to T (as many as still needed); each warp's output
// offset comes from counts exchanged across the cluster. Only cluster and block
// barriers are used: every CTA takes the same steps, so none can wait forever.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include "kvp_internal.cuh"
#include "kvp_ptx.cuh"

namespace cg = cooperative_groups;

namespace kvp {
namespace {

constexpr int kCl = 8;              // CTAs per row (portable cluster size)
constexpr int kSelThreads = 1024;
constexpr int kWarps = kSelThreads / 32;
constexpr int kBins = 2048;
constexpr int kSliceCap = 40960;    // keys per CTA held in shared memory

// Order-preserving map of fp32 bits to uint32 (-0 is treated as +0; NaN unsupported).
__device__ __forceinline__ uint32_t order_key(uint32_t bits) {
    if (bits == 0x80000000u) bits = 0u;
    return (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
}

struct SelShared {
    unsigned hist[kBins];      // this CTA's histogram
    unsigned merged[kBins];    // leader only: the cluster's histogram
    unsigned digit, krem;      // leader only: result of the current pass
    unsigned cta_gt[kCl], cta_eq[kCl];  // leader only: per-CTA counts for the emission
    unsigned warp_gt[kWarps], warp_eq[kWarps];
    unsigned warp_sel_off[kWarps], warp_eq_off[kWarps];
    int scan[kWarps + 1];
};

// Exclusive prefix sum over the block (kSelThreads threads); returns this thread's.
__device__ __forceinline__ int block_exclusive_scan(int x, int* ws) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) ws[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int v = ws[lane];
        int wi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        ws[lane] = wi - v;
    }
    __syncthreads();
    const int r = ws[warp] + inc - x;
    __syncthreads();
    return r;
}

// What a row is ranked by. Plain (s1 == nullptr): the score itself, over [0, L - w).
// Policy: candidates [sinks, L - w), ranked by a key formed from S1 and S2 in fp32:
//   pool(S1)[j] = max of S1 over [j - kernel/2, j + kernel/2] within [0, L - w)
//   mode 0: pool(S1) * S2 (IEEE multiply, no flush of subnormal operands); 1: pool(S1);
//   2: S2; a subnormal key counts as zero.
// The first `sinks` positions are always kept.
struct SelSource {
    const float* score;
    const float* s1;
    const float* s2;
    int sinks, kernel, mode;
};

__device__ __forceinline__ float mul_rn_noftz(float a, float b) {
    float r;
    asm("mul.rn.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Order-preserving key of candidate j of a row (row pointers already offset).
__device__ __forceinline__ uint32_t source_key(const SelSource& src, const float* srow, const float* s1row,
                                               const float* s2row, int j, int n) {
    if (srow) return order_key(__float_as_uint(__ldg(srow + j)));
    float key;
    if (src.mode == 2) {
        key = __ldg(s2row + j);
    } else {
        // S1 >= 0: the largest bit pattern is the largest value, subnormals included
        const int half = src.kernel >> 1;
        uint32_t pooled = __float_as_uint(__ldg(s1row + j));
        for (int t = max(0, j - half); t <= min(n - 1, j + half); ++t)
            pooled = max(pooled, __float_as_uint(__ldg(s1row + t)));
        key = src.mode == 1 ? __uint_as_float(pooled) : mul_rn_noftz(__uint_as_float(pooled), __ldg(s2row + j));
    }
    uint32_t bits = __float_as_uint(key);
    if ((bits & 0x7F800000u) == 0u) bits = 0u;     // zero or subnormal: zero
    return order_key(bits);
}

template <bool kInSmem>
__global__ void __launch_bounds__(kSelThreads, 1)
select_cluster(const SelSource src, int32_t* __restrict__ idx, int L, int w, int B, int slice) {
    extern __shared__ uint32_t keys[];   // [slice] when kInSmem
    __shared__ SelShared sh;
    ptx::grid_dependency_wait();         // the scores' producer has completed
    cg::cluster_group cluster = cg::this_cluster();
    const unsigned rank = cluster.block_rank();
    const int row = blockIdx.x / kCl;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = L - w, s0 = src.sinks, kk = B - w - s0;
    // plain when score is given; otherwise a policy key (s1 is NULL when mode 2 ranks by S2)
    const float* srow = src.score ? src.score + (size_t)row * L : nullptr;
    const float* s1row = src.s1 ? src.s1 + (size_t)row * L : nullptr;
    const float* s2row = src.s2 ? src.s2 + (size_t)row * L : nullptr;
    int32_t* out = idx + (size_t)row * B;

    // sinks, then the kk selected candidates, then the window: all ascending
    if (rank == 0) {
        for (int t = tid; t < s0; t += kSelThreads) out[t] = t;
        for (int t = tid; t < w; t += kSelThreads) out[s0 + kk + t] = n + t;
    }
    out += s0;
    if (kk == 0) return;                  // same decision in every CTA of the cluster
    if (kk == n - s0) {
        for (int t = (int)rank * kSelThreads + tid; t < n - s0; t += kCl * kSelThreads) out[t] = s0 + t;
        return;
    }

    // this CTA's slice of the candidates [s0, n)
    const int lo = min(n, s0 + (int)rank * slice), hi = min(n, lo + slice);
    auto key_at = [&](int j) -> uint32_t {  // j in [lo, hi)
        if (kInSmem) return keys[j - lo];
        return source_key(src, srow, s1row, s2row, j, n);
    };
    if (kInSmem) {
        for (int j = lo + tid; j < hi; j += kSelThreads) keys[j - lo] = source_key(src, srow, s1row, s2row, j, n);
    }
    SelShared* leader = cluster.map_shared_rank(&sh, 0);

    // ---- radix select: 11 + 11 + 10 bits from the top
    uint32_t prefix = 0, mask = 0, krem = (uint32_t)kk;
    const int shifts[3] = {21, 10, 0};
    const uint32_t widths[3] = {2047u, 2047u, 1023u};
    for (int b = tid; b < kBins; b += kSelThreads) {
        sh.hist[b] = 0;
        if (rank == 0) sh.merged[b] = 0;
    }
    cluster.sync();                        // histograms cleared (and keys staged)
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = shifts[pass];
        const uint32_t dmask = widths[pass];
        for (int j = lo + tid; j < hi; j += kSelThreads) {
            const uint32_t u = key_at(j);
            if ((u & mask) == prefix) atomicAdd(&sh.hist[(u >> shift) & dmask], 1u);
        }
        __syncthreads();
        for (int b = tid; b < kBins; b += kSelThreads)
            if (sh.hist[b]) atomicAdd(&leader->merged[b], sh.hist[b]);
        cluster.sync();                    // merged histogram complete
        if (rank == 0) {
            // thread t holds the bin pair (2047 - 2t, 2046 - 2t): count of all higher bins
            const int bh = kBins - 1 - 2 * tid, bl = bh - 1;
            const unsigned ch = sh.merged[bh], cl = sh.merged[bl];
            const unsigned above = (unsigned)block_exclusive_scan((int)(ch + cl), sh.scan);
            if (above < krem && krem <= above + ch) {
                sh.digit = (unsigned)bh;
                sh.krem = krem - above;
            } else if (above + ch < krem && krem <= above + ch + cl) {
                sh.digit = (unsigned)bl;
                sh.krem = krem - above - ch;
            }
            // every read of the merged histogram precedes the scan's barriers: clear it
            // for the next pass under the same cluster barrier that publishes the digit
            sh.merged[bh] = 0;
            sh.merged[bl] = 0;
        }
        for (int b = tid; b < kBins; b += kSelThreads) sh.hist[b] = 0;   // read above, by this thread
        cluster.sync();                    // digit published, histograms cleared
        const unsigned dg = leader->digit, kr = leader->krem;
        prefix |= dg << shift;
        mask |= dmask << shift;
        krem = kr;
    }
    const uint32_t T = prefix;             // key of the (B - w)-th largest score
    const unsigned need_eq = krem;         // keys equal to T that are kept (lowest positions)

    // ---- ordered emission: warp w covers a contiguous stretch of this CTA's slice
    const int span = hi - lo;
    const int per_warp = ((span + kWarps - 1) / kWarps + 31) / 32 * 32;
    const int wlo = lo + warp * per_warp, whi = min(hi, wlo + per_warp);
    unsigned cgt = 0, ceq = 0;
    for (int j0 = wlo; j0 < whi; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t u = j < whi ? key_at(j) : 0u;
        cgt += __popc(__ballot_sync(0xffffffffu, j < whi && u > T));
        ceq += __popc(__ballot_sync(0xffffffffu, j < whi && u == T));
    }
    if (lane == 0) {
        sh.warp_gt[warp] = cgt;
        sh.warp_eq[warp] = ceq;
    }
    __syncthreads();
    if (warp == 0) {
        unsigned g = sh.warp_gt[lane], e = sh.warp_eq[lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, o);
            e += __shfl_xor_sync(0xffffffffu, e, o);
        }
        if (lane == 0) {
            leader->cta_gt[rank] = g;
            leader->cta_eq[rank] = e;
        }
    }
    cluster.sync();                        // every CTA's counts at the leader
    if (warp == 0) {
        // offsets of this CTA: equal keys and kept keys in all lower-ranked CTAs
        unsigned eq_before = 0, sel_before = 0;
        for (unsigned r = 0; r < rank; ++r) {
            const unsigned g = leader->cta_gt[r], e = leader->cta_eq[r];
            const unsigned take = eq_before >= need_eq ? 0u : min(e, need_eq - eq_before);
            sel_before += g + take;
            eq_before += e;
        }
        // then per warp, in position order
        const unsigned g = sh.warp_gt[lane], e = sh.warp_eq[lane];
        unsigned einc = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, einc, o);
            if (lane >= o) einc += y;
        }
        const unsigned weq_before = eq_before + einc - e;
        const unsigned take = weq_before >= need_eq ? 0u : min(e, need_eq - weq_before);
        const unsigned s = g + take;
        unsigned sinc = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, sinc, o);
            if (lane >= o) sinc += y;
        }
        sh.warp_sel_off[lane] = sel_before + sinc - s;
        sh.warp_eq_off[lane] = weq_before;
    }
    __syncthreads();
    unsigned pos = sh.warp_sel_off[warp], eq_run = sh.warp_eq_off[warp];
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int j0 = wlo; j0 < whi; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t u = j < whi ? key_at(j) : 0u;
        const bool gt = j < whi && u > T, eq = j < whi && u == T;
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const unsigned eq_rank = eq_run + __popc(eqm & lt_mask);
        const bool sel = gt || (eq && eq_rank < need_eq);
        const unsigned selm = __ballot_sync(0xffffffffu, sel);
        if (sel) {
            const unsigned slot = pos + __popc(selm & lt_mask);
            if (KVP_CHECK(slot < (unsigned)kk, 101, row, (int)slot)) out[slot] = j;
        }
        pos += __popc(selm);
        eq_run += __popc(eqm);
    }
    cluster.sync();                        // the leader's shared memory outlives its readers
}

}  // namespace

namespace {

// rows rows of L scores each: candidates [sinks, L - w), budget B (window and sinks included)
cudaError_t launch_select_source(int rows, int L, int w, int B, const SelSource& src, int32_t* idx,
                                 cudaStream_t st) {
    const int nc = L - w - src.sinks;                     // candidates
    const int slice = (nc + kCl - 1) / kCl;
    const bool in_smem = slice <= kSliceCap;
    const size_t dyn = in_smem ? (size_t)slice * sizeof(uint32_t) : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rows * kCl);
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // launched as a programmatic dependent: its launch overlaps the producer's tail, and
    // every CTA waits for the producer (grid_dependency_wait) before reading
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e;
    if (in_smem) {
        if ((e = allow_dynamic_smem((const void*)select_cluster<true>, dyn)) != cudaSuccess) return e;
        return cudaLaunchKernelEx(&cfg, select_cluster<true>, src, idx, L, w, B, slice);
    }
    return cudaLaunchKernelEx(&cfg, select_cluster<false>, src, idx, L, w, B, slice);
}

}  // namespace

cudaError_t launch_select_rows(int rows, int L, int w, int B, const float* score, int32_t* idx,
                               cudaStream_t st) {
    const SelSource src = {score, nullptr, nullptr, 0, 1, 0};
    return launch_select_source(rows, L, w, B, src, idx, st);
}

cudaError_t launch_select(const kvp_shape& s, const Plan& p, const float* score, int32_t* idx,
                          void* scratch, cudaStream_t st) {
    (void)p;
    (void)scratch;
    const SelSource src = {score, nullptr, nullptr, 0, 1, 0};
    return launch_select_source(s.batch * s.hkv, s.seq_len, s.window, s.budget, src, idx, st);
}

cudaError_t launch_select_policy(const kvp_shape& s, const kvp_policy& pol, const float* s1,
                                 const float* s2, int32_t* idx, cudaStream_t st) {
    const SelSource src = {nullptr, s1, s2, pol.sinks, pol.pool_kernel, pol.mode};
    return launch_select_source(s.batch * s.hkv, s.seq_len, s.window, s.budget, src, idx, st);
}

#ifdef KVP_CHECKS
KVP_DEFINE_CHECK_READER(take_check_select)
#endif

}  // namespace kvp
