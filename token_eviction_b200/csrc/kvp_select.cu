// Per-(sequence, KV head) top-(B - w) selection with the window always kept.
//
// "Preserving Large Activations: The Key to KV Cache Pruning" (SlimKV), Listing 1:
// window_size (w) and max_capacity_prompt (B). Kept: the w window positions
// [L - w, L) and the B - w highest scores among [0, L - w); equal scores go to the
// lower position; the list is written in ascending position order.
//
// One CTA per row. A radix select over an order-preserving 32-bit image of the fp32
// scores finds the exact threshold value T (the (B - w)-th largest) in four 8-bit
// passes, and how many elements equal to T are still needed; an ordered pass then
// emits, in position order, every element above T and the first needed ones equal to
// T, with block-wide prefix sums giving each its output slot.
#include <cuda_runtime.h>

#include "kvp_internal.cuh"

namespace kvp {
namespace {

constexpr int kSelectThreads = 1024;

// Order-preserving map of fp32 bits to uint32 (-0 is treated as +0; NaN unsupported).
__device__ __forceinline__ uint32_t order_key(uint32_t bits) {
    if (bits == 0x80000000u) bits = 0u;
    return (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
}

// Exclusive block-wide prefix sum of `x` over kSelectThreads threads; *total gets the sum.
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int ws = warp_sums[lane];
        int wi = ws;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        warp_sums[lane] = wi - ws;  // exclusive prefix of warp totals
        if (lane == 31) warp_sums[32] = wi;
    }
    __syncthreads();
    const int result = warp_sums[warp] + inc - x;
    *total = warp_sums[32];
    __syncthreads();  // warp_sums is reused by the next call
    return result;
}

__global__ void __launch_bounds__(kSelectThreads) select_topk_rows(const float* __restrict__ score,
                                                                   int32_t* __restrict__ idx,
                                                                   int L, int w, int B) {
    __shared__ unsigned hist[256];
    __shared__ int warp_sums[33];
    __shared__ unsigned s_digit, s_krem;
    const int row = blockIdx.x;
    const uint32_t* key = reinterpret_cast<const uint32_t*>(score + (size_t)row * L);
    int32_t* out = idx + (size_t)row * B;
    const int n = L - w;   // candidates
    const int kk = B - w;  // to keep among them
    const int tid = threadIdx.x;

    for (int t = tid; t < w; t += blockDim.x) out[kk + t] = n + t;
    if (kk == 0) return;
    if (kk == n) {
        for (int t = tid; t < n; t += blockDim.x) out[t] = t;
        return;
    }

    // Radix select of the kk-th largest order key, 8 bits at a time from the top.
    uint32_t prefix = 0, mask = 0, krem = (uint32_t)kk;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int t = tid; t < 256; t += blockDim.x) hist[t] = 0;
        __syncthreads();
        for (int j = tid; j < n; j += blockDim.x) {
            const uint32_t u = order_key(__ldg(key + j));
            if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid == 0) {
            uint32_t cum = 0;
            for (int dg = 255; dg >= 0; --dg) {
                const uint32_t c = hist[dg];
                if (cum + c >= krem) {
                    s_digit = (uint32_t)dg;
                    s_krem = krem - cum;
                    break;
                }
                cum += c;
            }
        }
        __syncthreads();
        prefix |= s_digit << shift;
        mask |= 255u << shift;
        krem = s_krem;
        __syncthreads();
    }
    const uint32_t T = prefix;      // order key of the kk-th largest score
    const int need_eq = (int)krem;  // how many keys equal to T are kept (lowest positions)

    int carry_eq = 0, carry_sel = 0;
    for (int base = 0; base < n; base += blockDim.x) {
        const int j = base + tid;
        const uint32_t u = j < n ? order_key(__ldg(key + j)) : 0u;
        const int gt = (j < n && u > T) ? 1 : 0;
        const int eq = (j < n && u == T) ? 1 : 0;
        int tot_eq, tot_sel;
        const int eq_rank = carry_eq + block_exclusive_scan(eq, warp_sums, &tot_eq);
        const int sel = (gt || (eq && eq_rank < need_eq)) ? 1 : 0;
        const int slot = carry_sel + block_exclusive_scan(sel, warp_sums, &tot_sel);
        if (sel) out[slot] = j;
        carry_eq += tot_eq;
        carry_sel += tot_sel;
    }
}

}  // namespace

cudaError_t launch_select(const kvp_shape& s, const Plan& p, const float* score, int32_t* idx,
                          void* scratch, cudaStream_t st) {
    (void)p;
    (void)scratch;
    select_topk_rows<<<s.batch * s.hkv, kSelectThreads, 0, st>>>(score, idx, s.seq_len, s.window,
                                                                 s.budget);
    return cudaGetLastError();
}

}  // namespace kvp
