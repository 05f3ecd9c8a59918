// Compaction of the K/V cache to the kept positions: a 16-byte vectorised row gather.
//
// k_out[b, h, t, :] = k[b, h, idx[b, h, t], :] and the same for v, as a bit copy (the
// eviction step of "Preserving Large Activations: The Key to KV Cache Pruning",
// Listing 1: the cache keeps max_capacity_prompt positions). Each thread moves one
// 16-byte piece of one kept K row and the same piece of the V row; a grid of
// whole waves over the SMs strides over all pieces.
#include <cuda_runtime.h>

#include "kvp_internal.cuh"

namespace kvp {
namespace {

__global__ void __launch_bounds__(256) gather_rows(const uint4* __restrict__ k,
                                                   const uint4* __restrict__ v,
                                                   const int32_t* __restrict__ idx,
                                                   uint4* __restrict__ k_out,
                                                   uint4* __restrict__ v_out, int L, int B,
                                                   int piece_shift, int total, int rows_total) {
    const int stride = gridDim.x * blockDim.x;
    const int pmask = (1 << piece_shift) - 1;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
        const int rt = e >> piece_shift;      // (row, t): which kept row
        const int c = e & pmask;              // which 16-byte piece of it
        const int row = rt / B;
        const int j = __ldg(idx + rt);
        uint4 a = make_uint4(0, 0, 0, 0), b = a;
        if (j >= 0 && j < L) {
            const size_t src = (((size_t)row * L + j) << piece_shift) + c;
            a = __ldg(k + src);
            b = __ldg(v + src);
        }
        if (!KVP_CHECK(row < rows_total, 301, row, rt)) continue;
        __stcs(k_out + e, a);
        __stcs(v_out + e, b);
    }
}

}  // namespace

cudaError_t launch_compact(const kvp_shape& s, const uint16_t* k, const uint16_t* v,
                           const int32_t* idx, uint16_t* k_out, uint16_t* v_out, cudaStream_t st) {
    const int piece_shift = s.head_dim == 128 ? 4 : 3;  // 16-byte pieces per row: 16 or 8
    const long long total = ((long long)s.batch * s.hkv * s.budget) << piece_shift;
    if (total > INT32_MAX) return cudaErrorInvalidValue;
    const long long want = (total + 255) / 256;
    const int sms = num_sms();
    const long long cap = (long long)sms * 8;  // 8 resident CTAs of 256 threads per SM
    const int grid = (int)(want < cap ? want : cap);
    gather_rows<<<grid, 256, 0, st>>>((const uint4*)k, (const uint4*)v, idx, (uint4*)k_out,
                                      (uint4*)v_out, s.seq_len, s.budget, piece_shift, (int)total,
                                      s.batch * s.hkv);
    return cudaGetLastError();
}

#ifdef KVP_CHECKS
KVP_DEFINE_CHECK_READER(take_check_compact)
#endif

}  // namespace kvp
