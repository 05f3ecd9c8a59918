// Compaction of the K/V cache to the kept positions: a vectorised row gather.
//
// k_out[b, h, t, :] = k[b, h, idx[b, h, t], :] and the same for v, as a bit copy (the
// eviction step of "Preserving Large Activations: The Key to KV Cache Pruning",
// Listing 1: the cache keeps max_capacity_prompt positions). Each thread moves four
// 16-byte pieces of the kept K rows (32 pieces apart, so that a warp's every instruction
// covers 512 contiguous bytes) and the same pieces of V, with all eight loads issued
// before any store so that enough bytes are in flight to keep HBM busy; a grid of whole
// waves over the SMs strides over all pieces.
#include <cuda_runtime.h>

#include "kvp_internal.cuh"
#include "kvp_ptx.cuh"

namespace kvp {
namespace {

constexpr int kPiecesPerThread = 4;   // 16-byte pieces of K (and of V) per thread
constexpr int kThreads = 256;

// Each warp moves a block of 128 consecutive 16-byte output pieces of K and the same of V:
// lane l takes pieces l, l + 32, l + 64 and l + 96, so that every load and store
// instruction of the warp covers 512 contiguous bytes, and all eight loads are issued
// before any store.
__global__ void __launch_bounds__(kThreads) gather_rows(const uint4* __restrict__ k,
                                                        const uint4* __restrict__ v,
                                                        const int32_t* __restrict__ idx,
                                                        uint4* __restrict__ k_out,
                                                        uint4* __restrict__ v_out, int L, int B,
                                                        int piece_shift, int total, int rows_total) {
    ptx::grid_dependency_wait();         // the indices' producer has completed
    constexpr int kBlock = 32 * kPiecesPerThread;
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kThreads / 32);
    const int pmask = (1 << piece_shift) - 1;
    for (int w = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); (long long)w * kBlock < total;
         w += nwarps) {
        int e[kPiecesPerThread], j[kPiecesPerThread];
#pragma unroll
        for (int q = 0; q < kPiecesPerThread; ++q) {
            e[q] = w * kBlock + q * 32 + lane;
            j[q] = e[q] < total ? __ldg(idx + (e[q] >> piece_shift)) : -1;
        }
        uint4 a[kPiecesPerThread], b[kPiecesPerThread];
#pragma unroll
        for (int q = 0; q < kPiecesPerThread; ++q) {
            const int rt = e[q] >> piece_shift;           // which kept row (row * B + t)
            if (e[q] < total && j[q] >= 0 && j[q] < L) {
                const size_t src = (((size_t)(rt / B) * L + j[q]) << piece_shift) + (e[q] & pmask);
                a[q] = __ldg(k + src);
                b[q] = __ldg(v + src);
            } else {
                a[q] = b[q] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int q = 0; q < kPiecesPerThread; ++q) {
            if (e[q] >= total || !KVP_CHECK((e[q] >> piece_shift) / B < rows_total, 301, e[q], B)) continue;
            __stcs(k_out + e[q], a[q]);
            __stcs(v_out + e[q], b[q]);
        }
    }
}

}  // namespace

cudaError_t launch_compact(const kvp_shape& s, const uint16_t* k, const uint16_t* v,
                           const int32_t* idx, uint16_t* k_out, uint16_t* v_out, cudaStream_t st) {
    const int piece_shift = s.head_dim == 128 ? 4 : 3;  // 16-byte pieces per row: 16 or 8
    const long long total = ((long long)s.batch * s.hkv * s.budget) << piece_shift;
    if (total > INT32_MAX) return cudaErrorInvalidValue;
    const long long want = (total + 32 * kPiecesPerThread * (kThreads / 32) - 1) /
                           (32 * kPiecesPerThread * (kThreads / 32));
    // whole waves over the SMs (8 resident CTAs of 256 threads each), so that no SM
    // carries a second round of CTAs while the others idle
    const long long sms = num_sms(), cap = sms * 8;
    const long long grid = want < cap ? (want + sms - 1) / sms * sms : cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlaps the launch
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // launched with cudaLaunchKernelEx: its return value is this launch's own error, never
    // a sticky error left by an earlier, unrelated launch
    return cudaLaunchKernelEx(&cfg, gather_rows, (const uint4*)k, (const uint4*)v, idx, (uint4*)k_out,
                              (uint4*)v_out, s.seq_len, s.budget, piece_shift, (int)total,
                              s.batch * s.hkv);
}

#ifdef KVP_CHECKS
KVP_DEFINE_CHECK_READER(take_check_compact)
#endif

}  // namespace kvp
