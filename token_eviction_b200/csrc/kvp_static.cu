// kvp_score_static: the scoring call with its scratch memory built into the library.
//
// Some callers cannot allocate device memory when they evict: a serving engine that
// reserves the whole device for its own memory pool at start-up (a later cudaMalloc
// fails or fragments the pool), code running where allocation is forbidden after
// initialisation, or a host runtime that hands this library only the tensors it owns.
// For them this entry point takes the same inputs and outputs as kvp_score but no
// workspace: the scratch lives in a fixed-size array in device memory that the library
// defines, which every GPU that loads the library keeps until the process exits.
#include <cuda_runtime.h>

#include <cstdint>

#include "kvp.h"
#include "kvp_internal.cuh"

namespace kvp {
namespace {

// Largest scratch a shape may need here (its kvp_workspace_bytes); bigger shapes are
// rejected with KVP_ERR_WORKSPACE. 2 MiB covers e.g. b1 x 32/8 heads at L = 128K and
// b8 x 28/4 heads at L = 16K.
constexpr size_t kStaticScratchBytes = KVP_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of the scratch array on the current device (the array's name is only a
// host-side stand-in, not a device address). Looked up on every call: the lookup
// allocates nothing, and a cached address could outlive the device's context.
cudaError_t scratch_address(void** out) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess) return e;
    *out = ptr;
    return cudaSuccess;
}

}  // namespace
}  // namespace kvp

using namespace kvp;

extern "C" kvp_status kvp_score_static(const kvp_shape* shape, const uint16_t* q_win,
                                       const uint16_t* k, const uint16_t* v, float* score,
                                       float* s1, float* s2, void* stream) {
    if (!shape || !q_win || !k || !v || !score) return KVP_ERR_NULL;
    Plan p;
    if (!plan_of(*shape, &p)) return KVP_ERR_SHAPE;
    auto a16 = [](const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; };
    if (!a16(q_win) || !a16(k) || !a16(v) || !a16(score) || !a16(s1) || !a16(s2))
        return KVP_ERR_ALIGN;
    if (p.bytes > kStaticScratchBytes) return KVP_ERR_WORKSPACE;
    void* scratch = nullptr;
    cudaError_t e = scratch_address(&scratch);
    if (e == cudaSuccess)
        e = launch_score(*shape, p, q_win, k, v, scratch, score, s1, s2, (cudaStream_t)stream);
    if (e != cudaSuccess) return record_cuda_error(e);
    return KVP_OK;
}

extern "C" kvp_status kvp_score_static_status(void* stream) {
    void* scratch = nullptr;
    const cudaError_t e = scratch_address(&scratch);
    if (e != cudaSuccess) return record_cuda_error(e);
    return read_error_word(scratch, (cudaStream_t)stream);
}
