// C ABI of the kvp library: argument checks, workspace layout, launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <vector>
#include <cstdint>

#include "kvp.h"
#include "kvp_internal.cuh"

namespace kvp {

int num_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
        return n;
    return 148;
}

cudaError_t allow_dynamic_smem(const void* func, size_t bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    struct Entry {
        int dev;
        const void* func;
    };
    static std::mutex mu;
    static std::vector<Entry> raised;
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& r : raised)
        if (r.dev == dev && r.func == func) return cudaSuccess;
    int optin = 0;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, func)) != cudaSuccess) return e;
    // the opt-in maximum covers static and dynamic shared memory together
    const size_t max_dynamic = (size_t)optin > fa.sharedSizeBytes ? (size_t)optin - fa.sharedSizeBytes : 0;
    if (bytes > max_dynamic) return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_dynamic)) !=
        cudaSuccess)
        return e;
    raised.push_back({dev, func});
    return cudaSuccess;
}

}  // namespace kvp

using namespace kvp;

static bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

// The CUDA error behind the calling thread's last KVP_ERR_CUDA (cudaSuccess if none).
static thread_local cudaError_t t_last_cuda_error = cudaSuccess;

namespace kvp {

kvp_status record_cuda_error(cudaError_t e) {
    t_last_cuda_error = e;
    cudaGetLastError();  // clear the runtime's sticky copy of a launch error
    return KVP_ERR_CUDA;
}

kvp_status read_error_word(const void* workspace, cudaStream_t stream) {
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return record_cuda_error(e);
    return word != 0 ? KVP_ERR_TIMEOUT : KVP_OK;
}

}  // namespace kvp

static kvp_status cuda_failed(cudaError_t e) { return record_cuda_error(e); }

extern "C" size_t kvp_workspace_bytes(const kvp_shape* shape) {
    Plan p;
    if (!shape || !plan_of(*shape, &p)) return 0;
    return p.bytes;
}

extern "C" kvp_status kvp_score(const kvp_shape* shape, const uint16_t* q_win, const uint16_t* k,
                                const uint16_t* v, float* score, float* s1, float* s2,
                                void* workspace, size_t workspace_bytes, void* stream) {
    if (!shape || !q_win || !k || !v || !score) return KVP_ERR_NULL;
    Plan p;
    if (!plan_of(*shape, &p)) return KVP_ERR_SHAPE;
    if (!aligned16(q_win) || !aligned16(k) || !aligned16(v) || !aligned16(score) ||
        !aligned16(s1) || !aligned16(s2))
        return KVP_ERR_ALIGN;
    if (!workspace || workspace_bytes < p.bytes) return KVP_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KVP_ERR_ALIGN;
    const cudaError_t e =
        launch_score(*shape, p, q_win, k, v, workspace, score, s1, s2, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_failed(e);
    return KVP_OK;
}

extern "C" kvp_status kvp_select(const kvp_shape* shape, const float* score, int32_t* idx,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    if (!shape || !score || !idx) return KVP_ERR_NULL;
    Plan p;
    if (!plan_of(*shape, &p)) return KVP_ERR_SHAPE;
    if (!aligned16(score) || !aligned16(idx)) return KVP_ERR_ALIGN;
    if (!workspace || workspace_bytes < p.bytes) return KVP_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KVP_ERR_ALIGN;
    const cudaError_t e =
        launch_select(*shape, p, score, idx, (char*)workspace + p.off_select, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_failed(e);
    return KVP_OK;
}

extern "C" kvp_status kvp_select_policy(const kvp_shape* shape, const kvp_policy* policy,
                                        const float* s1, const float* s2, int32_t* idx, void* stream) {
    if (!shape || !policy || !idx) return KVP_ERR_NULL;
    const int mode = policy->mode;
    if (mode < KVP_RANK_PRODUCT || mode > KVP_RANK_S2) return KVP_ERR_SHAPE;
    if ((mode != KVP_RANK_S2 && !s1) || (mode != KVP_RANK_S1 && !s2)) return KVP_ERR_NULL;
    Plan p;
    if (!plan_of(*shape, &p)) return KVP_ERR_SHAPE;
    const int k = policy->pool_kernel, sinks = policy->sinks;
    if (k < 1 || k > 255 || k % 2 == 0) return KVP_ERR_SHAPE;
    if (sinks < 0 || sinks + shape->window > shape->budget || sinks > shape->seq_len - shape->window)
        return KVP_ERR_SHAPE;
    if (!aligned16(s1) || !aligned16(s2) || !aligned16(idx)) return KVP_ERR_ALIGN;
    const cudaError_t e = launch_select_policy(*shape, *policy, mode == KVP_RANK_S2 ? nullptr : s1,
                                               mode == KVP_RANK_S1 ? nullptr : s2, idx, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_failed(e);
    return KVP_OK;
}

extern "C" kvp_status kvp_leverage(const kvp_shape* shape, const uint16_t* k, const uint16_t* v,
                                   const uint16_t* g, int32_t r, float* score, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    if (!shape || !k || !v || !g || !score) return KVP_ERR_NULL;
    Plan p;
    if (!plan_of(*shape, &p)) return KVP_ERR_SHAPE;
    if (r < 1 || r > 32) return KVP_ERR_SHAPE;
    if (!aligned16(k) || !aligned16(v) || !aligned16(score) || ((uintptr_t)g & 1u)) return KVP_ERR_ALIGN;
    if (!workspace || workspace_bytes < p.bytes) return KVP_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KVP_ERR_ALIGN;
    int maxparts = 0;
    const int grid = std::min(kPlanGrid, p.total_tiles);
    if (p.off_part + leverage_part_bytes(*shape, p, grid, &maxparts) > p.off_select) return KVP_ERR_SHAPE;
    const cudaError_t e = launch_leverage(*shape, p, k, v, g, r, score, workspace, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_failed(e);
    return KVP_OK;
}

// KV heads per sequence that the adaptive calls accept (their offsets sit in shared memory)
static constexpr int kMaxAdaptiveHeads = 4096;

extern "C" size_t kvp_adaptive_workspace_bytes(const kvp_shape* shape) {
    Plan p;
    if (!shape || !plan_of(*shape, &p) || shape->hkv > kMaxAdaptiveHeads) return 0;
    return adaptive_workspace_bytes(*shape);
}

extern "C" kvp_status kvp_select_adaptive(const kvp_shape* shape, float alpha, const float* score,
                                          int32_t* idx, int32_t* counts, void* workspace,
                                          size_t workspace_bytes, void* stream) {
    if (!shape || !score || !idx || !counts) return KVP_ERR_NULL;
    Plan p;
    if (!plan_of(*shape, &p) || shape->hkv > kMaxAdaptiveHeads) return KVP_ERR_SHAPE;
    if (!(alpha >= 0.f && alpha <= 1.f)) return KVP_ERR_SHAPE;
    if (!aligned16(score) || !aligned16(idx) || !aligned16(counts)) return KVP_ERR_ALIGN;
    if (!workspace || workspace_bytes < adaptive_workspace_bytes(*shape)) return KVP_ERR_WORKSPACE;
    if (!aligned16(workspace)) return KVP_ERR_ALIGN;
    const cudaError_t e =
        launch_select_adaptive(*shape, alpha, score, idx, counts, workspace, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_failed(e);
    return KVP_OK;
}

extern "C" kvp_status kvp_compact_ragged(const kvp_shape* shape, const uint16_t* k, const uint16_t* v,
                                         const int32_t* idx, const int32_t* counts, uint16_t* k_out,
                                         uint16_t* v_out, void* stream) {
    if (!shape || !k || !v || !idx || !counts || !k_out || !v_out) return KVP_ERR_NULL;
    Plan p;
    if (!plan_of(*shape, &p) || shape->hkv > kMaxAdaptiveHeads) return KVP_ERR_SHAPE;
    if (!aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(counts) || !aligned16(k_out) ||
        !aligned16(v_out))
        return KVP_ERR_ALIGN;
    const cudaError_t e =
        launch_compact_ragged(*shape, k, v, idx, counts, k_out, v_out, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_failed(e);
    return KVP_OK;
}

extern "C" kvp_status kvp_compact(const kvp_shape* shape, const uint16_t* k, const uint16_t* v,
                                  const int32_t* idx, uint16_t* k_out, uint16_t* v_out,
                                  void* stream) {
    if (!shape || !k || !v || !idx || !k_out || !v_out) return KVP_ERR_NULL;
    Plan p;
    if (!plan_of(*shape, &p)) return KVP_ERR_SHAPE;
    if (!aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(k_out) ||
        !aligned16(v_out))
        return KVP_ERR_ALIGN;
    const cudaError_t e = launch_compact(*shape, k, v, idx, k_out, v_out, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_failed(e);
    return KVP_OK;
}

extern "C" kvp_status kvp_workspace_status(const void* workspace, void* stream) {
    if (!workspace) return KVP_ERR_NULL;
    if (!aligned16(workspace)) return KVP_ERR_ALIGN;
    return read_error_word(workspace, (cudaStream_t)stream);
}

#ifdef KVP_CHECKS
// Debug builds only: every later scoring call waits for `extra_peers` completions per head
// that never come, and gives up any device wait after `wait_limit_ns` (0: the default).
extern "C" KVP_API void kvp_debug_set_fault(int extra_peers, unsigned long long wait_limit_ns) {
    set_fault(extra_peers, wait_limit_ns);
}

// Debug builds only: copy out (and clear) the first failed device-side bounds check.
extern "C" KVP_API int kvp_debug_take_check_unit(int unit, int* out4) {
    int (*readers[5])(int*) = {take_check_score, take_check_select, take_check_compact,
                               take_check_leverage, take_check_adaptive};
    if (unit < 0 || unit > 4) return -1;
    return readers[unit](out4);
}

extern "C" KVP_API int kvp_debug_take_check(int* out4) {
    int (*readers[5])(int*) = {take_check_score, take_check_select, take_check_compact,
                               take_check_leverage, take_check_adaptive};
    out4[0] = out4[1] = out4[2] = out4[3] = 0;
    for (auto rd : readers) {
        int v[4];
        if (rd(v) != 0) return -1;
        if (v[0] != 0 && out4[0] == 0)
            for (int i = 0; i < 4; ++i) out4[i] = v[i];
    }
    return 0;
}
#endif

#ifdef KVP_TRACE
namespace kvp { int take_trace(unsigned long long* out); }
// Debug builds only: per-CTA %globaltimer stamps of the last scoring launch, [148][8].
extern "C" KVP_API int kvp_debug_trace(unsigned long long* out) { return kvp::take_trace(out); }
#endif

extern "C" const char* kvp_last_cuda_error(void) {
    return t_last_cuda_error == cudaSuccess ? "cudaSuccess" : cudaGetErrorName(t_last_cuda_error);
}

extern "C" const char* kvp_status_string(kvp_status status) {
    switch (status) {
        case KVP_OK: return "KVP_OK";
        case KVP_ERR_NULL: return "KVP_ERR_NULL: a required pointer is NULL";
        case KVP_ERR_SHAPE: return "KVP_ERR_SHAPE: shape outside the supported limits";
        case KVP_ERR_ALIGN: return "KVP_ERR_ALIGN: a pointer is not 16-byte aligned";
        case KVP_ERR_WORKSPACE: return "KVP_ERR_WORKSPACE: workspace missing or too small";
        case KVP_ERR_CUDA: return "KVP_ERR_CUDA: a CUDA call or kernel launch failed";
        case KVP_ERR_TIMEOUT: return "KVP_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "unknown kvp_status";
}
