// Internal declarations shared by the kvp CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvp.h"

namespace kvp {

// Largest group of window queries (G * w) one KV head may carry: the score pass keeps
// one fp32 accumulator column per query row in tensor memory (512 columns per SM).
constexpr int kMaxGroupRows = 512;

// How a shape is cut into work: 128-key tiles of the flattened (sequence, KV head, key)
// space dealt out in contiguous runs to the scoring kernel's CTAs, and the workspace
// layout. A pure function of the shape, so kvp_workspace_bytes, kvp_score and
// kvp_select agree. Runs are either aligned to the KV heads (every head cut into cph
// runs of its own, so no CTA pays for a change of head) or, when that would leave too
// many SMs idle, the flattened tiles cut evenly across all CTAs (cph = 0).
struct Plan {
    int G;               // query heads per KV head
    int rows;            // G * w: window queries per KV head
    int tiles_per_head;  // 128-key tiles per (sequence, KV head)
    int total_tiles;     // over all (sequence, KV head)
    int grid;            // CTAs of the scoring kernel (one per SM, at most one per tile)
    int cph;             // runs per KV head when runs are head-aligned; 0: flat runs
    int maxslots;        // partial-softmax slots per query row (CTAs touching one head)
    size_t off_err;      // int: first device-side error code (0 = none); always offset 0
    size_t off_done;     // uint32 per (sequence, KV head): CTAs done with phase 0
    size_t off_part;     // float2 (max, sum) partials [b*hq*w][maxslots], log2 domain
    size_t off_select;   // selection scratch
    size_t bytes;        // total workspace
};

// CTAs the scoring kernel is planned for (B200: 148 SMs); a device with fewer SMs runs
// fewer, provided the workspace's slot count still covers every head.
constexpr int kPlanGrid = 148;

// Partial-softmax slots a CTA fills per KV head it touches.
constexpr int kSlotsPerCta = 1;

bool plan_of(const kvp_shape& s, Plan* p);

// Runs of the scoring kernel's CTAs over the T tiles (tph per KV head). Flat (cph = 0):
// CTA c takes [floor(c T / grid), floor((c + 1) T / grid)). Head-aligned (cph > 0,
// grid = cph * heads): CTA c takes part c % cph of head c / cph, the same cut within the
// head's tph tiles.
__host__ __device__ __forceinline__ long long run_begin(long long c, long long T, long long grid,
                                                        long long tph, long long cph) {
    if (cph > 0) return (c / cph) * tph + (c % cph) * tph / cph;
    return c * T / grid;
}
// The CTA whose run holds tile t.
__host__ __device__ __forceinline__ int owner_of(long long t, long long T, long long grid,
                                                 long long tph, long long cph) {
    if (cph > 0) return (int)((t / tph) * cph + ((t % tph + 1) * cph + tph - 1) / tph - 1);
    return (int)(((t + 1) * grid + T - 1) / T - 1);
}

// Tiles by which a head-aligned cut's longest run may exceed the flat cut's and still be
// chosen. A run that changes head in mid-stream waits, at the start of its second head's
// scoring pass, for that head's other runs and a fresh query block: on the 32K layer
// (8 heads, 148 SMs) such runs ended about 16 us after the rest, while 15-tile aligned
// runs ended within 3 us of each other.
constexpr int kHeadSwitchTiles = 3;

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_score(const kvp_shape& s, const Plan& p, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, void* workspace, float* score, float* s1, float* s2,
                         cudaStream_t st);
cudaError_t launch_select(const kvp_shape& s, const Plan& p, const float* score, int32_t* idx,
                          void* scratch, cudaStream_t st);
cudaError_t launch_compact(const kvp_shape& s, const uint16_t* k, const uint16_t* v,
                           const int32_t* idx, uint16_t* k_out, uint16_t* v_out, cudaStream_t st);

int num_sms();

// Records `e` as the calling thread's last CUDA error (what kvp_last_cuda_error() names),
// clears the runtime's sticky copy of a launch error, and returns KVP_ERR_CUDA.
kvp_status record_cuda_error(cudaError_t e);

// Reads the error word at the start of a workspace (synchronising `stream`): KVP_OK,
// KVP_ERR_TIMEOUT when a bounded device wait gave up, or KVP_ERR_CUDA.
kvp_status read_error_word(const void* workspace, cudaStream_t stream);

// Lets `func` use up to `bytes` of dynamic shared memory on the current device. The limit
// is per-device state: it is raised once per device and kernel (to the opt-in maximum
// less the kernel's static shared memory), not on every call.
cudaError_t allow_dynamic_smem(const void* func, size_t bytes);

#ifdef KVP_CHECKS
// Debug builds only: the first failed device-side bounds check (code, a, b) is recorded
// here and the access skipped, instead of touching memory out of bounds.
// One copy per translation unit (no relocatable device code); each unit exports a reader.
static __device__ int g_kvp_check[4];
#define KVP_DEFINE_CHECK_READER(fn)                                                        \
    int fn(int* out4) {                                                                    \
        if (cudaMemcpyFromSymbol(out4, g_kvp_check, 4 * sizeof(int)) != cudaSuccess) return -1; \
        const int zero[4] = {0, 0, 0, 0};                                                  \
        return cudaMemcpyToSymbol(g_kvp_check, zero, sizeof(zero)) == cudaSuccess ? 0 : -1; \
    }
int take_check_score(int* out4);
void set_fault(int extra_peers, unsigned long long wait_limit_ns);
int take_check_select(int* out4);
int take_check_compact(int* out4);
static __device__ __noinline__ void kvp_check_fail(int code, int a, int b) {
    if (atomicCAS(&g_kvp_check[0], 0, code) == 0) {
        g_kvp_check[1] = a;
        g_kvp_check[2] = b;
    }
}
#define KVP_CHECK(cond, code, a, b) ((cond) ? true : (kvp_check_fail((code), (a), (b)), false))
#else
#define KVP_CHECK(cond, code, a, b) true
#endif

}  // namespace kvp
