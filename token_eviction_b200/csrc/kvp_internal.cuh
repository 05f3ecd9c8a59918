// Internal declarations shared by the kvp CUDA translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvp.h"

namespace kvp {

// Largest group of window queries (G * w) one KV head may carry: the score pass keeps
// one fp32 accumulator column per query row in tensor memory (512 columns per SM).
constexpr int kMaxGroupRows = 512;

// How a shape is cut into work: 128-key tiles of the flattened (sequence, KV head, key)
// space dealt out to the scoring kernel's CTAs, and the workspace layout. A pure function
// of the shape, so kvp_workspace_bytes, kvp_score and kvp_select agree.
//   Head-aligned (cph > 0): every KV head is cut into cph parts of consecutive tiles, and
//     each CTA takes nseg parts (segments) of different heads. With two segments a CTA
//     sweeps phase 0 over both heads before phase 1 over either, so the wait for the
//     first head's other CTAs overlaps the second head's phase 0.
//   Flat (cph = 0, nseg = 1): the flattened tiles cut evenly across the CTAs, for shapes
//     with more KV heads than SMs; a run may then cross heads.
struct Plan {
    int G;               // query heads per KV head
    int rows;            // G * w: window queries per KV head
    int tiles_per_head;  // 128-key tiles per (sequence, KV head)
    int total_tiles;     // over all (sequence, KV head)
    int grid;            // CTAs of the scoring kernel (one per SM)
    int cph;             // parts per KV head when head-aligned; 0: flat runs
    int nseg;            // segments per CTA (1 or 2 when head-aligned; 1 when flat)
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

// Flat runs over the T tiles: CTA c takes [floor(c T / grid), floor((c + 1) T / grid)).
__host__ __device__ __forceinline__ long long run_begin(long long c, long long T, long long grid) {
    return c * T / grid;
}
// The CTA whose flat run holds tile t.
__host__ __device__ __forceinline__ int owner_of(long long t, long long T, long long grid) {
    return (int)(((t + 1) * grid + T - 1) / T - 1);
}

// Segment s of CTA c: tiles [b, e). Head-aligned: global part g = s * grid + c, of head
// g / cph, part g % cph, the same cut within every head's tph tiles (grid * nseg =
// cph * heads, so the two segments of a CTA lie in heads grid / cph apart). Flat: the run.
__host__ __device__ __forceinline__ void segment_of(long long c, int s, long long T, long long grid,
                                                    long long tph, long long cph, long long& b,
                                                    long long& e) {
    if (cph > 0) {
        const long long g = s * grid + c, h = g / cph, part = g % cph;
        b = h * tph + part * tph / cph;
        e = h * tph + (part + 1) * tph / cph;
    } else {
        b = run_begin(c, T, grid);
        e = run_begin(c + 1, T, grid);
    }
}
// Slot of CTA c's partial among the CTAs touching head h (reached through segment s).
__host__ __device__ __forceinline__ int slot_in_head(long long c, int s, long long h, long long T,
                                                     long long grid, long long tph, long long cph) {
    if (cph > 0) return (int)((s * grid + c) % cph);
    return (int)(c - owner_of(h * tph, T, grid));
}
// Number of CTAs that touch head h.
__host__ __device__ __forceinline__ int ctas_touching(long long h, long long T, long long grid,
                                                      long long tph, long long cph) {
    if (cph > 0) return (int)cph;
    return owner_of(h * tph + tph - 1, T, grid) - owner_of(h * tph, T, grid) + 1;
}

// The same three in unsigned 32-bit arithmetic, for device code: the plan keeps
// T * (kPlanGrid + 1) below 2^32 and cph <= kPlanGrid, so no product below overflows.
__device__ __forceinline__ void segment_of_u32(uint32_t c, uint32_t s, uint32_t T, uint32_t grid,
                                               uint32_t tph, uint32_t cph, uint32_t& b, uint32_t& e) {
    if (cph > 0) {
        const uint32_t g = s * grid + c, h = g / cph, part = g - h * cph;
        b = h * tph + part * tph / cph;
        e = h * tph + (part + 1) * tph / cph;
    } else {
        b = c * T / grid;
        e = (c + 1) * T / grid;
    }
}
__device__ __forceinline__ uint32_t owner_of_u32(uint32_t t, uint32_t T, uint32_t grid) {
    return ((t + 1) * grid + T - 1) / T - 1;
}
__device__ __forceinline__ uint32_t slot_in_head_u32(uint32_t c, uint32_t s, uint32_t h, uint32_t T,
                                                     uint32_t grid, uint32_t tph, uint32_t cph) {
    if (cph > 0) return (s * grid + c) % cph;
    return c - owner_of_u32(h * tph, T, grid);
}
__device__ __forceinline__ uint32_t ctas_touching_u32(uint32_t h, uint32_t T, uint32_t grid, uint32_t tph,
                                                      uint32_t cph) {
    if (cph > 0) return cph;
    return owner_of_u32(h * tph + tph - 1, T, grid) - owner_of_u32(h * tph, T, grid) + 1;
}

// Tiles by which a head-aligned cut's longest run may exceed the flat cut's and still be
// chosen. A flat run that changes head in mid-stream waits, at the start of its second
// head's scoring pass, for that head's other runs and a fresh query block: on the 32K layer
// (8 heads, 148 SMs) such runs ended about 16 us after the rest.
constexpr int kHeadSwitchTiles = 3;

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_score(const kvp_shape& s, const Plan& p, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, void* workspace, float* score, float* s1, float* s2,
                         cudaStream_t st);
cudaError_t launch_select(const kvp_shape& s, const Plan& p, const float* score, int32_t* idx,
                          void* scratch, cudaStream_t st);
cudaError_t launch_select_policy(const kvp_shape& s, const kvp_policy& pol, const float* s1,
                                 const float* s2, int32_t* idx, cudaStream_t st);
cudaError_t launch_leverage(const kvp_shape& s, const Plan& p, const uint16_t* k, const uint16_t* v,
                            const uint16_t* g, int r, float* score, void* workspace, cudaStream_t st);
// Bytes of the leverage kernel's partial sums with `grid` CTAs (they live in the
// workspace's partial-softmax region) and the slots per KV head.
size_t leverage_part_bytes(const kvp_shape& s, const Plan& p, int grid, int* maxparts);
// Adaptive per-head budgets (kvp_adaptive.cu).
size_t adaptive_workspace_bytes(const kvp_shape& s);
int adaptive_floor(const kvp_shape& s, float alpha);
cudaError_t launch_select_adaptive(const kvp_shape& s, float alpha, const float* score, int32_t* idx,
                                   int32_t* counts, void* workspace, cudaStream_t st);
cudaError_t launch_compact_ragged(const kvp_shape& s, const uint16_t* k, const uint16_t* v,
                                  const int32_t* idx, const int32_t* counts, uint16_t* k_out,
                                  uint16_t* v_out, cudaStream_t st);
cudaError_t launch_compact(const kvp_shape& s, const uint16_t* k, const uint16_t* v,
                           const int32_t* idx, uint16_t* k_out, uint16_t* v_out, cudaStream_t st);

int num_sms();

// A bf16 tensor map of `rank` dimensions (innermost first) with tile box `box`; false if
// the driver's encoder is unavailable or rejects the layout.
bool make_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides_bytes, const cuuint32_t* box, CUtensorMapSwizzle swz);

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
int take_check_leverage(int* out4);
int take_check_adaptive(int* out4);
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
