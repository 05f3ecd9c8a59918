// Internal declarations shared by the kvp CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvp.h"

namespace kvp {

// Largest group of window queries (G * w) one KV head may carry: the score pass keeps
// one fp32 accumulator column per query row in tensor memory (512 columns per SM).
constexpr int kMaxGroupRows = 512;

// How a shape is cut into work: the split of L for the log-sum-exp pass and the
// workspace layout. A pure function of the shape, so kvp_workspace_bytes, kvp_score
// and kvp_select agree.
struct Plan {
    int G;             // query heads per KV head
    int rows;          // G * w: window queries per KV head
    int nsplit;        // L-splits of the log-sum-exp pass
    int keys_per_split;
    size_t off_part;   // float2 (max, sum) partials [b*hq*w][nsplit], log2 domain
    size_t off_select; // selection scratch
    size_t bytes;      // total workspace
};

bool plan_of(const kvp_shape& s, Plan* p);

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_lse_partial(const kvp_shape& s, const Plan& p, const uint16_t* q,
                               const uint16_t* k, float2* part, cudaStream_t st);
cudaError_t launch_score(const kvp_shape& s, const Plan& p, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const float2* part, float* score, float* s1,
                         float* s2, cudaStream_t st);
cudaError_t launch_select(const kvp_shape& s, const Plan& p, const float* score, int32_t* idx,
                          void* scratch, cudaStream_t st);
cudaError_t launch_compact(const kvp_shape& s, const uint16_t* k, const uint16_t* v,
                           const int32_t* idx, uint16_t* k_out, uint16_t* v_out, cudaStream_t st);

int num_sms();

}  // namespace kvp
