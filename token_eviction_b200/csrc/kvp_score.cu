// S1 * S2 scoring: split-L log-sum-exp pass and the scoring pass.
//
// "Preserving Large Activations: The Key to KV Cache Pruning" (SlimKV), Section 3,
// Eq. 3-5: S1[j] = sum over the GQA group's query heads and the window queries of
// softmax_j(q . k_j / sqrt(d)), S2[j] = max_c |V[j, c]|, S[j] = S1[j] * S2[j].
//
// The softmax needs each window query's log-sum-exp over all visible keys before any
// column (key) sum can be formed, so the work is two passes over K:
//   pass 1: every (L-split, KV head) CTA produces, per window query, the running max m
//           and sum l of exp2(t - m) over its keys (t = logit * log2(e), log2 domain);
//   pass 2: every (key tile, KV head) CTA merges the splits into lse2 per query, then
//           recomputes the logits of its keys, sums exp2(t - lse2) over the group's
//           window queries (causal: query i sees key j <= L - w + i), reads V once
//           for max |V| and writes S, S1, S2.
// This translation unit is the straightforward CUDA-core version of both passes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cmath>

#include "kvp_internal.cuh"

namespace kvp {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kKeyChunk = 32;

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float((uint32_t)b << 16);
}

// grid (nsplit, b*hkv, ceil(rows/128)), block 128: thread = one window query row.
template <int D>
__global__ void __launch_bounds__(128) lse_partial_simple(const uint16_t* __restrict__ q,
                                                          const uint16_t* __restrict__ k,
                                                          float2* __restrict__ part, int hq,
                                                          int hkv, int L, int w, int nsplit,
                                                          int keys_per_split) {
    __shared__ float ks[kKeyChunk][D];
    const int split = blockIdx.x, bh = blockIdx.y;
    const int b = bh / hkv, h = bh % hkv;
    const int G = hq / hkv, rows = G * w;
    const int r = blockIdx.z * 128 + threadIdx.x;
    const bool active = r < rows;
    const int i = active ? r % w : 0;
    const int p = L - w + i;  // last key this query sees
    const size_t row0 = ((size_t)b * hq + (size_t)h * G) * w;  // first query row of the group
    float qr[D];
#pragma unroll
    for (int c = 0; c < D; ++c) qr[c] = active ? bf16_bits_to_float(q[(row0 + r) * D + c]) : 0.f;
    const float scale = kLog2e * rsqrtf((float)D);
    const int j0 = split * keys_per_split;
    const int j1 = min(L, j0 + keys_per_split);
    const uint16_t* kh = k + (size_t)bh * L * D;
    float m = -INFINITY, l = 0.f;
    for (int jb = j0; jb < j1; jb += kKeyChunk) {
        __syncthreads();
        for (int e = threadIdx.x; e < kKeyChunk * D; e += 128) {
            const int jj = jb + e / D;
            ks[e / D][e % D] = jj < j1 ? bf16_bits_to_float(kh[(size_t)jj * D + e % D]) : 0.f;
        }
        __syncthreads();
        if (!active) continue;
        float t[kKeyChunk];
        float cm = -INFINITY;
#pragma unroll
        for (int kk = 0; kk < kKeyChunk; ++kk) {
            float dot = 0.f;
#pragma unroll
            for (int c = 0; c < D; ++c) dot = fmaf(qr[c], ks[kk][c], dot);
            const int jj = jb + kk;
            t[kk] = (jj < j1 && jj <= p) ? dot * scale : -INFINITY;
            cm = fmaxf(cm, t[kk]);
        }
        if (cm == -INFINITY) continue;
        const float mn = fmaxf(m, cm);
        float acc = l * exp2f(m - mn);
#pragma unroll
        for (int kk = 0; kk < kKeyChunk; ++kk) acc += exp2f(t[kk] - mn);
        l = acc;
        m = mn;
    }
    if (active) part[(row0 + r) * nsplit + split] = make_float2(m, l);
}

// grid (ceil(L/128), b*hkv), block 128: thread = one key position.
// dynamic smem: lse2[rows] floats, then the group's query rows as bf16 [rows][D].
template <int D>
__global__ void __launch_bounds__(128) score_simple(const uint16_t* __restrict__ q,
                                                    const uint16_t* __restrict__ k,
                                                    const uint16_t* __restrict__ v,
                                                    const float2* __restrict__ part,
                                                    float* __restrict__ score,
                                                    float* __restrict__ s1_out,
                                                    float* __restrict__ s2_out, int hq, int hkv,
                                                    int L, int w, int nsplit) {
    extern __shared__ float smem[];
    const int bh = blockIdx.y;
    const int b = bh / hkv, h = bh % hkv;
    const int G = hq / hkv, rows = G * w;
    float* lse2 = smem;
    uint16_t* qs = (uint16_t*)(smem + ((rows + 3) & ~3));
    const size_t row0 = ((size_t)b * hq + (size_t)h * G) * w;
    // cross-split merge: lse2 = M + log2(sum_s l_s * 2^(m_s - M)), M = max_s m_s
    for (int r = threadIdx.x; r < rows; r += blockDim.x) {
        const float2* pr = part + (row0 + r) * nsplit;
        float M = -INFINITY;
        for (int s = 0; s < nsplit; ++s) M = fmaxf(M, pr[s].x);
        float sum = 0.f;
        for (int s = 0; s < nsplit; ++s)
            if (pr[s].x != -INFINITY) sum += pr[s].y * exp2f(pr[s].x - M);
        lse2[r] = M + log2f(sum);
    }
    for (int e = threadIdx.x; e < rows * D; e += blockDim.x) qs[e] = q[row0 * D + e];
    __syncthreads();
    const int j = blockIdx.x * 128 + threadIdx.x;
    if (j >= L) return;
    const size_t krow = ((size_t)bh * L + j) * D;
    float kr[D];
#pragma unroll
    for (int c = 0; c < D; ++c) kr[c] = bf16_bits_to_float(k[krow + c]);
    const float scale = kLog2e * rsqrtf((float)D);
    float acc = 0.f;
    for (int r = 0; r < rows; ++r) {
        const int i = r % w;
        if (j > L - w + i) continue;  // causal mask inside the window
        const uint16_t* qr = qs + (size_t)r * D;
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) dot = fmaf(bf16_bits_to_float(qr[c]), kr[c], dot);
        acc += exp2f(dot * scale - lse2[r]);
    }
    float vmax = 0.f;
#pragma unroll
    for (int c = 0; c < D; ++c) vmax = fmaxf(vmax, fabsf(bf16_bits_to_float(v[krow + c])));
    const size_t o = (size_t)bh * L + j;
    score[o] = acc * vmax;
    if (s1_out) s1_out[o] = acc;
    if (s2_out) s2_out[o] = vmax;
}

}  // namespace

cudaError_t launch_lse_partial(const kvp_shape& s, const Plan& p, const uint16_t* q,
                               const uint16_t* k, float2* part, cudaStream_t st) {
    dim3 grid(p.nsplit, s.batch * s.hkv, (p.rows + 127) / 128);
    if (s.head_dim == 128)
        lse_partial_simple<128><<<grid, 128, 0, st>>>(q, k, part, s.hq, s.hkv, s.seq_len,
                                                      s.window, p.nsplit, p.keys_per_split);
    else
        lse_partial_simple<64><<<grid, 128, 0, st>>>(q, k, part, s.hq, s.hkv, s.seq_len,
                                                     s.window, p.nsplit, p.keys_per_split);
    return cudaGetLastError();
}

cudaError_t launch_score(const kvp_shape& s, const Plan& p, const uint16_t* q, const uint16_t* k,
                         const uint16_t* v, const float2* part, float* score, float* s1,
                         float* s2, cudaStream_t st) {
    dim3 grid((s.seq_len + 127) / 128, s.batch * s.hkv);
    const size_t smem = (size_t)((p.rows + 3) & ~3) * 4 + (size_t)p.rows * s.head_dim * 2;
    cudaError_t e;
    if (s.head_dim == 128) {
        e = cudaFuncSetAttribute(score_simple<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        score_simple<128><<<grid, 128, smem, st>>>(q, k, v, part, score, s1, s2, s.hq, s.hkv,
                                                  s.seq_len, s.window, p.nsplit);
    } else {
        e = cudaFuncSetAttribute(score_simple<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        score_simple<64><<<grid, 128, smem, st>>>(q, k, v, part, score, s1, s2, s.hq, s.hkv,
                                                 s.seq_len, s.window, p.nsplit);
    }
    return cudaGetLastError();
}

}  // namespace kvp
