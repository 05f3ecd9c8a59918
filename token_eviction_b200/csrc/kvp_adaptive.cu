// Adaptive per-head budgets (AdaKV with a safeguard floor) and the ragged compaction.
//
// CurDKV rebuttal page (paperhub.cn/paper/klmc4fwPLd), "On the sensitivity of the
// safeguard parameter (alpha)", Tables 5-6: the KV heads of a layer share its budget,
// and alpha is the share every head keeps for itself. Readings (the page gives no
// formula): per sequence, each KV head keeps its w window positions and its best
// f = floor(alpha (B - w)) candidates (score descending, position ascending); the other
// hkv (B - w - f) positions go to the best of all the heads' remaining candidates (score
// descending, then head, then position). The sequence keeps hkv B positions in all.
//
// On the GPU, in four steps on one stream:
//   1. every head's floor: the cluster radix select with budget f + w;
//   2. a copy of the scores with the window and the floors set to -inf;
//   3. one cluster radix select per sequence over its heads' rows taken as one row of
//      hkv L keys (no window): the R = hkv (B - w - f) best, in flat order (head, then
//      position), which is also the tie order;
//   4. per head, the floor and its share of the picks merged in position order, then the
//      window, written at the head's offset (the sum of the lower heads' counts).
// kvp_compact_ragged then gathers the kept rows of K and V in the same packed layout.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "kvp_internal.cuh"

namespace kvp {

cudaError_t launch_select_rows(int rows, int L, int w, int B, const float* score, int32_t* idx,
                               cudaStream_t st);

namespace {

// First index in a[0, n) (ascending) whose value is >= x.
__device__ __forceinline__ long long lower_bound(const int32_t* a, long long n, int x) {
    long long lo = 0, hi = n;
    while (lo < hi) {
        const long long mid = (lo + hi) >> 1;
        if (a[mid] < x) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// masked[row][j] = score[row][j] before the window, -inf in it. Grid-stride over floats.
__global__ void __launch_bounds__(256)
mask_window(const float* __restrict__ score, float* __restrict__ masked, long long total, int L, int n) {
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < total; i += (long long)gridDim.x * 256) {
        const int j = (int)(i % L);
        masked[i] = j < n ? score[i] : -INFINITY;
    }
}

// masked[row][floor_idx[row][t]] = -inf for the row's f floor positions.
__global__ void __launch_bounds__(256)
mask_floors(float* __restrict__ masked, const int32_t* __restrict__ floor_idx, int rows, int L, int f,
            int fw) {
    const long long total = (long long)rows * f;
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < total; i += (long long)gridDim.x * 256) {
        const int row = (int)(i / f), t = (int)(i % f);
        const int j = floor_idx[(size_t)row * fw + t];
        if (KVP_CHECK(j >= 0 && j < L, 401, row, j)) masked[(size_t)row * L + j] = -INFINITY;
    }
}

// Block (h, b): head h of sequence b. picks: the sequence's R flat indices (h L + j),
// ascending.
__global__ void __launch_bounds__(256)
merge_heads(const int32_t* __restrict__ floor_idx, const int32_t* __restrict__ picks, int hkv, int L,
            int w, int f, long long R, int B, int32_t* __restrict__ idx, int32_t* __restrict__ counts) {
    __shared__ long long sh_lo, sh_x, sh_off;
    const int h = blockIdx.x, b = blockIdx.y, fw = f + w, n = L - w;
    const int32_t* pk = picks + (size_t)b * R;
    if (threadIdx.x == 0) {
        long long off = 0, lo = 0, x = 0;
        for (int g = 0; g <= h; ++g) {
            const long long a = lower_bound(pk, R, g * L), e = lower_bound(pk, R, (g + 1) * L);
            if (g < h) off += f + (e - a) + w;
            else {
                lo = a;
                x = e - a;
            }
        }
        sh_lo = lo;
        sh_x = x;
        sh_off = off;
        counts[(size_t)b * hkv + h] = (int32_t)(f + x + w);
    }
    __syncthreads();
    const long long lo = sh_lo, x = sh_x;
    const int32_t* F = floor_idx + ((size_t)b * hkv + h) * fw;   // f floor positions, ascending
    const int32_t* P = pk + lo;                                  // x flat indices of head h
    int32_t* out = idx + (size_t)b * hkv * B + sh_off;
    const int base = h * L;
    // the two lists hold distinct positions: each element's place is its index in its own
    // list plus the number of the other list's elements below it
    for (int t = threadIdx.x; t < f; t += 256) {
        const int p = F[t];
        long long a = 0, e = x;                                  // picks of this head below p
        while (a < e) {
            const long long mid = (a + e) >> 1;
            if (P[mid] - base < p) a = mid + 1;
            else e = mid;
        }
        out[t + a] = p;
    }
    for (long long t = threadIdx.x; t < x; t += 256) {
        const int q = P[t] - base;
        out[t + lower_bound(F, f, q)] = q;
    }
    for (int t = threadIdx.x; t < w; t += 256) out[f + x + t] = n + t;
}

// k_out[b][r] = k[b][h][idx[b][r]] for the rows r of head h (offsets from counts); the
// same for v. 16-byte pieces; an index outside [0, L) yields a zero row.
__global__ void __launch_bounds__(256)
gather_ragged(const uint4* __restrict__ k, const uint4* __restrict__ v, const int32_t* __restrict__ idx,
              const int32_t* __restrict__ counts, uint4* __restrict__ k_out, uint4* __restrict__ v_out,
              int hkv, int L, int B, int pieces) {
    extern __shared__ int32_t offs[];                     // [hkv + 1] row offsets of the heads
    constexpr int kPer = 4;                               // 16-byte pieces of K (and of V) per item
    asm volatile("griddepcontrol.wait;" ::: "memory");    // the indices' producer has completed
    const int b = blockIdx.y;
    if (threadIdx.x == 0) {
        int o = 0;
        for (int h = 0; h < hkv; ++h) {
            offs[h] = o;
            o += counts[(size_t)b * hkv + h];
        }
        offs[hkv] = o;
    }
    __syncthreads();
    const long long rows = min((long long)offs[hkv], (long long)hkv * B);   // hkv B when consistent
    const long long total = rows * pieces;                // output pieces of this sequence
    const int lane = threadIdx.x & 31;
    const int ps = __ffs(pieces) - 1;                     // pieces per row: a power of two
    const long long nwarps = (long long)gridDim.x * 8;
    // each warp a block of 32 kPer consecutive pieces; lane l takes l, l + 32, l + 64, l + 96
    for (long long w = blockIdx.x * 8ll + (threadIdx.x >> 5); w * 32 * kPer < total; w += nwarps) {
        long long e[kPer];
        int j[kPer], h[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            e[q] = w * 32 * kPer + q * 32 + lane;
            const long long r = e[q] >> ps;
            int lo = 0, hi = hkv - 1;                     // the head whose rows hold r
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (offs[mid] <= r) lo = mid;
                else hi = mid - 1;
            }
            h[q] = lo;
            j[q] = e[q] < total ? __ldg(idx + (size_t)b * hkv * B + r) : -1;
        }
        uint4 ka[kPer], va[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            if (e[q] < total && j[q] >= 0 && j[q] < L) {
                const size_t src = ((((size_t)b * hkv + h[q]) * L + j[q]) << ps) + (e[q] & (pieces - 1));
                ka[q] = __ldg(k + src);
                va[q] = __ldg(v + src);
            } else {
                ka[q] = va[q] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            if (e[q] >= total) continue;
            const size_t dst = (size_t)b * hkv * B * pieces + e[q];
            __stcs(k_out + dst, ka[q]);
            __stcs(v_out + dst, va[q]);
        }
    }
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t adaptive_workspace_bytes(const kvp_shape& s) {
    const size_t rows = (size_t)s.batch * s.hkv;
    return align256(rows * s.budget * 4) + align256(rows * s.seq_len * 4) + align256(rows * s.budget * 4);
}

int adaptive_floor(const kvp_shape& s, float alpha) {
    return (int)std::floor((double)alpha * (double)(s.budget - s.window));
}

cudaError_t launch_select_adaptive(const kvp_shape& s, float alpha, const float* score, int32_t* idx,
                                   int32_t* counts, void* workspace, cudaStream_t st) {
    const int rows = s.batch * s.hkv, L = s.seq_len, w = s.window, B = s.budget, n = L - w;
    const int f = adaptive_floor(s, alpha), fw = f + w;
    const long long R = (long long)s.hkv * (B - w - f);
    char* ws = (char*)workspace;
    int32_t* floor_idx = (int32_t*)ws;                                  // [rows][f + w]
    float* masked = (float*)(ws + align256((size_t)rows * B * 4));      // [rows][L]
    int32_t* picks = (int32_t*)(ws + align256((size_t)rows * B * 4) + align256((size_t)rows * L * 4));
    cudaError_t e;
    // 1. the floors
    if ((e = launch_select_rows(rows, L, w, fw, score, floor_idx, st)) != cudaSuccess) return e;
    // 2. the masked copy
    const int sms = std::max(1, num_sms());
    {
        const long long total = (long long)rows * L;
        const int grid = (int)std::max<long long>(1, std::min<long long>((total + 255) / 256, sms * 8ll));
        mask_window<<<grid, 256, 0, st>>>(score, masked, total, L, n);
        if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    }
    if (f > 0) {
        const long long total = (long long)rows * f;
        const int grid = (int)std::max<long long>(1, std::min<long long>((total + 255) / 256, sms * 8ll));
        mask_floors<<<grid, 256, 0, st>>>(masked, floor_idx, rows, L, f, fw);
        if ((e = cudaPeekAtLastError()) != cudaSuccess) return e;
    }
    // 3. the shared positions: each sequence's heads as one row of hkv L keys
    if (R > 0 && (e = launch_select_rows(s.batch, s.hkv * L, 0, (int)R, masked, picks, st)) != cudaSuccess)
        return e;
    // 4. per head: floor and picks in position order, then the window
    merge_heads<<<dim3(s.hkv, s.batch), 256, 0, st>>>(floor_idx, picks, s.hkv, L, w, f, R, B, idx, counts);
    return cudaPeekAtLastError();
}

cudaError_t launch_compact_ragged(const kvp_shape& s, const uint16_t* k, const uint16_t* v,
                                  const int32_t* idx, const int32_t* counts, uint16_t* k_out,
                                  uint16_t* v_out, cudaStream_t st) {
    const int pieces = s.head_dim * 2 / 16;
    const long long items = (long long)s.hkv * s.budget * pieces;
    const int sms = std::max(1, num_sms());
    // four 16-byte pieces per thread and per row: whole waves over the SMs, at most 8 CTAs each
    const long long want = (items / 4 + 255) / 256;
    const long long per_b = std::max(1, sms * 8 / s.batch);
    const int gx = (int)std::max<long long>(1, std::min<long long>(want, per_b));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gx, (unsigned)s.batch);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = (s.hkv + 1) * sizeof(int32_t);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlaps the launch
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gather_ragged, (const uint4*)k, (const uint4*)v, idx, counts,
                              (uint4*)k_out, (uint4*)v_out, s.hkv, s.seq_len, s.budget, pieces);
}

#ifdef KVP_CHECKS
KVP_DEFINE_CHECK_READER(take_check_adaptive)
#endif

}  // namespace kvp
