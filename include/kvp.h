/*
 * kvp.h - prefill KV-cache token eviction on NVIDIA B200 (sm_100a): C ABI.
 *
 * The method ("Preserving Large Activations: The Key to KV Cache Pruning", SlimKV,
 * Section 3) scores every cached position j of every KV head with S = S1 * S2:
 *
 *   S1[j]  (Eq. 3) the softmax attention weight that each of the last w queries of the
 *          prefill (the observation window) gives key j, summed over those queries and
 *          over the G query heads that share the KV head (Section 3.1, grouped-wise
 *          scoring for GQA). The softmax is the attention softmax(q . k / C) with
 *          C = sqrt(d) (the CurDKV rebuttal page's statement of attention). Window query
 *          i sits at position L - w + i and sees keys j <= L - w + i.
 *   S2[j]  (Eq. 4) the largest |V[j, c]| over the head dimension c, so positions that
 *          carry large activations in the value cache survive.
 *   S[j]   (Eq. 5) S1[j] * S2[j].
 *
 * It then keeps B positions per (sequence, KV head) - Listing 1's window_size (w) and
 * max_capacity_prompt (B): the w window positions always, plus the B - w highest-S
 * positions before the window - and compacts K and V to those rows.
 *
 * Conventions for every call:
 *   - All tensors are device memory, contiguous, row-major, innermost dimension last.
 *     bf16 tensors are passed as their 16-bit patterns (uint16_t).
 *   - Query head hq belongs to KV head hq / G, G = hq_count / hkv_count.
 *   - The caller owns and allocates every buffer. No call allocates device memory
 *     (kvp_score_static uses a fixed array that the library defines instead of a
 *     workspace) and no call keeps data for the next; calls with distinct workspaces
 *     may run concurrently from several host threads.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls only enqueue
 *     work and never synchronise the host.
 *   - Argument errors are detected on the host before anything is launched; the outputs
 *     are then untouched. A launch failure returns KVP_ERR_CUDA; kvp_last_cuda_error()
 *     names the CUDA error.
 *   - Every device-side wait is bounded in time, so no kernel can hang. A wait that gives
 *     up records an error code in the workspace and its kernel returns early: the call
 *     has already returned KVP_OK, and its outputs are undefined. kvp_workspace_status()
 *     reads that code back.
 */
#ifndef KVP_H_
#define KVP_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVP_API __attribute__((visibility("default")))
#else
#define KVP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Problem shape. budget (B) counts every kept position, window included. */
typedef struct {
    int32_t batch;     /* b   >= 1 */
    int32_t hq;        /* query heads, a multiple of hkv */
    int32_t hkv;       /* KV heads >= 1 */
    int32_t head_dim;  /* d: 64 or 128 */
    int32_t seq_len;   /* L >= 1 */
    int32_t window;    /* w: 1 <= w <= L, and G * w <= 512 */
    int32_t budget;    /* B: w <= B <= L */
} kvp_shape;

typedef enum {
    KVP_OK = 0,
    KVP_ERR_NULL = 1,      /* a required pointer is NULL */
    KVP_ERR_SHAPE = 2,     /* shape outside the limits above */
    KVP_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned */
    KVP_ERR_WORKSPACE = 4, /* workspace NULL or smaller than kvp_workspace_bytes() */
    KVP_ERR_CUDA = 5,      /* a CUDA runtime/driver call or kernel launch failed */
    KVP_ERR_TIMEOUT = 6    /* a bounded device-side wait gave up (see kvp_workspace_status) */
} kvp_status;

/* Bytes of device workspace that kvp_score and kvp_select need for `shape`
 * (split-L softmax partials, log-sum-exp values, selection scratch); 0 for an invalid
 * shape. The workspace holds no state between calls. */
KVP_API size_t kvp_workspace_bytes(const kvp_shape* shape);

/*
 * Scores S, and optionally S1 and S2, of every position (window included).
 *   q_win  [b, hq, w, d]   bf16: the last w queries of the prefill, Q[:, :, L-w:, :]
 *   k, v   [b, hkv, L, d]  bf16: the layer's key and value cache
 *   score  [b, hkv, L]     fp32 output, S = S1 * S2
 *   s1, s2 [b, hkv, L]     fp32 outputs, may be NULL
 *   workspace  device scratch of at least kvp_workspace_bytes(shape) bytes
 * Arithmetic: bf16 products accumulated in fp32, fp32 exponentials.
 */
KVP_API kvp_status kvp_score(const kvp_shape* shape, const uint16_t* q_win, const uint16_t* k,
                             const uint16_t* v, float* score, float* s1, float* s2,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Kept positions of every (b, KV head): the B - w highest scores among positions
 * [0, L - w) (equal scores: lower position first) and the window [L - w, L), listed in
 * ascending position order.
 *   score [b, hkv, L] fp32, non-negative (as kvp_score writes it)
 *   idx   [b, hkv, B] int32 output
 * B == L gives the identity; B == w keeps the window alone.
 */
KVP_API kvp_status kvp_select(const kvp_shape* shape, const float* score, int32_t* idx,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Selection policies: the variants named around the method. */
typedef enum {
    KVP_RANK_PRODUCT = 0, /* pool(S1) * S2: Eq. 5 of SlimKV (with pooling when kernel > 1) */
    KVP_RANK_S1 = 1,      /* pool(S1) alone: the SlimKV ablation without S2 (review of Sec. 4.6) */
    KVP_RANK_S2 = 2       /* S2 alone: the SlimKV ablation without S1 (same review) */
} kvp_rank_mode;

typedef struct {
    int32_t sinks;        /* s >= 0: positions [0, s) are always kept (attention sinks; CurDKV
                             rebuttal, "how our method processes the KV cache", step 5) */
    int32_t pool_kernel;  /* k, odd, 1 <= k <= 255: S1 is max-pooled over [j - k/2, j + k/2]
                             within [0, L - w) before ranking (the "kernel size" of the SlimKV
                             review of Sec. 4.6, read as SnapKV-style 1-D max pooling); 1: none */
    int32_t mode;         /* a kvp_rank_mode */
} kvp_policy;

/*
 * Kept positions under a policy: the first s positions, the B - w - s candidates of
 * [s, L - w) with the highest keys (equal keys: lower position first), and the window
 * [L - w, L), listed in ascending position order. The key of candidate j is formed in
 * fp32 from S1 and S2 (as kvp_score writes them):
 *   p_j = max of s1 over [j - k/2, j + k/2] within [0, L - w)
 *   mode PRODUCT: p_j * s2_j (rounded to nearest, subnormal operands kept); S1: p_j; S2: s2_j
 *   a key below the smallest normal fp32 counts as zero.
 *   s1, s2  [b, hkv, L] fp32, non-negative; s1 may be NULL in mode S2, s2 in mode S1
 *   idx     [b, hkv, B] int32 output
 * Needs s + w <= B and s <= L - w (else KVP_ERR_SHAPE, as for a bad kernel or mode).
 * No workspace: the call keeps its keys in shared memory.
 */
KVP_API kvp_status kvp_select_policy(const kvp_shape* shape, const kvp_policy* policy,
                                     const float* s1, const float* s2, int32_t* idx, void* stream);

/*
 * CurDKV leverage scores (CurDKV rebuttal page, "A clearer description of Algorithm 1",
 * steps 1-4), an alternative to kvp_score for the same selection and compaction:
 *   lk_j = ||K_j G||^2, lv_j = ||V_j G||^2   (squared row norms of the projected key and
 *                                             value of position j)
 *   score_j = lk_j * lv_j / sum over the KV head's L positions of lk * lv   (0 if that is 0)
 *   k, v   [b, hkv, L, d] bf16
 *   g      [d, r] bf16: the Gaussian projection, drawn by the caller; 1 <= r <= 32
 *   score  [b, hkv, L] fp32 output (sums to 1 per (b, KV head))
 *   workspace  as for kvp_score (kvp_workspace_bytes); its error word is cleared and set
 *              as by kvp_score (kvp_workspace_status reads it)
 * Arithmetic: bf16 products accumulated in fp32 on the tensor cores, fp32 squares, sums
 * and product; the normalising sum is taken in a fixed order (repeat calls agree bit for
 * bit). Rank with kvp_select_policy in KVP_RANK_S1 mode (score as s1), with CurDKV's sinks.
 */
KVP_API kvp_status kvp_leverage(const kvp_shape* shape, const uint16_t* k, const uint16_t* v,
                                const uint16_t* g, int32_t r, float* score, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * Adaptive per-head budgets: the AdaKV scheme with its safeguard alpha, as the CurDKV
 * rebuttal page describes it ("On the sensitivity of the safeguard parameter (alpha)",
 * Tables 5-6; the AdaKV default alpha is 0.20). The KV heads of a sequence share its
 * budget hkv * B. Every head keeps its window [L - w, L) and its best
 * f = floor(alpha * (B - w)) candidates of [0, L - w) (score descending, then position);
 * the other hkv * (B - w - f) positions go to the best of all the heads' remaining
 * candidates (score descending, then head, then position). alpha = 1 is kvp_select's
 * uniform budget; alpha = 0 one shared top-k.
 *   score   [b, hkv, L] fp32, non-negative (kvp_score's S, or kvp_leverage's)
 *   idx     [b, hkv * B] int32 output: head 0's kept positions ascending, then head 1's, ...
 *   counts  [b, hkv] int32 output: kept positions of each head (window included); they sum
 *           to hkv * B per sequence
 *   workspace  at least kvp_adaptive_workspace_bytes(shape) bytes (0 for a bad shape)
 * Needs 0 <= alpha <= 1 and hkv <= 4096 (else KVP_ERR_SHAPE).
 */
KVP_API size_t kvp_adaptive_workspace_bytes(const kvp_shape* shape);
KVP_API kvp_status kvp_select_adaptive(const kvp_shape* shape, float alpha, const float* score,
                                       int32_t* idx, int32_t* counts, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * Compaction of a ragged selection (kvp_select_adaptive's layout): row r of sequence b's
 * output belongs to the head h whose rows [sum of counts[b, :h], + counts[b, h]) hold it,
 * and k_out[b, r, :] = k[b, h, idx[b, r], :]; the same for v; a bit copy.
 *   idx     [b, hkv * B] int32;  counts [b, hkv] int32 (summing to hkv * B)
 *   k_out, v_out  [b, hkv * B, d] bf16 outputs; an index outside [0, L) yields a zero row
 */
KVP_API kvp_status kvp_compact_ragged(const kvp_shape* shape, const uint16_t* k, const uint16_t* v,
                                      const int32_t* idx, const int32_t* counts, uint16_t* k_out,
                                      uint16_t* v_out, void* stream);

/*
 * Compaction: k_out[b, h, t, :] = k[b, h, idx[b, h, t], :], the same for v; a bit copy.
 *   k, v          [b, hkv, L, d] bf16
 *   idx           [b, hkv, B]    int32, entries in [0, L) (an entry outside that range
 *                                yields a zero row instead of an out-of-bounds read)
 *   k_out, v_out  [b, hkv, B, d] bf16 outputs; must not overlap k or v
 */
KVP_API kvp_status kvp_compact(const kvp_shape* shape, const uint16_t* k, const uint16_t* v,
                               const int32_t* idx, uint16_t* k_out, uint16_t* v_out, void* stream);

/*
 * Device-side status of the last kvp_score call that used `workspace`: KVP_ERR_TIMEOUT if
 * one of its bounded waits gave up (the call's score, s1 and s2 are then undefined, and so
 * is whatever kvp_select and kvp_compact made from them), KVP_OK otherwise. The code sits in
 * the workspace's first 4 bytes; kvp_score clears it when it starts.
 *   workspace  the device workspace passed to kvp_score (16-byte aligned)
 *   stream     the stream kvp_score ran on
 * This call synchronises `stream` (it copies the 4 bytes to the host), so it cannot be
 * made during stream capture: it then returns KVP_ERR_CUDA. NULL workspace: KVP_ERR_NULL.
 */
KVP_API kvp_status kvp_workspace_status(const void* workspace, void* stream);

/*
 * kvp_score without a workspace, for callers that cannot allocate device memory at the
 * time they evict: a serving engine that reserved the device for its own memory pool at
 * start-up, code that may not allocate after initialisation, or a runtime that only
 * passes in tensors it already owns. (The eviction method has no counterpart to this
 * call; it is a deployment convenience.)
 *
 * Inputs, outputs and results are those of kvp_score. The scratch is a fixed array of
 * KVP_STATIC_SCRATCH_BYTES bytes of device memory defined inside the library; every GPU
 * that loads the library holds it until the process exits. A shape whose
 * kvp_workspace_bytes() exceeds KVP_STATIC_SCRATCH_BYTES is rejected with
 * KVP_ERR_WORKSPACE before anything is launched.
 *   - Every call looks up the array's device address with cudaGetSymbolAddress, which
 *     allocates nothing; the first lookup on a device may load the library's device code
 *     there, so make the first call on each device before any stream capture.
 *   - All calls share the one array: calls that may overlap on the GPU (other streams,
 *     other host threads, concurrent graphs) race and must be serialised by the caller.
 *     Each call clears the parts of the array that must start at zero.
 *   - The call allocates nothing (no cudaMalloc, no allocating library routine).
 */
#define KVP_STATIC_SCRATCH_BYTES ((size_t)2 << 20)

KVP_API kvp_status kvp_score_static(const kvp_shape* shape, const uint16_t* q_win,
                                    const uint16_t* k, const uint16_t* v, float* score,
                                    float* s1, float* s2, void* stream);

/* kvp_workspace_status for kvp_score_static: the device-side status of the last call on
 * this device, read from the library's scratch array (synchronises `stream`). */
KVP_API kvp_status kvp_score_static_status(void* stream);

/* The name of the CUDA error behind the calling thread's most recent KVP_ERR_CUDA
 * ("cudaSuccess" if there was none). Host-only; never fails. */
KVP_API const char* kvp_last_cuda_error(void);

/* A static, human-readable name of a status code. */
KVP_API const char* kvp_status_string(kvp_status status);

#ifdef __cplusplus
}
#endif

#endif /* KVP_H_ */
