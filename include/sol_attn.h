/*
 * sol_attn.h — C ABI of the Sol-Attn single-pass sparse attention forward for
 * NVIDIA B200 (sm_100a).
 *
 * Method: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
 * Attention Sparsification".  For every query block i of 64 tokens the forward
 *   1. mean-pools 64-token blocks into Q̄_i, K̄_j and sums values into V̂_j
 *      (method: threshold routing, Eq. 3; proxy-score reuse, V̂ before Eq. 9);
 *   2. derives τ_i = μ_i + β σ_i from the first and second moments of the
 *      pooled keys, never forming the N x N proxy map (Eq. 4-5);
 *   3. in one online-softmax pass scans the pooled keys in chunks of C, selects
 *      block j when ŝ_ij = Q̄_i·K̄_j/sqrt(d) >= τ_i (Eq. 6-7), runs exact
 *      attention over the selected K/V blocks, and adds the zeroth-order
 *      approximation exp(q_r·K̄_j/sqrt(d)) for every unselected block, weighted
 *      by its token count n_j in the denominator and applied to V̂_j in the
 *      numerator (Eq. 8-10, batched as the token-to-block tile of Eq. 11).
 *
 * Conventions shared by every entry point:
 *   - Tensors q, k, v, out are contiguous row-major [B, H, L, d] bf16 (raw
 *     16-bit patterns), device memory unless stated otherwise, each base
 *     address 16-byte aligned.  out must not overlap q, k or v.
 *   - block must be 64 (fixed 64x64 physical blocks, experiments: setup);
 *     d must be 64 or 128; N = ceil(L / 64); the last block may be ragged and
 *     is pooled over its valid tokens.  1 <= L <= 1,048,576, chunk >= 1,
 *     1 <= B*H <= 65535.
 *   - beta: any finite value; -INFINITY selects every block (dense mode),
 *     +INFINITY selects none (every block approximated); NaN is rejected.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued without a host synchronisation unless a flag asks for
 *     one; errors detected while enqueuing are returned immediately.
 *   - The library owns a per-device workspace (pooled tensors, thresholds,
 *     per-row counts, a work counter and a status word) that grows on demand
 *     with cudaMalloc; the first call for a larger shape therefore must not be
 *     inside a stream capture.  Calls on one device share the workspace: do
 *     not run two forwards concurrently on different streams of one device.
 *   - Return value: SOL_ATTN_OK (0) or a negative sol_attn_status code.
 *     sol_attn_error_string() describes the last error in words.
 */
#ifndef SOL_ATTN_H_
#define SOL_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sol_attn_status {
  SOL_ATTN_OK = 0,
  SOL_ATTN_ERR_ARG = -1,          /* null pointer, non-positive size, NaN beta, chunk < 1,
                                     unknown or conflicting flags */
  SOL_ATTN_ERR_UNSUPPORTED = -2,  /* d not in {64,128}, block != 64, L too large, B*H > 65535,
                                     not sm_100 */
  SOL_ATTN_ERR_ALIGN = -3,        /* a tensor base address is not 16-byte aligned */
  SOL_ATTN_ERR_CUDA = -4,         /* a CUDA runtime call or kernel launch failed */
  SOL_ATTN_ERR_TIMEOUT = -5,      /* a bounded device-side wait gave up (status word) */
  SOL_ATTN_ERR_STATE = -6,        /* stats/stage call without a matching earlier forward */
  SOL_ATTN_ERR_DEVICE = -7        /* a device-side consistency check failed (status word):
                                     the fused kernel range-checks every tile descriptor
                                     (head, query pair, key blocks) before its copies and
                                     stops instead of issuing an out-of-range one */
} sol_attn_status;

/* Flags for sol_attn_forward_ex. */
#define SOL_ATTN_FLAG_SELECT_ALL 0x1u  /* ignore beta; select every block (dense baseline) */
#define SOL_ATTN_FLAG_EXACT_ONLY 0x2u  /* keep-or-drop: skip the approximation of unselected
                                          blocks (ablation: exact-only vs exact-or-approx) */
#define SOL_ATTN_FLAG_SYNC_CHECK 0x4u  /* synchronise the stream after the forward and read
                                          the device status word (timeouts, device checks) */
#define SOL_ATTN_FLAG_TEST_STALL 0x8u  /* test of the failure path only: the fused kernel's
                                          routing step publishes no work, every bounded wait
                                          gives up after 1 ms, the kernel exits cleanly and
                                          the status word reports SOL_ATTN_ERR_TIMEOUT; out
                                          is left unwritten */
#define SOL_ATTN_FLAG_FIRST_ORDER 0x10u /* extension (the method keeps the zeroth order only):
                                          every block goes through the exact tile path and a
                                          block the row did not select gets the first-order
                                          expansion of Eq. 8 around its row-wise mean score
                                          c = q.K̄_j/sqrt(d), weight e^c (1 + (s - c)) per key,
                                          instead of the zeroth-order e^c; costs as much as
                                          the select-all mode.  Excludes EXACT_ONLY. */

/* Optional device buffers filled by sol_attn_forward_ex (any member may be NULL).
 * Shapes use N = ceil(L/64); all are row-major and owned by the caller. */
typedef struct sol_attn_debug {
  float* qbar;     /* [B,H,N,d] pooled queries Q̄ (mean over valid tokens), fp32 */
  float* kbar;     /* [B,H,N,d] pooled keys K̄, fp32 */
  float* vhat;     /* [B,H,N,d] summed values V̂ (sum over valid tokens), fp32 */
  float* mu;       /* [B,H,N] proxy-row mean μ_i from the key moments */
  float* sigma;    /* [B,H,N] proxy-row standard deviation σ_i from the key moments */
  float* tau;      /* [B,H,N] threshold τ_i (±inf in select-all / select-none) */
  uint32_t* mask;  /* [B,H,N,ceil(N/32)] selection bits: block j of row i is bit (j%32)
                      of word j/32; written by the fused kernel's routing step */
} sol_attn_debug;

/* Sol-Attn forward (method: Eq. 3-11).  q, k, v: input [B,H,L,d] bf16 device
 * tensors; out: output [B,H,L,d] bf16 device tensor, every valid row written.
 * chunk: C, the number of pooled keys routed per outer-loop step (Eq. 6); it
 * changes the schedule, not the result.  Enqueues a memset of the work counter
 * and four kernels (pool, moments, thresholds, fused attention) on stream. */
int sol_attn_forward(const void* q, const void* k, const void* v, void* out,
                     int B, int H, int L, int d, int block, int chunk, float beta,
                     void* stream);

/* As sol_attn_forward, with SOL_ATTN_FLAG_* flags and optional debug exports
 * (dbg may be NULL). */
int sol_attn_forward_ex(const void* q, const void* k, const void* v, void* out,
                        int B, int H, int L, int d, int block, int chunk, float beta,
                        unsigned flags, const sol_attn_debug* dbg, void* stream);

/* Per-row selected-block counts |S_i| (density analysis, ablation: Fig. 7):
 * copies the [B,H,N] int32 counts written by the last forward on this device
 * into counts (device memory), enqueued on stream.  Returns SOL_ATTN_ERR_STATE
 * if the last forward had a different (B,H,L,block). */
int sol_attn_stats(int32_t* counts, int B, int H, int L, int block, void* stream);

/* End-to-end call on HOST buffers (pinned or pageable; pinned lets the copies
 * overlap): the B*H independent (batch, head) slices go through in up to 16
 * groups; for each group q, k, v are copied to the device, sol_attn_forward_ex
 * runs on the group and out is copied back, on three internal streams so that
 * the copies of neighbouring groups overlap the kernels.  Synchronises before
 * returning.  Device staging buffers (two groups) are owned and cached by the
 * library.  sol_attn_stats afterwards refers to the last group only. */
int sol_attn_forward_host(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          uint16_t* out, int B, int H, int L, int d, int block,
                          int chunk, float beta, unsigned flags);

/* The three stages of sol_attn_forward_ex as separate calls on one stream, for
 * per-kernel timing and staged checks.  They must be called in this order with
 * the same shape; a later stage returns SOL_ATTN_ERR_STATE otherwise.
 *   stage_pool:      block pooling of q, k, v into the workspace (method: Eq. 3, V̂).
 *   stage_threshold: key moments and τ_i = μ_i + β σ_i (Eq. 4-5).
 *   stage_fused:     routing, exact inner loop and approximation (Eq. 6-11). */
int sol_attn_stage_pool(const void* q, const void* k, const void* v, int B, int H, int L,
                        int d, int block, const sol_attn_debug* dbg, void* stream);
int sol_attn_stage_threshold(int B, int H, int L, int d, int block, float beta,
                             unsigned flags, const sol_attn_debug* dbg, void* stream);
int sol_attn_stage_fused(const void* q, const void* k, const void* v, void* out, int B,
                         int H, int L, int d, int block, int chunk, unsigned flags,
                         const sol_attn_debug* dbg, void* stream);

/* Bytes of device workspace the library holds for this shape. */
size_t sol_attn_workspace_bytes(int B, int H, int L, int d, int block);

/* Frees the calling thread's current-device workspace (no work may be in flight). */
int sol_attn_release(void);

/* Text for a status code, including detail of the most recent failure. */
const char* sol_attn_error_string(int code);

/* Number of kernels one sol_attn_forward enqueues (for launch accounting). */
int sol_attn_kernels_per_forward(void);

/* Per-role cycle accounting of the fused kernel (tracing aid; no counterpart in
 * the paper).  Only a library built with -DSOL_ATTN_PROFILE (libsol_attn_profile.so)
 * collects it; the regular build returns SOL_ATTN_ERR_UNSUPPORTED.  Copies up to
 * n (<= 48) counters, summed over CTAs, into cycles (host memory) after a device
 * synchronisation; reset != 0 clears them.  Slot order: the ProfSlot enum in
 * fused.cuh (wait cycles per role and barrier, per-role totals, softmax phases). */
int sol_attn_profile_read(uint64_t* cycles, int n, int reset);

/* Allocation-free variant of sol_attn_forward (the paper has no counterpart;
 * it exists for callers that may not allocate device memory, e.g. code inside
 * a fixed memory pool or a serving loop where cudaMalloc could synchronise).
 * Same arguments, layout and result as sol_attn_forward.  Its scratch lives in
 * one fixed 96 MiB device array inside the library, reserved on every GPU that
 * loads it and held until the process exits; shapes whose scratch does not fit
 * (about B*H*ceil(L/64)*d*14 + B*H*d*d*8 bytes) return SOL_ATTN_ERR_UNSUPPORTED.
 * Nothing is allocated or freed.  The first call on a device looks up that
 * array's device address and clears its status word, so make that first call
 * outside any stream capture.  All calls on a device share the array and it
 * keeps the last call's contents: calls that overlap on the GPU (different
 * streams, or host threads racing) race on it and must be serialised by the
 * caller.  sol_attn_stats does not report on these calls; sol_attn_noalloc_status
 * reads the call's device status word. */
int sol_attn_forward_noalloc(const void* q, const void* k, const void* v, void* out,
                             int B, int H, int L, int d, int block, int chunk, float beta,
                             void* stream);

/* Comparison router for the routing-cost report (a measurement aid, not a step
 * of the method; experiments: routing latency against top-k / top-p routers
 * that materialise and traverse the proxy map, Fig. 5b/5c).  From the pooled
 * Q̄, K̄ of the last sol_attn_stage_pool or forward of this shape on this
 * device, writes the full proxy map ŝ_ij = Q̄_i·K̄_j/sqrt(d) of every head to
 * HBM (fp32, B*H*N*N values, in a library-owned buffer grown with cudaMalloc)
 * and keeps each row's k largest entries (ties: lower block index first) as
 * bits of mask (device, [B,H,N,ceil(N/32)] uint32, caller-owned; k <= 0 keeps
 * none, k >= N all).  Two kernels enqueued on stream.  SOL_ATTN_ERR_STATE
 * without a matching earlier pooling. */
int sol_attn_topk_route(int B, int H, int L, int d, int block, int k, uint32_t* mask, void* stream);

/* Status of the last allocation-free forward on this device (the paper has no
 * counterpart).  That forward clears the device status word when it is
 * enqueued; this call synchronises stream, copies the word to the host (no
 * allocation), clears it and returns SOL_ATTN_OK, SOL_ATTN_ERR_TIMEOUT (a
 * bounded wait of the fused kernel gave up; out is not valid) or
 * SOL_ATTN_ERR_DEVICE.  SOL_ATTN_ERR_STATE if no allocation-free forward has
 * run on this device.  Pass the stream the forward was enqueued on. */
int sol_attn_noalloc_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SOL_ATTN_H_ */
