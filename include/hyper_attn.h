/*
 * hyper_attn.h -- C ABI of the B200-native HyperAttention forward pass (sm_100a).
 *
 * The method ("HyperAttention: Long-context Attention in Near-Linear Time"; research-map summary page,
 * section "Approach", and the OpenReview abstract): hash the rows of Q and K with sortLSH (signs of r
 * random Gaussian projections read as a Gray-code rank), sort both by rank, compute exact softmax
 * attention inside aligned diagonal blocks of the sorted order, estimate the softmax normaliser by adding
 * a rescaled uniform sample of m key columns to the exact block row sums, approximate the product with V
 * from the same sampled columns, and merge the two parts. The causal variant (same page, one-line summary
 * and "Limitations") splits recursively into a causal upper-left half, a causal lower-right half and a
 * non-causal off-diagonal block, with exact causal attention below a base size, and merges the parts in
 * log space.
 *
 * Conventions for every entry point:
 *   - Return value: HA_OK (0) or a negative ha_status. Argument errors are detected on the host before
 *     anything is enqueued; the text of the last error is available from hyper_attn_last_error().
 *   - Device pointers are plain CUDA device addresses owned by the caller; the library never frees them.
 *     Host pointers are ordinary host memory owned by the caller (page-locked memory makes copies faster).
 *   - Tensors Q, K, V, O are dense row-major [batch, heads, n, d] with element type given by the options
 *     (bf16 by default), 16-byte aligned base addresses.
 *   - A handle is used by one host thread at a time. Work is enqueued on the handle's stream
 *     (hyper_attn_set_options) and runs asynchronously unless stated otherwise.
 *   - There is no CPU fallback: without a usable sm_100 device the calls fail with HA_ERR_CUDA or
 *     HA_ERR_UNSUPPORTED.
 */
#ifndef HYPER_ATTN_H
#define HYPER_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HA_API __attribute__((visibility("default")))
#else
#define HA_API
#endif

typedef struct hyper_attn_s *hyper_attn_t;

typedef enum {
    HA_OK = 0,
    HA_ERR_INVALID_ARG = -1,  /* a shape, pointer or option is outside what the method accepts */
    HA_ERR_UNSUPPORTED = -2,  /* valid for the method but not implemented on this device or dtype */
    HA_ERR_CUDA = -3,         /* a CUDA runtime call failed (message in hyper_attn_last_error) */
    HA_ERR_OOM = -4,          /* workspace allocation failed */
    HA_ERR_TIMEOUT = -5       /* a bounded device-side wait gave up (reported by hyper_attn_status) */
} ha_status;

typedef enum { HA_DTYPE_BF16 = 0, HA_DTYPE_FP32 = 1 } ha_dtype;

/* Attention kernel family. AUTO: tensor-core (tcgen05) kernels for bf16 inputs, SIMT fp32 kernels for
 * fp32 inputs. SIMT: SIMT fp32 kernels for any input type. TC: tensor-core kernels (bf16 only). */
typedef enum { HA_KERNEL_AUTO = 0, HA_KERNEL_SIMT = 1, HA_KERNEL_TC = 2 } ha_kernel;

/* How the sampled part of the product with V is estimated ("HyperAttention: Long-context Attention in
 * Near-Linear Time", research-map summary, "Approach").
 * UNIFORM: the m uniform column samples of the normaliser also serve the product with V (weight N/m).
 * ROWNORM: the normaliser keeps the uniform samples; the product with V takes m draws with replacement,
 *   row j with probability p_j = ||v_j||^2 / sum ||v||^2 over the problem's key rows, weight 1/(m p_j).
 *   The squared norms are sequential fp32 multiply-adds, the draws Philox4x64-10 under key (seed, 3) at
 *   counter (t/4, node, bh, 0), word t mod 4, u = (w >> 11) 2^-53, the smallest j whose cumulative sum
 *   exceeds u times the total; all of it runs on the device. The tensor-core kernels take m <= 256 (bf16);
 *   beyond that AUTO falls back to the SIMT kernels and HA_KERNEL_TC returns HA_ERR_UNSUPPORTED. */
typedef enum { HA_SAMPLING_UNIFORM = 0, HA_SAMPLING_ROWNORM = 1 } ha_sampling;

typedef struct {
    int dtype;            /* ha_dtype of Q, K, V. Default HA_DTYPE_BF16. */
    int out_dtype;        /* ha_dtype of O, or -1 for "same as dtype". Default -1. */
    int64_t batch;        /* B >= 1; the problems are the B*heads (batch, head) pairs. Default 1. */
    int64_t causal_base;  /* c: size below which the causal recursion is exact causal attention.
                             Default 4096. Causal calls need n = c * 2^L (L >= 0) or n <= c. */
    void *stream;         /* cudaStream_t to enqueue on; NULL = the legacy default stream. */
    int kernel;           /* ha_kernel. Default HA_KERNEL_AUTO. */
    int debug_captures;   /* 1: also store the per-row log normaliser (HA_DBG_LSE, non-causal). Default 0. */
    int64_t bh_offset;    /* Global index of this call's first (batch, head) problem, >= 0. The sample draws
                             of local problem i are those of problem bh_offset + i, so a run split over
                             several calls or GPUs (each taking a contiguous range of problems) gives the
                             same result as one call over all problems. Default 0. */
    int test_stall_ms;    /* Test hook for the failure path, 0..1000. When > 0, the tensor-core level kernel
                             (uniform sampling; a separate instance of it) makes its first softmax wait target a
                             barrier that nothing ever completes and give up after this many milliseconds:
                             every role of the kernel then stops, the output is undefined, and
                             hyper_attn_status reports HA_ERR_TIMEOUT. The device stays usable. Default 0. */
    int sampling;         /* ha_sampling of the product with V. Default HA_SAMPLING_UNIFORM. */
} ha_options;

/* Create a handle bound to CUDA device `device`. The handle owns a grow-only device workspace (ranks,
 * permutations, per-level partial results, the draws) and a small page-locked staging buffer.
 * Fails with HA_ERR_CUDA if the device cannot be used, HA_ERR_UNSUPPORTED if it is not sm_100. */
HA_API int hyper_attn_create(hyper_attn_t *out, int device);

/* Replace the handle's options (copied). Invalid values return HA_ERR_INVALID_ARG and keep the old ones. */
HA_API int hyper_attn_set_options(hyper_attn_t h, const ha_options *opt);

/* Fill *opt with the defaults listed above. */
HA_API void hyper_attn_default_options(ha_options *opt);

/*
 * HyperAttention forward on device memory: O = approx softmax(Q K^T) V for every (batch, head).
 *   Q, K, V (in), O (out): device pointers, [batch, heads, n, d]; O must not alias Q, K or V.
 *   No softmax scale is applied inside exp: callers fold it into Q and K (e.g. both times d^-1/4).
 *   n      rows per head; n % min(block, n) == 0.
 *   d      head dimension, 64 or 128.
 *   block  b: sorted rows per diagonal block (b' = min(b, N) for a problem of N rows).
 *   m      columns sampled uniformly without replacement per problem, 0 <= m <= N of every problem.
 *   r      LSH projections (hash bits), 0 <= r <= 16; r = 0 puts every row in one bucket.
 *   causal 0: one problem of n queries and n keys. 1: the recursive causal variant with the handle's
 *          causal_base; every off-diagonal problem has N >= causal_base rows and needs b | N, m <= N.
 *   seed   drives the projection matrix and the column samples (see hyper_attn_draw).
 * Enqueued on the handle's stream; returns after enqueueing. Argument errors return synchronously and
 * enqueue nothing. The workspace is reused by the next call on the same handle (stream-ordered).
 */
HA_API int hyper_attn_forward(hyper_attn_t h, const void *Q, const void *K, const void *V, void *O,
                       int64_t n, int d, int heads, int block, int m, int r, int causal, uint64_t seed);

/*
 * Exact softmax attention O = softmax(Q K^T) V for every (batch, head) problem: no sampling, hashing or
 * blocks; causal = 1 lets query i see keys 0..i. This is the reference the approximation is measured
 * against ("HyperAttention: Long-context Attention in Near-Linear Time", research-map summary, "Key
 * results": speed-ups are quoted against exact attention), computed here on the same tensor-core kernel
 * as the method's exact causal leaves. Arguments as for hyper_attn_forward (device pointers, the
 * handle's dtype, batch, out_dtype and stream), with these limits: bf16 inputs, d in {64, 128}, n a
 * multiple of 128 (HA_ERR_UNSUPPORTED otherwise). Enqueued on the handle's stream; device-side wait
 * timeouts surface through hyper_attn_status.
 */
HA_API int hyper_attn_exact(hyper_attn_t h, const void *Q, const void *K, const void *V, void *O,
                            int64_t n, int d, int heads, int causal);

/*
 * Backward pass: the gradients of sum(dO * O) with respect to Q, K and V, where O is the forward estimate of
 * hyper_attn_forward with the same arguments and options (the sort permutations and the sample draws are
 * held fixed: they are constants of the forward pass). Every row's estimate is a weighted softmax over a
 * sparse key set (its sortLSH block or causal leaf with weight 1, uniform samples outside the block with N/m,
 * row-norm draws with 1/(m p_j) in the numerator only), so ("HyperAttention: Long-context Attention in
 * Near-Linear Time", research-map summary, "Key results": the speed-ups are for forward and backward):
 *   dS_qk = Wn e^{s_qk - L_q} (dO_q . v_k) - Wd e^{s_qk - L_q} (dO_q . O_q),
 *   dQ = dS K, dK = dS^T Q, dV_k = sum_q Wn e^{s_qk - L_q} dO_q.
 *   Q, K, V, dO  device pointers, [batch, heads, n, d] of the options' dtype (read only).
 *   dQ, dK, dV   device pointers, [batch, heads, n, d] fp32, written (overwritten); no aliasing.
 * The forward pass is recomputed (its O in fp32 and the log normalisers stay in the workspace); the gradients
 * are accumulated by SIMT fp32 kernels, dK and dV with atomic adds, so the last bits may vary between runs.
 * Enqueued on the options' stream; same argument checks and error codes as hyper_attn_forward.
 */
HA_API int hyper_attn_backward(hyper_attn_t h, const void *Q, const void *K, const void *V, const void *dO, float *dQ,
                               float *dK, float *dV, int64_t n, int d, int heads, int block, int m, int r, int causal,
                               uint64_t seed);

/*
 * Hardness diagnostics of the attention matrices of small non-causal problems ("HyperAttention: Long-context
 * Attention in Near-Linear Time", research-map summary, "Approach" and "Key results", abstract page: the
 * guarantee rests on the max column norm of the normalised attention matrix and on the ratio of row norms
 * once the large entries are removed). For each (batch, head) problem b, with A_ij = exp(q_i . k_j) and
 * W = D^-1 A (the softmax matrix):
 *   alpha[b] = n * max_{j >= first_col} sum_i W_ij^2   (1 for uniform attention; first_col > 0 leaves out
 *              the first columns, e.g. sink-like heavy columns);
 *   kappa[b] = max_i R_i / min_i R_i, R_i = the sum of A_ij over the columns outside row i's block of the
 *              sortLSH order that hyper_attn_forward would use for (block, r, seed) (NaN when no row has
 *              such columns, +inf when only some rows have none).
 * Q, K: device pointers as for hyper_attn_forward (the handle's dtype and batch). alpha, kappa: HOST arrays
 * of batch*heads doubles. Every entry of A is visited, so n <= 16384. Synchronous: returns after the values
 * are on the host. Errors: HA_ERR_INVALID_ARG for null pointers, n > 16384, first_col outside [0, n) or an
 * invalid shape.
 */
HA_API int hyper_attn_diagnostics(hyper_attn_t h, const void *Q, const void *K, int64_t n, int d, int heads,
                                  int block, int r, uint64_t seed, int64_t first_col, double *alpha,
                                  double *kappa);

/*
 * Same computation with HOST buffers: copies Q, K, V to handle-owned device buffers, runs the forward
 * pass, copies O back and waits. Returns when O is valid on the host. The (batch, head) problems go
 * through in up to 8 contiguous groups so that host-to-device copies, the forward pass (on the handle's
 * stream, after any work already queued there) and device-to-host copies of different groups overlap, on
 * two copy streams the handle owns; the result equals one pass over all problems (each group's draws are
 * keyed by global problem index). The overlap needs page-locked host memory; pageable memory is staged by
 * the CUDA runtime and mostly serialises. With debug captures on, all problems form one group.
 */
HA_API int hyper_attn_forward_host(hyper_attn_t h, const void *Q, const void *K, const void *V, void *O,
                            int64_t n, int d, int heads, int block, int m, int r, int causal, uint64_t seed);

/*
 * The random draws the forward pass makes for these arguments, computed on the host:
 *   P_out  [d][r] float: projection matrix, i.i.d. N(0,1) (Philox4x64-10 + Box-Muller), one per call,
 *          shared by Q and K, all heads and all causal nodes. May be NULL.
 *   S_out  [bh][nodes][m] int32 (bh = batch*heads): ascending column indices in [0, N) of each problem.
 *          Problems are numbered from 0; a forward call with option bh_offset = o uses rows o, o+1, ...
 *          of this array (draw with bh = o + its own problem count).
 *          nodes = 1 (non-causal) or 2^L - 1 (causal; node k is heap node k+1: root 1, children 2i, 2i+1).
 *          May be NULL.
 * Host-only, no device needed.
 */
HA_API int hyper_attn_draw(uint64_t seed, int d, int r, int64_t bh, int64_t n, int m, int causal, int64_t base,
                    float *P_out, int32_t *S_out);

/* Number of causal levels L (0 for non-causal) and sample sets per problem for these arguments;
 * returns HA_ERR_INVALID_ARG for an invalid causal shape. */
HA_API int hyper_attn_levels(int64_t n, int causal, int64_t base, int *levels_out, int64_t *nodes_out);

/* Debug captures of the last forward call on this handle, copied to host memory after synchronising
 * the handle's stream. `level` selects the sort level (0 for non-causal, 1..L for causal). */
typedef enum {
    HA_DBG_RANK = 0,   /* uint16 [bh][2][n]: sortLSH rank of each Q row (index 0) and K row (index 1) */
    HA_DBG_NEAR = 1,   /* uint8  [bh][2][n]: 1 when some projection of the row is below 1e-4 * ||row||  */
    HA_DBG_PERM = 2,   /* int32  [bh][nodes_l][2][N_l]: sorted position -> local row, Q then K segment   */
    HA_DBG_INV = 3,    /* int32  [bh][nodes_l][2][N_l]: local row -> sorted position                     */
    HA_DBG_LSE = 4,    /* float  [bh][n]: log of the estimated normaliser of each query row (non-causal) */
    HA_DBG_RN_S = 5,   /* int32  [bh][nodes][m]: row-norm draws, row index local to the set's key rows    */
    HA_DBG_RN_LOGW = 6 /* float  [bh][nodes][m]: their log weights log(1 / (m p_j))                       */
} ha_debug_what;
HA_API int hyper_attn_debug_copy(hyper_attn_t h, int what, int level, void *host_dst, size_t bytes);

/* Synchronise the handle's stream and report device-side status: HA_OK, HA_ERR_TIMEOUT if a bounded
 * wait gave up, or HA_ERR_CUDA if the stream holds an error or (HA_DEBUG build, libhyper_attn_debug.so) a
 * tensor-core kernel read a row index out of range from a permutation or a sample list (it then read row 0
 * instead). Clears the device status word. */
HA_API int hyper_attn_status(hyper_attn_t h);

/* Kernel classes for profiling. */
typedef enum {
    HA_KC_HASH = 0,        /* sortLSH hash */
    HA_KC_SORT = 1,        /* counting-sort passes (count, scan, scatter) */
    HA_KC_ATTN = 2,        /* block + sampled attention of one level, including the gather and the merge */
    HA_KC_CAUSAL_BASE = 3, /* exact causal leaves and the final log-space merge */
    HA_KC_DRAWS = 4,       /* row-norm draws on the device (norms, cumulative sums, draws) */
    HA_KC_COUNT = 5
} ha_kernel_class;

/* enable = 1: record a CUDA event pair on the handle's stream around every kernel class launch of the
 * following forward calls; 0: stop recording. Recording adds two event records per launch.
 * Independently of this switch, the host-side enqueue of every kernel class sits in an NVTX range named
 * "ha:hash", "ha:sort", "ha:attn", "ha:causal_base" or "ha:draws", which tracing tools (Nsight Systems) show
 * next to the kernels; without such a tool attached the ranges cost a few nanoseconds. */
HA_API int hyper_attn_profile(hyper_attn_t h, int enable);

/* Synchronise the handle's stream and add, per kernel class (array index = ha_kernel_class, n entries),
 * the summed device time in milliseconds and the number of kernel launches recorded since the previous
 * read; then forget the recorded events. ms and launches may be NULL. */
HA_API int hyper_attn_profile_read(hyper_attn_t h, double *ms, int *launches, int n);

/* Attention kernel family the last forward call used: HA_KERNEL_SIMT or HA_KERNEL_TC (0 before any call). */
HA_API int hyper_attn_last_kernel(hyper_attn_t h);

/* Kernels launched by the last forward call (for launch accounting). */
HA_API int hyper_attn_last_launch_count(hyper_attn_t h);

/* Text of the last error on this handle ("" if none). Valid until the next call on the handle. */
HA_API const char *hyper_attn_last_error(hyper_attn_t h);

/* Test hook for the allocation-failure path: the handle's next `count` allocations (its device workspace, its
 * page-locked staging buffer, the device copies of hyper_attn_forward_host) fail as if the device or the host
 * had no memory left, without calling CUDA. The call that meets one returns HA_ERR_OOM before it enqueues any
 * kernel or copy, the caller's buffers are left as they were, and the handle stays usable: the next call
 * allocates again. count = 0 clears the hook. Returns HA_ERR_INVALID_ARG for a null handle or count < 0. */
HA_API int hyper_attn_test_fail_alloc(hyper_attn_t h, int count);

/* Release the workspace and the handle. NULL is accepted. Synchronises the handle's stream first. */
HA_API int hyper_attn_destroy(hyper_attn_t h);

/*
 * Non-causal forward pass that allocates nothing. The pages describe no such entry point; it exists for
 * callers that cannot call cudaMalloc: plugins inside engines that reserve all device memory up front and
 * forbid allocation while enqueueing, and latency-critical loops that cannot afford the synchronisation an
 * allocation may cause.
 *   Q, K, V, O  device pointers, [heads, n, d] of type `dtype` (HA_DTYPE_BF16 or HA_DTYPE_FP32), each
 *               16-byte aligned; O has the same type; O must not alias Q, K or V. Other arguments as in
 *               hyper_attn_forward (causal = 0).
 *   stream      cudaStream_t to enqueue on (NULL = legacy default stream) on the CURRENT device.
 * Limits (HA_ERR_INVALID_ARG beyond them, checked on the host before anything is enqueued):
 *   heads * n <= 65536, heads <= 64, m <= 512 and m <= n, r <= 10, d in {64, 128}, n a multiple of
 *   min(block, n), pointers 16-byte aligned.
 * All scratch memory (2.5 MiB at most) is one file-scope __device__ array that every GPU loading this
 * library holds until the process exits; no cudaMalloc, cudaFree or other allocating call is made.
 * The first call on a device resolves that array's device address with cudaGetSymbolAddress (with the
 * device current). Every call reuses the same array and leaves its contents behind; calls that overlap on
 * the GPU race with each other, so order them (for example, one stream). Host threads are serialised by a
 * lock. The draws are copied from pageable host arrays that the next call overwrites, so calls must not
 * be made while the stream is capturing: such a call returns HA_ERR_UNSUPPORTED and enqueues nothing.
 * Attention uses the SIMT kernels, which have no device-side waits (no status word to read).
 * Returns after enqueueing; HA_ERR_CUDA if a CUDA call fails (the CUDA error is cleared before returning).
 */
HA_API int hyper_attn_forward_noalloc(const void *Q, const void *K, const void *V, void *O, int64_t n, int d,
                                      int heads, int block, int m, int r, uint64_t seed, int dtype, void *stream);

/* Library version as major*10000 + minor*100 + patch. */
HA_API int hyper_attn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HYPER_ATTN_H */
