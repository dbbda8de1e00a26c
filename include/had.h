/*
 * had.h -- C ABI of the B200 (sm_100a) library for the inference forward pass
 * of Hamming Attention Distillation (HAD).
 *
 * Source of the method: "Hamming Attention Distillation: Binarizing Keys and
 * Queries for Efficient Long-Context Transformers" (arXiv 2502.01770), as
 * summarised by its pith.science review page, section "What carries the
 * argument" and the circularity audit (Eqs. 4-7, Eq. 12), and by the abstract
 * on the mlsanity.com index page.  Queries and keys are standardized by
 * per-head coefficients sigma_Q, sigma_K and sign-quantized to {-1,+1}; the
 * logit of query i and key j is the +/-1 dot product
 *     s_ij = d - 2 * popcount(q_i XOR k_j)         (an integer in [-d, d]);
 * each query row keeps its N largest logits (ties go to the lower key index),
 * a softmax with temperature tau runs over those N only, and the output is
 *     O_i = sum_{j kept} p_ij V_j,   p_ij = exp(tau (s_ij - m_i)) / Z_i
 * with V kept in full precision and O returned as fp32.
 *
 * Entry points
 *   - the forward in one call (had_attention_fwd, _noalloc) or in two
 *     stages (had_attention_prepare + had_attention_core), and its building
 *     blocks had_binarize_pack, had_hamming_topn, had_sparse_softmax_av;
 *   - the causal form (had_attention_causal_fwd; had_hamming_topn_causal);
 *   - the top-N mass-retention diagnostic (had_topn_mass);
 *   - the soft-code (tanh) forward of the training stages
 *     (had_soft_attention_fwd; had_soft_binarize, had_soft_topn,
 *     had_soft_softmax_av);
 *   - the straight-through backward (had_attention_bwd);
 *   - had_workspace_bytes, had_launch_count, had_status_string,
 *     had_set_wait_limit_ns.
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major, contiguous, in device memory, 16-byte
 *     aligned: Q, K, V and O are [B, H, n, d]; packed bits are
 *     [B, H, n, d/32] uint32; idx / logits / p are [B, H, n, N].
 *   - Packed bits: bit k of word w of a row is 1 iff element 32*w + k of
 *     that row has sign -1.  sign(z) = -1 iff z < 0, where z = x / sigma_h is
 *     an IEEE fp32 round-to-nearest division with subnormals kept; +0, -0 and
 *     NaN give +1.
 *   - sigma arrays are device float[H], one coefficient per head.
 *   - Supported: d in {64, 128}; 1 <= N <= n; n * N < 2^31; B, H, n >= 1.
 *   - Ownership: the caller allocates and frees every buffer, workspace
 *     included.  The library allocates nothing.  Its only state between
 *     calls is the wait limit of had_set_wait_limit_ns and the device
 *     address cache of had_attention_fwd_noalloc.
 *   - Calls are asynchronous on `stream` and never synchronize.  Argument
 *     errors are returned before anything is launched.  A launch failure
 *     returns HAD_ERR_CUDA.  Conditions only the device can see are OR-ed
 *     into *dev_status as bit (1 << code) (for example 1 << HAD_ERR_BAD_SIGMA
 *     when a sigma is <= 0 or not finite); dev_status is an optional device
 *     int32 the caller zeroes beforehand and reads after synchronizing.
 *     Outputs of a call that flagged a device condition are unspecified.
 */
#ifndef HAD_H
#define HAD_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define HAD_API __attribute__((visibility("default")))
#else
#define HAD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HAD_OK = 0,
    HAD_ERR_INVALID_ARG = 1,  /* null pointer, bad size, N outside [1, n], misalignment */
    HAD_ERR_UNSUPPORTED = 2,  /* d not in {64, 128}, or sizes beyond the stated limits */
    HAD_ERR_WORKSPACE = 3,    /* workspace null or smaller than had_workspace_bytes() */
    HAD_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
    HAD_ERR_BAD_SIGMA = 5,    /* device flag: a sigma is <= 0, NaN or infinite */
    HAD_ERR_TIMEOUT = 6       /* device flag: a bounded on-chip wait gave up */
} had_status_t;

typedef enum {
    HAD_BF16 = 0,             /* bfloat16 storage */
    HAD_F32 = 1               /* IEEE binary32 storage */
} had_dtype_t;

typedef enum {
    HAD_OP_BINARIZE_PACK = 0,     /* had_binarize_pack */
    HAD_OP_HAMMING_TOPN = 1,      /* had_hamming_topn */
    HAD_OP_ATTENTION_FWD = 2,     /* had_attention_fwd */
    HAD_OP_SPARSE_SOFTMAX_AV = 3, /* had_sparse_softmax_av */
    HAD_OP_ATTENTION_PREPARE = 4, /* had_attention_prepare */
    HAD_OP_ATTENTION_CORE = 5,    /* had_attention_core */
    HAD_OP_TOPN_MASS = 6,         /* had_topn_mass */
    HAD_OP_ATTENTION_CAUSAL = 7,  /* had_attention_causal_fwd */
    HAD_OP_SOFT_BINARIZE = 8,     /* had_soft_binarize */
    HAD_OP_SOFT_TOPN = 9,         /* had_soft_topn */
    HAD_OP_SOFT_SOFTMAX_AV = 10,  /* had_soft_softmax_av */
    HAD_OP_SOFT_ATTENTION_FWD = 11, /* had_soft_attention_fwd */
    HAD_OP_ATTENTION_BWD = 12     /* had_attention_bwd */
} had_op_t;

/*
 * Standardize + sign + bit-pack (Eqs. 4-5 with the Eq. 12 coefficients).
 *   x      [B,H,n,d] of dtype dt (device)
 *   sigma  [H] float (device); flags HAD_ERR_BAD_SIGMA if any is <= 0 or
 *          not finite (the bits are still written from the division)
 *   bits   [B,H,n,d/32] uint32 out (device)
 */
HAD_API had_status_t had_binarize_pack(const void *x, had_dtype_t dt, const float *sigma,
                               int B, int H, int n, int d, uint32_t *bits,
                               int32_t *dev_status, cudaStream_t stream);

/*
 * Hamming logits and top-N selection (Eq. 5 and Eq. 6), unfused.
 *   qbits, kbits  [B,H,n,d/32] packed as above (device)
 *   idx     [B,H,n,N] int32 out: kept key indices of each row, ascending
 *   logits  [B,H,n,N] int16 out, or NULL: s_ij of the kept keys, same order
 *   ws      workspace of had_workspace_bytes(HAD_OP_HAMMING_TOPN, ...) bytes
 *           (may be NULL when that size is 0)
 * The kept set is exact: the N largest s_ij, the lower key index winning at
 * the threshold.
 */
HAD_API had_status_t had_hamming_topn(const uint32_t *qbits, const uint32_t *kbits,
                              int B, int H, int n, int d, int N,
                              int32_t *idx, int16_t *logits,
                              void *ws, size_t ws_bytes,
                              int32_t *dev_status, cudaStream_t stream);

/*
 * Softmax over the kept logits and sparse product with V (Eq. 7).
 *   idx, logits  [B,H,n,N] as produced by had_hamming_topn (device)
 *   V      [B,H,n,d] of dtype dt (device), full precision
 *   tau    softmax temperature (1/sqrt(d) in the reference workloads)
 *   out    [B,H,n,d] float out
 *   p      [B,H,n,N] float out, or NULL: the probabilities, same order as idx
 * An idx entry of -1 is an empty slot (as had_hamming_topn_causal writes
 * them): it gets probability 0 and no error; a row of empty slots gets zeros.
 * Every other idx entry must lie in [0, n); entries outside it are skipped
 * and flag HAD_ERR_INVALID_ARG in *dev_status.
 */
HAD_API had_status_t had_sparse_softmax_av(const int32_t *idx, const int16_t *logits,
                                   const void *V, had_dtype_t dt,
                                   int B, int H, int n, int d, int N, float tau,
                                   float *out, float *p,
                                   int32_t *dev_status, cudaStream_t stream);

/*
 * The whole forward pass, fused: O = sparse_softmax_topN(binarized logits) V.
 *   Q, K, V   [B,H,n,d] of dtype dt (device)
 *   sigma_q, sigma_k  [H] float (device)
 *   out       [B,H,n,d] float out
 *   dbg_idx, dbg_logits  [B,H,n,N] optional outputs of the kept set (may be
 *             NULL; when given they hold exactly what had_hamming_topn would)
 *   tau       softmax temperature, finite and >= 0 (else HAD_ERR_INVALID_ARG)
 *   ws        workspace of had_workspace_bytes(HAD_OP_ATTENTION_FWD, ...)
 * The n x n logit matrix never goes to memory.
 */
HAD_API had_status_t had_attention_fwd(const void *Q, const void *K, const void *V,
                               had_dtype_t dt,
                               const float *sigma_q, const float *sigma_k,
                               int B, int H, int n, int d, int N, float tau,
                               float *out, int32_t *dbg_idx, int16_t *dbg_logits,
                               void *ws, size_t ws_bytes,
                               int32_t *dev_status, cudaStream_t stream);

/*
 * had_attention_fwd in two stages sharing one workspace (same size as
 * had_attention_fwd's): had_attention_prepare standardizes and signs Q and K
 * into tensor-core operand tiles and packed bits and converts V, and
 * had_attention_core runs the fused kernel (and the exact recomputation of
 * any row whose threshold fell outside its sampled window) on them.  The
 * two in order on one stream compute exactly what had_attention_fwd does;
 * core reads only the workspace and V.  Arguments as had_attention_fwd.
 */
HAD_API had_status_t had_attention_prepare(const void *Q, const void *K, const void *V,
                                           had_dtype_t dt, const float *sigma_q,
                                           const float *sigma_k, int B, int H, int n, int d,
                                           int N, void *ws, size_t ws_bytes,
                                           int32_t *dev_status, cudaStream_t stream);

HAD_API had_status_t had_attention_core(const void *V, had_dtype_t dt, int B, int H, int n,
                                        int d, int N, float tau, float *out, int32_t *dbg_idx,
                                        int16_t *dbg_logits, void *ws, size_t ws_bytes,
                                        int32_t *dev_status, cudaStream_t stream);

/*
 * Diagnostic of the fused forward: how many query rows of the last
 * had_attention_fwd / _core / had_attention_causal_fwd call on this
 * workspace had their threshold level fall outside the window the fused
 * kernel resolves exactly, and so were recomputed whole by the exact fix-up
 * kernel (they get the same result; only the time differs).  Enqueues on
 * `stream` a copy of that int32 count into *dst (device or host memory).
 * ws, ws_bytes and the sizes as in that call.
 */
HAD_API had_status_t had_attention_window_misses(const void *ws, size_t ws_bytes, int B, int H,
                                                 int n, int d, int N, int32_t *dst,
                                                 cudaStream_t stream);

/*
 * Causal variant.  The pages print no causal rule; this is the plain reading
 * for decoder use: query i of a head sees keys 0 .. i only and keeps the
 * N_i = min(N, i + 1) largest visible logits (ties to the lower index), in
 * ascending key order.  Slots N_i .. N-1 of a row hold idx -1 and logit 0;
 * had_sparse_softmax_av treats idx -1 as an empty slot (no weight, no
 * error), so the two compose.  Arguments as had_hamming_topn (no workspace).
 */
HAD_API had_status_t had_hamming_topn_causal(const uint32_t *qbits, const uint32_t *kbits,
                                             int B, int H, int n, int d, int N, int32_t *idx,
                                             int16_t *logits, int32_t *dev_status,
                                             cudaStream_t stream);

/*
 * Causal forward in one call, on the fused tensor-core path of
 * had_attention_fwd: query i sees keys 0 .. i and keeps min(N, i + 1) of
 * them (the rule of had_hamming_topn_causal).  Each CTA streams keys only up
 * to its last query row, so the call does about half the work of the
 * non-causal one.  Arguments, workspace (had_workspace_bytes(
 * HAD_OP_ATTENTION_CAUSAL, ...) = that of HAD_OP_ATTENTION_FWD), launch
 * count and errors as had_attention_fwd; dbg_idx / dbg_logits, when given,
 * hold the kept set with empty slots as idx -1, logit 0.
 */
HAD_API had_status_t had_attention_causal_fwd(const void *Q, const void *K, const void *V,
                                              had_dtype_t dt, const float *sigma_q,
                                              const float *sigma_k, int B, int H, int n, int d,
                                              int N, float tau, float *out, int32_t *dbg_idx,
                                              int16_t *dbg_logits, void *ws, size_t ws_bytes,
                                              int32_t *dev_status, cudaStream_t stream);

/*
 * Soft codes for the tanh training stages ("Hamming Attention
 * Distillation", pith.science review: the annealing schedule trains first
 * with a c-scaled tanh, Eq. 13, that approaches the sign as c grows).
 * t = tanh(c * (x / sigma[h])) in fp32: the division and the product are
 * IEEE round-to-nearest, tanh is CUDA's tanhf (within 2 ulp).
 *   x      [B,H,n,d] of dtype dt (device); sigma [H] float (device)
 *   c      the tanh scale, finite and > 0
 *   t      [B,H,n,d] float out
 * A sigma <= 0 or non-finite flags HAD_ERR_BAD_SIGMA in *dev_status.
 * Non-finite x follow tanhf (+-inf -> +-1, NaN -> NaN); NaN codes are
 * outside the contract of the calls below.
 */
HAD_API had_status_t had_soft_binarize(const void *x, had_dtype_t dt, const float *sigma,
                                       float c, int B, int H, int n, int d, float *t,
                                       int32_t *dev_status, cudaStream_t stream);

/*
 * Top-N of the soft logits s_ij = sum_k tq_ik tk_jk (fp32 FMA in the order
 * k = 0 .. d-1).  Same selection rule as had_hamming_topn: the N largest
 * (ties to the lower key index, -0 equal to +0), ascending key order.
 *   tq, tk   [B,H,n,d] float codes (device)
 *   idx      [B,H,n,N] int32 out;  logits [B,H,n,N] float out, or NULL
 *   ws       device scratch of had_workspace_bytes(HAD_OP_SOFT_TOPN, ...)
 *            bytes: the fp32 logit matrices of a group of heads (up to
 *            2 GiB); groups run one after another (2 launches each)
 * n is limited to 32768 (HAD_ERR_UNSUPPORTED beyond).
 */
HAD_API had_status_t had_soft_topn(const float *tq, const float *tk, int B, int H, int n, int d,
                                   int N, int32_t *idx, float *logits, void *ws, size_t ws_bytes,
                                   int32_t *dev_status, cudaStream_t stream);

/*
 * had_sparse_softmax_av for fp32 logits (the output of had_soft_topn); same
 * arguments, empty slots and error behaviour.
 */
HAD_API had_status_t had_soft_softmax_av(const int32_t *idx, const float *logits, const void *V,
                                         had_dtype_t dt, int B, int H, int n, int d, int N,
                                         float tau, float *out, float *p, int32_t *dev_status,
                                         cudaStream_t stream);

/*
 * Soft forward in one call: had_soft_binarize of Q and K with scale c, then
 * had_soft_topn, then had_soft_softmax_av, inside a caller workspace of
 * had_workspace_bytes(HAD_OP_SOFT_ATTENTION_FWD, ...) bytes (codes, kept
 * set and the logit scratch).  Other arguments as had_attention_fwd.
 */
HAD_API had_status_t had_soft_attention_fwd(const void *Q, const void *K, const void *V,
                                            had_dtype_t dt, const float *sigma_q,
                                            const float *sigma_k, float c, int B, int H, int n,
                                            int d, int N, float tau, float *out, void *ws,
                                            size_t ws_bytes, int32_t *dev_status,
                                            cudaStream_t stream);

/*
 * Backward pass of had_attention_fwd for the straight-through training stage
 * ("Hamming Attention Distillation", pith.science review: a straight-through
 * estimator finishes the binarization after the tanh stages).  The kept set
 * is recomputed and held fixed; softmax and value product are
 * differentiated exactly; the sign passes the gradient where
 * |x / sigma| <= clip (clip = 1 is the usual choice, +inf passes it
 * everywhere); the standardization contributes 1 / sigma and sigma gets no
 * gradient.
 *   Q, K, V, dt, sigma_q, sigma_k, N, tau   as had_attention_fwd
 *   dout   [B,H,n,d] float (device): gradient of the loss w.r.t. the output
 *   idx, logits  the forward's kept set ([B,H,n,N] int32 / int16, as
 *          had_attention_fwd's debug outputs or had_hamming_topn give it),
 *          or both NULL: then it is recomputed (one more launch)
 *   clip   >= 0 (NaN rejected)
 *   dq, dk, dv  [B,H,n,d] float out
 *   ws     device workspace of had_workspace_bytes(HAD_OP_ATTENTION_BWD, ...)
 *          bytes (about 36 + 30 N bytes per query row)
 * The key-side sums (dk, dv) run over per-key lists that atomics fill, so
 * their fp32 rounding is not reproducible bit for bit run to run.
 */
HAD_API had_status_t had_attention_bwd(const void *Q, const void *K, const void *V,
                                       had_dtype_t dt, const float *sigma_q,
                                       const float *sigma_k, const float *dout,
                                       const int32_t *idx, const int16_t *logits, int B, int H,
                                       int n, int d, int N, float tau, float clip, float *dq,
                                       float *dk, float *dv, void *ws, size_t ws_bytes,
                                       int32_t *dev_status, cudaStream_t stream);

/*
 * Top-N mass retention diagnostic ("Hamming Attention Distillation",
 * pith.science review: the concrete test of the premise that a small N keeps
 * most of the softmax mass, and the free-parameter notes on N).  For every
 * query row and every threshold p[k]: the smallest N such that the N
 * largest weights of the full softmax over all n keys (temperature tau,
 * binarized logits s = d - 2 Hamming) hold at least p[k] of the row's total.
 * Computed from the row's histogram of logit levels, in fp64.
 *   qbits, kbits  [B,H,n,d/32] uint32 (device), as had_binarize_pack writes
 *   tau           >= 0
 *   p             np thresholds in (0, 1] (HOST memory, read during the call)
 *   np            1 .. 8
 *   nmin          [B,H,n,np] int32 out (device)
 * No workspace.  Invalid arguments return HAD_ERR_INVALID_ARG before any
 * launch; d outside {64, 128} returns HAD_ERR_UNSUPPORTED.
 */
HAD_API had_status_t had_topn_mass(const uint32_t *qbits, const uint32_t *kbits, int B, int H,
                                   int n, int d, float tau, const double *p, int np,
                                   int32_t *nmin, int32_t *dev_status, cudaStream_t stream);

/*
 * had_attention_fwd for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot call cudaMalloc (code running under another runtime's
 * allocator, plugins handed only their input and output buffers, processes
 * whose device memory is reserved up front).  It computes exactly what
 * had_attention_fwd computes, with the same kernels, but takes its
 * workspace from a fixed device array inside the library instead of a
 * caller buffer, and allocates nothing.
 *   - Limit: had_workspace_bytes(HAD_OP_ATTENTION_FWD, ...) must not exceed
 *     had_noalloc_scratch_bytes() (96 MiB, enough for B=4 H=16 n=4096
 *     d=64 N=512); larger sizes return HAD_ERR_WORKSPACE before any launch.
 *   - The array is part of the loaded module: every GPU that loads the
 *     library holds it until the process exits.
 *   - The array's device address belongs to the CUDA context the module
 *     was loaded in.  The first call in each context (the one current on
 *     the calling thread: a device's primary context, or one the caller
 *     created and made current) looks the address up with
 *     cudaGetSymbolAddress and caches it under that context; later calls in
 *     the same context reuse it.  Make that first call before any stream
 *     capture.
 *   - Every call shares the one array per device and leaves its contents
 *     behind; the call re-initialises everything it reads.  Calls whose
 *     kernels overlap on the GPU (different streams, or host threads
 *     without ordering) race on the array and give undefined results.
 * Arguments are those of had_attention_fwd without the debug outputs and
 * the workspace.
 */
HAD_API had_status_t had_attention_fwd_noalloc(const void *Q, const void *K, const void *V,
                                               had_dtype_t dt, const float *sigma_q,
                                               const float *sigma_k, int B, int H, int n,
                                               int d, int N, float tau, float *out,
                                               int32_t *dev_status, cudaStream_t stream);

/* Size in bytes of the fixed array had_attention_fwd_noalloc works in. */
HAD_API size_t had_noalloc_scratch_bytes(void);

/*
 * Limit, in nanoseconds, of every on-chip wait of the fused forward kernels
 * for another role of the same CTA (an operand copy, a tensor-core MMA, an
 * epilogue warp).  A wait that runs out flags HAD_ERR_TIMEOUT in
 * *dev_status; the CTA then lets its copies and MMAs in flight complete
 * (those drain waits keep a limit of 0.5 s), frees its tensor memory and
 * returns, so the context stays usable; the outputs of that call are
 * unspecified.  Applies to non-causal calls of had_attention_fwd, _core and
 * _noalloc launched afterwards, process-wide.  ns = 0 restores the default
 * (2 s, far beyond any real wait).  Returns the previous limit.  Not a
 * tuning knob: it exists so that the timeout path can be exercised.
 */
HAD_API unsigned long long had_set_wait_limit_ns(unsigned long long ns);

/*
 * Workspace bytes an operation needs for these sizes (0 if none), or
 * (size_t)-1 for unsupported or invalid sizes.
 */
HAD_API size_t had_workspace_bytes(int op, int B, int H, int n, int d, int N);

/* Static, human-readable name of a status code. */
HAD_API const char *had_status_string(had_status_t status);

/*
 * Number of kernels one call of `op` enqueues for these sizes (-1 for
 * unsupported or invalid sizes).  Lets a caller count launches without a
 * profiler.  HAD_OP_ATTENTION_BWD counts the recomputation of the kept set;
 * a call given the forward's kept set enqueues one kernel fewer.
 */
HAD_API int had_launch_count(int op, int B, int H, int n, int d, int N);

#ifdef __cplusplus
}
#endif

#endif /* HAD_H */
