/*
 * kdn.h -- C ABI of the B200 (sm_100a) Diagonal Kalman Delta Network memory recurrence.
 *
 * The method (Kalman Delta Networks explainer, sections "把记忆问题重新想成一个滤波问题"
 * and "对角近似"; aifromscratch "Kalman Delta Networks", "Approximation 1: Diagonal KDN";
 * delta-rule tutorial "Память с поправкой"; KDA article "معماری KDA", per-channel decay):
 * per head, with a memory S (d_k x d_v, read as S^T k), a per-channel key-space
 * uncertainty P (d_k), and for every token t
 *
 *     P^-_t = alpha_t^2 * P_{t-1} + sigma_t                        (predict; diagonal stays diagonal)
 *     g_t   = P^-_t * k_t / (r_t + sum_i P^-_{t,i} k_{t,i}^2)      (Kalman gain)
 *     W     = diag(alpha_t) S_{t-1};  u_t = v_t - W^T k_t;  S_t = W + g_t u_t^T   (decayed delta write)
 *     o_t   = S_t^T q_t                                            (readout after the write)
 *     P_t   = P^-_t / (1 + mu * P^-_t * k_t^2 / r_t)               (mean-field projection, scaled by mu)
 *
 * Products and divisions of vectors are elementwise.  alpha in [0,1], sigma >= 0 and
 * r > 0 are variances; mu > 0 scales the precision increment (1 = plain mean-field).
 *
 * Isotropic variant (explainer "各向同性近似"; aifromscratch "Approximation 2: Isotropic
 * KDN"): one uncertainty p per head instead of P (d_k), with the same memory update and
 *
 *     p^-_t = mean_i(alpha_{t,i}^2) p_{t-1} + mean_i(sigma_{t,i})  (trace-keeping predict)
 *     g_t   = p^-_t k_t / (r_t + p^-_t |k_t|^2)                   (exact for an isotropic prior)
 *     p_t   = p^-_t / (1 + mu p^-_t |k_t|^2 / (d_k r_t))          (precision averaged over d_k)
 *
 * Its uncertainty states are [N, H] where the diagonal ones are [N, H, d_k].
 *
 * Conventions shared by every entry point
 *  - Memory: the caller owns every buffer; the library never allocates.  Pointers
 *    marked "device" must be device memory of the current CUDA device; buffers must
 *    not overlap unless stated.
 *  - Layout: contiguous row-major.  Token tensors are [B, T, H, d] (dense batch) or
 *    [1, T_total, H, d] with cu_seqlens (packed varlen); r is [B, T, H].  States are
 *    per sequence: S [N, H, d_k, d_v] fp32, P [N, H, d_k] fp32, N = B or num_seqs.
 *  - Types: token inputs and o are all fp32 or all bf16 (kdn_dtype_t); states fp32.
 *  - Sizes: d_k in {32, 64, 128}, d_v in {32, 64, 128, 256}; other sizes return
 *    KDN_ERR_UNSUPPORTED.  Empty problems (T == 0 or B == 0) are a no-op.
 *  - Streams: every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  Argument validation is synchronous and returns an
 *    error before anything is launched.  A failed launch returns KDN_ERR_CUDA.
 *  - Device-side conditions (a bounded wait that gave up, a packed sequence longer than
 *    the max_seqlen given to the gain scan or the backward) are recorded in a device error
 *    word and reported, after
 *    a stream synchronisation, by kdn_last_device_error().  The outputs of a call whose
 *    kernels recorded such a condition are undefined.
 *  - Thread safety: calls may come from several host threads on different streams.
 *    Calls that share output or state buffers must be ordered by the caller.
 */
#ifndef KDN_H_
#define KDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDN_OK = 0,
    KDN_ERR_INVALID_ARG = 1,   /* null pointer, bad size, non-monotone cu_seqlens (host copy), mu <= 0 */
    KDN_ERR_UNSUPPORTED = 2,   /* d_k / d_v / chunk / dtype combination not built */
    KDN_ERR_CUDA = 3,          /* a CUDA runtime call or a launch failed */
    KDN_ERR_TIMEOUT = 4,       /* a bounded device wait gave up (kernel returned early) */
    KDN_ERR_RANGE = 5,         /* reserved: no path limits the decay range (every alpha in [0,1] is supported) */
    KDN_ERR_WORKSPACE = 6      /* workspace missing or smaller than kdn_workspace_size() */
} kdn_status_t;

typedef enum { KDN_DTYPE_F32 = 0, KDN_DTYPE_BF16 = 1 } kdn_dtype_t;

/* Which uncertainty the recurrence tracks (the `variant` field of kdn_problem_t). */
typedef enum { KDN_VARIANT_DIAGONAL = 0, KDN_VARIANT_ISOTROPIC = 1 } kdn_variant_t;

/* Execution paths of kdn_forward_chunkwise (the `chunk` field):
 *  0        token-serial fused recurrence (any dtype; exact fp32 arithmetic);
 *  16/32/64 chunkwise: for bf16 inputs, d_k = 128 and chunk 64, when the call gets a
 *           workspace of kdn_workspace_size() bytes, the tcgen05 tensor cores in two
 *           launches (a chunk-parallel prep kernel, then the chunk-serial state kernel);
 *           otherwise the fp32 CUDA-core chunk kernel (same algebra, fp32 FMA, exact but
 *           several times slower).  Every path accepts any alpha in [0, 1], alpha = 0
 *           resets included: the tensor-core path forms the intra-chunk decay factors on the
 *           CUDA cores for a chunk whose decay falls below 2^-100 on some channel. */
typedef struct {
    int B, T, H, d_k, d_v;          /* varlen: B == 1 and T = total tokens */
    const int32_t *cu_seqlens;      /* device int32 [num_seqs + 1], cu[0] = 0, cu[num_seqs] = T; NULL = dense batch */
    int num_seqs;                   /* number of packed sequences; ignored (taken as B) when cu_seqlens == NULL */
    kdn_dtype_t in_dtype;           /* dtype of q, k, v, alpha, sigma, r and o */
    float mu;                       /* information scaling, > 0 */
    int chunk;                      /* execution path, see above */
    int max_seqlen;                 /* varlen: upper bound on every sequence length (0 = unknown, taken as T);
                                       sizes the gain scan's work list and the backward's chunk-parallel
                                       uncertainty work lists (the forward needs no bound).  A sequence
                                       longer than it makes kdn_gain_scan / kdn_backward record
                                       KDN_ERR_INVALID_ARG in the device error word. */
    int variant;                    /* kdn_variant_t; 0 (zero-initialised struct) = diagonal */
} kdn_problem_t;

/* Bytes of device workspace for `p`: the larger of what kdn_gain_scan() and the two-launch
 * tensor-core forward use.  The forward's part is about 70 KB per 64-token chunk and head
 * (per-chunk operand records and look-back state); packed sequences hold at most
 * T/64 + num_seqs chunks per head, so it does not depend on `max_seqlen`.  The forward
 * also accepts workspace = NULL and then runs the fp32 CUDA-core paths.  Host-only. */
kdn_status_t kdn_workspace_size(const kdn_problem_t *p, size_t *bytes);

/* Prefill / training forward over whole sequences (KDA article, "chunkwise" regime;
 * explainer, "对角近似").
 *  q, k, alpha, sigma : device [B, T, H, d_k]        (in_dtype)
 *  v                  : device [B, T, H, d_v]        (in_dtype)
 *  r                  : device [B, T, H]             (in_dtype)
 *  S0, P0             : device fp32 [N, H, d_k, d_v], [N, H, d_k] ([N, H] isotropic); NULL -> S0 = 0, P0 = 1
 *  o                  : device [B, T, H, d_v]        (in_dtype), written for every token
 *  S_out, P_out       : device fp32, final states per sequence (shapes as S0, P0); either may be NULL.
 *                       They may not alias S0 / P0.
 *  workspace          : device, 256-byte aligned, or NULL.  The tensor-core path (bf16,
 *                       d_k = 128, chunk 64) runs only with >= kdn_workspace_size() bytes;
 *                       with less or NULL the call takes the fp32 CUDA-core chunk kernel.
 *                       Contents on entry do not matter; concurrent calls must use distinct
 *                       workspaces.
 * Every sequence starts from its own S0/P0 (chunks restart at sequence starts). */
kdn_status_t kdn_forward_chunkwise(const kdn_problem_t *p,
                                   const void *q, const void *k, const void *v,
                                   const void *alpha, const void *sigma, const void *r,
                                   const float *S0, const float *P0,
                                   void *o, float *S_out, float *P_out,
                                   void *workspace, size_t workspace_bytes, void *stream);

/* One autoregressive step for N independent sequences (KDA article, "fused
 * recurrent kernel" regime): predict, gain, write, readout and uncertainty update
 * of one token, with the state read from and written back to HBM in place.
 *  q, k, alpha, sigma : device [N, H, d_k] (in_dtype);  v : device [N, H, d_v];  r : device [N, H]
 *  S                  : device fp32 [N, H, d_k, d_v], updated in place
 *  P                  : device fp32 [N, H, d_k], updated in place
 *  o                  : device [N, H, d_v] (in_dtype) */
kdn_status_t kdn_decode_step(int N, int H, int d_k, int d_v, kdn_dtype_t in_dtype, float mu,
                             const void *q, const void *k, const void *v,
                             const void *alpha, const void *sigma, const void *r,
                             float *S, float *P, void *o, void *stream);

/* Several autoregressive tokens per launch for N independent sequences (multi-token /
 * speculative decode): the n_tokens tokens of each sequence are applied in order to the
 * state, which is read once and written back once in place -- the state traffic of one
 * step is shared by n_tokens tokens (KDA article, fused recurrent regime; its closing
 * remark pairs chunkwise processing with speculative decoding).
 *  q, k, alpha, sigma : device [N, n_tokens, H, d_k] (in_dtype);  v : device [N, n_tokens, H, d_v]
 *  r                  : device [N, n_tokens, H];  o : device [N, n_tokens, H, d_v] (in_dtype)
 *  S, P               : device fp32 [N, H, d_k, d_v], [N, H, d_k], updated in place
 * n_tokens == 1 is kdn_decode_step with the token axis made explicit. */
kdn_status_t kdn_decode_tokens(int N, int n_tokens, int H, int d_k, int d_v, kdn_dtype_t in_dtype, float mu,
                               const void *q, const void *k, const void *v,
                               const void *alpha, const void *sigma, const void *r,
                               float *S, float *P, void *o, void *stream);

/* kdn_decode_tokens() for the isotropic variant: P is device fp32 [N, H] (one
 * uncertainty per head), updated in place; everything else as kdn_decode_tokens(). */
kdn_status_t kdn_decode_tokens_iso(int N, int n_tokens, int H, int d_k, int d_v, kdn_dtype_t in_dtype, float mu,
                                   const void *q, const void *k, const void *v,
                                   const void *alpha, const void *sigma, const void *r,
                                   float *S, float *P, void *o, void *stream);

/* The uncertainty / gain scan on its own (explainer, closing paragraph of "各向同性近似":
 * the uncertainty recursion is a Moebius map whose 2x2 matrices compose, so it runs
 * as an associative scan).  Independent of the memory S.
 *  k, alpha, sigma : device [B, T, H, d_k];  r : device [B, T, H]   (in_dtype)
 *  P0              : device fp32 [N, H, d_k] or NULL (ones)
 *  g               : device fp32 [B, T, H, d_k], the gain of every token, or NULL
 *  beta_eff        : device fp32 [B, T, H], k_t^T g_t (the effective write strength), or NULL
 *  P_out           : device fp32 [N, H, d_k], uncertainty after the last token, or NULL
 *  workspace       : device, >= kdn_workspace_size() bytes, 256-byte aligned; its contents
 *                    on entry do not matter (the call resets what it uses).
 * Single pass: every 64-token chunk composes its tokens' maps, publishes the composite,
 * and takes its starting uncertainty from its predecessors by decoupled look-back
 * (bounded waits; a wait that gives up records KDN_ERR_TIMEOUT).  Concurrent calls
 * must use distinct workspaces.  Diagonal variant only (isotropic: KDN_ERR_UNSUPPORTED). */
kdn_status_t kdn_gain_scan(const kdn_problem_t *p,
                           const void *k, const void *alpha, const void *sigma, const void *r,
                           const float *P0, float *g, float *beta_eff, float *P_out,
                           void *workspace, size_t workspace_bytes, void *stream);

/* kdn_gain_scan() for callers that cannot allocate device memory at call time -- for
 * example a plugin hosted by a framework that owns every device buffer and exposes no
 * allocator, or a serving loop that bans cudaMalloc/cudaFree after start-up (cudaFree
 * synchronises the device).  The paper has no counterpart: this entry point only changes
 * where the scan keeps its scratch.
 *  Arguments: as kdn_gain_scan() without the workspace; inputs and outputs stay the
 *  caller's.  Scratch: a fixed 32 MiB device array inside the library, one per GPU that
 *  loads it, held until the process exits.  A problem whose scan needs more (more than
 *  about 8000 (chunk of 64 tokens, sequence x head) pairs at d_k = 128) returns
 *  KDN_ERR_UNSUPPORTED before anything runs.
 *  Set-up: the first call on a device looks up that device's array address (with the
 *  device current); make that first call before any stream capture.  No cudaMalloc,
 *  cudaFree or allocating library routine is called.
 *  Sharing: every call uses the same array and leaves its last contents there (each call
 *  clears the part that must start at zero).  Calls that overlap on the GPU -- on
 *  different streams, or from different host threads -- race on the array and must be
 *  ordered by the caller. */
kdn_status_t kdn_gain_scan_noalloc(const kdn_problem_t *p,
                                   const void *k, const void *alpha, const void *sigma, const void *r,
                                   const float *P0, float *g, float *beta_eff, float *P_out, void *stream);

/* Backward pass of the KDN, for training (KDA article, "chunkwise" section: the chunkwise
 * regime serves training; explainer "对角近似" and "各向同性近似" for the recurrences
 * differentiated).
 * Computes the gradients of  L = <o, d_o> + <S_T, dS_T> + <P_T, dP_T>, where o, S_T and P_T are
 * what kdn_forward_chunkwise() returns for the same problem and inputs, with respect to every
 * input: the vector-Jacobian products of one training step.
 *  p                  : as for the forward, either variant (`chunk` is ignored; `max_seqlen`, for
 *                       packed sequences, bounds the chunk-parallel work lists as for the forward)
 *  q ... P0           : the forward's inputs, same layouts (S0 / P0 NULL = 0 / 1; P0 [N, H] isotropic)
 *  d_o                : device [B, T, H, d_v] (in_dtype), gradient of L with respect to o
 *  dS_T, dP_T         : device fp32 [N, H, d_k, d_v], [N, H, d_k] ([N, H] isotropic), gradients
 *                       with respect to the final S and P, or NULL (zero)
 *  dq, dk, dalpha, dsigma : device fp32 [B, T, H, d_k];  dv : device fp32 [B, T, H, d_v]
 *  dr                 : device fp32 [B, T, H]
 *  dS0, dP0           : device fp32 [N, H, d_k, d_v], [N, H, d_k] ([N, H] isotropic), or NULL (not written)
 *  workspace          : device, >= kdn_backward_workspace_size() bytes, 256-byte aligned
 *                       (contents on entry do not matter; distinct per concurrent call).
 * Method: the uncertainty forward is taped (P before each token, den, g), the memory forward
 * is checkpointed every 16 tokens, and the reverse sweep recomputes each chunk from its
 * checkpoint (the state before every token is re-stepped forward, never reconstructed by
 * dividing by alpha); fp32 CUDA-core arithmetic.  The uncertainty tape (bf16, d_k = 128) and
 * the uncertainty adjoint (diagonal variant) run as chunk-parallel scans with decoupled
 * look-back whenever their work lists (N x H x the chunks of the longest sequence) fit the
 * checkpoint region, else as one serial walk per (sequence, head); both give the same result
 * to fp32 rounding.  The isotropic variant's scalar uncertainty walks run one warp per
 * (sequence, head) between per-token parallel launches.  The d_v column blocks of a (sequence, head)
 * add their shares of the sums over d_v with atomic adds, so the last bits of every gradient
 * except dv and dS0 can differ from run to run.  Workspace: about 7.0 KB per token and head
 * at d_k = d_v = 128.  Every pointer 16-byte aligned.  Outputs may not alias inputs.
 * Asynchronous on `stream`; errors as for the forward. */
kdn_status_t kdn_backward_workspace_size(const kdn_problem_t *p, size_t *bytes);
kdn_status_t kdn_backward(const kdn_problem_t *p,
                          const void *q, const void *k, const void *v,
                          const void *alpha, const void *sigma, const void *r,
                          const float *S0, const float *P0,
                          const void *d_o, const float *dS_T, const float *dP_T,
                          float *dq, float *dk, float *dv, float *dalpha, float *dsigma, float *dr,
                          float *dS0, float *dP0,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Which execution path kdn_forward_chunkwise() takes for `p` (host-only; no CUDA call
 * besides resolving the driver's tensor-map encoder once): 0 token-serial recurrence,
 * 1 fp32 CUDA-core chunk kernel, 3 the tcgen05 tensor-core path in two launches (taken when
 * the call also gets a workspace of kdn_workspace_size() bytes; without one such a problem
 * runs path 1); -1 if `p` is invalid.  (2 is not returned.) */
int kdn_execution_path(const kdn_problem_t *p);

/* Self-test of failure detection: launches one kernel whose two bounded waits -- a poll of a
 * device word that nothing writes (the look-back's wait) and an mbarrier phase that nothing
 * completes (the tensor-core kernels' wait) -- each give up after `limit_cycles` SM clock cycles
 * (1e3 .. 4e9; 2e6 is about a millisecond) and record KDN_ERR_TIMEOUT in the device error word.
 * Nothing faults or hangs; kdn_last_device_error() then reports KDN_ERR_TIMEOUT and clears it.
 * The method has no counterpart on the pages: this checks the library's own error path. */
kdn_status_t kdn_selftest_bounded_wait(long long limit_cycles, void *stream);

/* Synchronises `stream`, then returns and clears the device error word
 * (KDN_ERR_TIMEOUT or KDN_ERR_INVALID_ARG if a kernel recorded one, else KDN_OK). */
kdn_status_t kdn_last_device_error(void *stream);

/* Static description of a status code. */
const char *kdn_status_string(kdn_status_t s);

/* Library version, e.g. "kdn-b200 0.1 sm_100a". */
const char *kdn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KDN_H_ */
