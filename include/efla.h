/*
 * efla.h - C ABI of the EFLA (Exact Flow Linear Attention) token mixer for
 * NVIDIA B200 (sm_100a).
 *
 * The method ("Exact Flow Linear Attention: Exact Solution from
 * Continuous-Time Dynamics", papernotes.org summary of arXiv 2512.12602):
 *
 *   lambda_t = ||k_t||^2                                   (关键设计 2)
 *   alpha_t  = (1 - e^{-beta_t lambda_t}) / lambda_t       (关键设计 2)
 *            = -expm1(-beta_t lc) / lc, lc = max(lambda_t, 1e-12), in fp32
 *                                                          (损失函数 / 训练策略)
 *   S_t      = (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T
 *   o_t      = S_t^T q_t                (post-update state; 整体框架 flowchart)
 *
 * EFLA_MODE_EULER replaces alpha_t by beta_t, which is the DeltaNet
 * (explicit Euler) update of section 关键设计 1; everything else is shared.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The
 *    library allocates nothing; efla_chunk_fwd takes caller-owned scratch.
 *  - Layouts are dense row-major (C-contiguous):
 *      q, k      [B][H][L][d_k]       v, o      [B][H][L][d_v]
 *      beta, alpha, lambda [B][H][L]  (fp32)
 *      S0, S_L, S          [B][H][d_k][d_v] (fp32)
 *    For decode L is absent: q,k [B][H][d_k], v,o [B][H][d_v], beta [B][H].
 *  - q, k and v share one storage dtype (`dtype`); the output o has its
 *    own dtype (`o_dtype`, fp32 or bf16); beta, alpha, lambda and every
 *    state are fp32.  Arithmetic is fp32 throughout (the bf16 chunk path
 *    feeds bf16 operands to tensor-core products that accumulate in fp32;
 *    the state is kept in fp32).  A bf16 o adds its own rounding (up to
 *    2^-8 relative per element) on top of the arithmetic error.
 *  - Supported head sizes: d_k == d_v in {32, 64, 128}; anything else
 *    returns EFLA_ERR_UNSUPPORTED.  B, H >= 0; L >= 0 (L = 0 copies S0 to
 *    S_L); L need not be a multiple of the internal chunk size.
 *  - Every pointer must be 16-byte aligned (EFLA_ERR_ALIGN otherwise).
 *  - Validation is synchronous and happens before anything is enqueued; on
 *    any error nothing is launched.  Work is enqueued on `stream` and runs
 *    asynchronously.  Launch failures return EFLA_ERR_CUDA.  Faults that
 *    happen later on the device surface through efla_last_error() or the
 *    caller's next synchronising CUDA call.
 *  - beta may be any real number; NaN and Inf propagate into the outputs
 *    and are not reported as errors.
 *  - The calls are thread-safe and keep no host state between calls except
 *    the sticky device error word read by efla_last_error().
 */
#ifndef EFLA_H
#define EFLA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream.  NULL selects the legacy default stream. */
typedef struct CUstream_st *efla_stream_t;

typedef enum {
    EFLA_OK = 0,
    EFLA_ERR_NULL = 1,        /* a required pointer is NULL                        */
    EFLA_ERR_SHAPE = 2,       /* a negative size, or an overflowing element count  */
    EFLA_ERR_DTYPE = 3,       /* unknown efla_dtype_t / efla_mode_t                */
    EFLA_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned                  */
    EFLA_ERR_UNSUPPORTED = 5, /* head size outside {32,64,128} or d_k != d_v       */
    EFLA_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed       */
    EFLA_ERR_TIMEOUT = 7,     /* a device-side bounded wait gave up (sticky word)  */
    EFLA_ERR_WORKSPACE = 8,   /* workspace missing or smaller than required        */
    EFLA_ERR_ALIAS = 9        /* an output overlaps an input it must not overlap   */
} efla_status_t;

typedef enum { EFLA_F32 = 0, EFLA_BF16 = 1 } efla_dtype_t;

typedef enum {
    EFLA_MODE_EXACT = 0, /* exact-flow gate alpha_t (EFLA)                 */
    EFLA_MODE_EULER = 1  /* alpha_t = beta_t (DeltaNet / explicit Euler)   */
} efla_mode_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char *efla_status_string(efla_status_t status);

/* Library version as 10000*major + 100*minor + patch. */
int efla_version(void);

/*
 * Sticky device error word of the current device.  Synchronises the
 * current device, returns EFLA_ERR_TIMEOUT if a kernel's bounded wait gave
 * up since the last call (and clears the word), EFLA_ERR_CUDA if the CUDA
 * context holds an error, else EFLA_OK.
 */
efla_status_t efla_last_error(void);

/*
 * Diagnostic: launch one CTA that waits on an mbarrier nothing ever arrives
 * on, through the same clock-bounded wait the prefill kernel uses, with a
 * limit of `limit_cycles` SM clock cycles.  The wait gives up, the kernel
 * sets the sticky error word and returns; the next efla_last_error()
 * reports EFLA_ERR_TIMEOUT and the CUDA context stays usable.  Exists so the
 * failure path can be tested without faulting or hanging a GPU.
 */
efla_status_t efla_diag_wait_timeout(long long limit_cycles, efla_stream_t stream);

/*
 * efla_gate - the exact-flow gate (关键设计 2; numerics per 损失函数 /
 * 训练策略): for every row t of k,
 *     lambda[t] = sum_i k[t][i]^2                (fp32 accumulation, unclamped)
 *     alpha[t]  = -expm1(-beta[t]*lc)/lc,  lc = max(lambda[t], 1e-12)
 * (alpha[t] = beta[t] in EFLA_MODE_EULER).
 *   k      [B][H][L][d_k], dtype `dtype`            (input)
 *   beta   [B][H][L] fp32                            (input)
 *   alpha  [B][H][L] fp32                            (output)
 *   lambda [B][H][L] fp32                            (output; may be NULL)
 * alpha must not overlap k or beta.
 */
efla_status_t efla_gate(const void *k, efla_dtype_t dtype, efla_mode_t mode,
                        const float *beta, float *alpha, float *lambda,
                        int B, int H, int L, int d_k, efla_stream_t stream);

/*
 * Bytes of scratch efla_chunk_fwd needs for these sizes (0 if none).  The
 * value depends only on the arguments.
 */
size_t efla_chunk_fwd_workspace_size(efla_dtype_t dtype, int B, int H, int L,
                                     int d_k, int d_v);

/*
 * efla_chunk_fwd - prefill over a whole sequence: runs the recurrence above
 * for t = 0..L-1 from S0 and writes every o_t and the final state.  It
 * evaluates the recurrence chunk by chunk in the UT form of the chunked
 * scheme the pages cite (整体框架: "WY / UT" chunk-parallel products):
 *     A = strictly-lower(diag(alpha) K K^T),  T = (I + A)^{-1},
 *     W = T diag(alpha) K,  U = T diag(alpha) V,
 *     D = U - W S,  O = Q S + lower-incl-diag(Q K^T) D,  S <- S + K^T D,
 * which equals the token-by-token recurrence up to rounding.
 *   q, k  [B][H][L][d_k]   v [B][H][L][d_v]   dtype `dtype`   (inputs)
 *   beta  [B][H][L] fp32                                        (input)
 *   S0    [B][H][d_k][d_v] fp32, or NULL for the zero state     (input)
 *   o     [B][H][L][d_v] dtype `o_dtype`                        (output)
 *   S_L   [B][H][d_k][d_v] fp32, or NULL if not wanted          (output)
 *   workspace / workspace_bytes: caller-owned device scratch of at least
 *     efla_chunk_fwd_workspace_size(...) bytes (may be NULL when that is 0);
 *     its contents on entry are ignored and on exit undefined.
 * S_L may be the same pointer as S0 (in-place state update).  o must not
 * overlap any input; S_L must not overlap q, k, v, beta or o.
 */
efla_status_t efla_chunk_fwd(const void *q, const void *k, const void *v,
                             efla_dtype_t dtype, efla_mode_t mode,
                             const float *beta, const float *S0, void *o,
                             efla_dtype_t o_dtype, float *S_L, int B, int H,
                             int L, int d_k, int d_v,
                             void *workspace, size_t workspace_bytes,
                             efla_stream_t stream);

/*
 * efla_decode_step - one token of the recurrence for B*H independent
 * states, updated in place:
 *     S <- (I - alpha k k^T) S + alpha k v^T,   o = S^T q  (updated S)
 *   q, k [B][H][d_k]   v [B][H][d_v]   dtype `dtype`   (inputs)
 *   beta [B][H] fp32                                    (input)
 *   S    [B][H][d_k][d_v] fp32                          (input/output)
 *   o    [B][H][d_v] dtype `o_dtype`                    (output)
 * o must not overlap S or any input.
 */
efla_status_t efla_decode_step(const void *q, const void *k, const void *v,
                               efla_dtype_t dtype, efla_mode_t mode,
                               const float *beta, float *S, void *o,
                               efla_dtype_t o_dtype, int B, int H, int d_k,
                               int d_v, efla_stream_t stream);

/*
 * efla_prefill_bwd - reverse-mode derivative of efla_chunk_fwd.  The pages
 * train with this mixer but print no backward; it is derived from the
 * recurrence of 关键设计 2 (S_t = S_{t-1} + alpha_t k_t e_t^T with
 * e_t = v_t - S_{t-1}^T k_t, o_t = S_t^T q_t) and the gate of 关键设计 2 /
 * 损失函数 (d alpha/d beta = e^{-beta lambda}, d alpha/d lambda =
 * (beta lambda e^{-beta lambda} - (1 - e^{-beta lambda})) / lambda^2, zero
 * where lambda <= 1e-12).  For the loss sum(dO * o) + sum(dSL * S_L) it
 * returns the gradients with respect to every input:
 *   q, k [B][H][L][d]  v [B][H][L][d]  dtype `dtype`    (forward inputs)
 *   beta [B][H][L] fp32, S0 [B][H][d][d] fp32 or NULL (zero state)
 *   dO [B][H][L][d] fp32; dSL [B][H][d][d] fp32 or NULL (zero)
 *   dq, dk, dv [B][H][L][d] fp32; dbeta [B][H][L] fp32; dS0 [B][H][d][d] fp32
 *   workspace / workspace_bytes: caller-owned device scratch of at least
 *     efla_prefill_bwd_workspace_size(...) bytes.
 * d = d_k = d_v in {32, 64, 128}.  Exact fp32 arithmetic, one CTA per (b,h)
 * walking the sequence three times (forward, backward, forward).  Outputs
 * must not overlap inputs or each other.  Asynchronous on `stream`.
 */
size_t efla_prefill_bwd_workspace_size(int B, int H, int L, int d_k, int d_v);
efla_status_t efla_prefill_bwd(const void *q, const void *k, const void *v, efla_dtype_t dtype, efla_mode_t mode,
                               const float *beta, const float *S0, const float *dO, const float *dSL,
                               float *dq, float *dk, float *dv, float *dbeta, float *dS0,
                               int B, int H, int L, int d_k, int d_v,
                               void *workspace, size_t workspace_bytes, efla_stream_t stream);

/*
 * efla_state_affine - one step of composing the state maps of consecutive
 * sequence segments: for every (b, h),
 *     out = (SI - SZ) X + SZ
 * The state after a segment is affine in the state before it (the
 * recurrence of 关键设计 2 is linear in S): S_out = M S_in + S_Z, where
 * S_Z is the final state from S_in = 0, S_I the final state from the
 * identity and M = S_I - S_Z.  With SI = S_I, SZ = S_Z and X a segment's
 * true initial state, `out` is the next segment's true initial state.  The
 * pages have no such call; sequence-parallel prefill (across GPUs or SMs)
 * is built on it.
 *   SI, SZ, X, out [B][H][d][d] fp32, d = d_k = d_v in {32, 64, 128}.
 *   out must not overlap SI, SZ or X.  Asynchronous on `stream`.
 */
efla_status_t efla_state_affine(const float *SI, const float *SZ, const float *X, float *out,
                                int B, int H, int d, efla_stream_t stream);

/*
 * efla_chunk_fwd_noalloc - the same prefill as efla_chunk_fwd, for callers
 * that cannot allocate device memory.  The pages describe no such call; it
 * exists for this library's users.  Some hosts (inference engines and
 * plugins that budget every byte of GPU memory through their own pool, or
 * latency-critical loops where cudaMalloc/cudaFree would synchronise the
 * device) cannot hand this library a scratch buffer or let it allocate one.
 * This entry point takes no workspace and allocates nothing: its scratch is
 * a fixed array of EFLA_NOALLOC_SCRATCH_BYTES (32 MiB) that the library
 * places in device memory of every GPU on which it is loaded and keeps until
 * the process exits.
 *   Arguments, layouts and results are those of efla_chunk_fwd.  It always
 *   runs the CUDA-core (exact fp32) chunked kernels, for every dtype and head
 *   size.  Problems whose scratch would not fit
 *   (efla_chunk_fwd_workspace_size_simt > EFLA_NOALLOC_SCRATCH_BYTES, e.g.
 *   more than 409 head-chunks of 64 tokens at d = 128) return
 *   EFLA_ERR_WORKSPACE before anything is launched.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before capturing a stream
 *   into a CUDA graph.
 *   Every call on a device shares the one array and leaves its contents
 *   behind; nothing in it needs to start zeroed.  Calls whose kernels overlap
 *   on the GPU (other streams, other host threads) race on it: serialise them.
 */
#define EFLA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* Scratch bytes the CUDA-core chunked kernels need for these sizes. */
size_t efla_chunk_fwd_workspace_size_simt(int B, int H, int L, int d_k, int d_v);

efla_status_t efla_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                     efla_dtype_t dtype, efla_mode_t mode,
                                     const float *beta, const float *S0,
                                     void *o, efla_dtype_t o_dtype, float *S_L,
                                     int B, int H, int L, int d_k, int d_v,
                                     efla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EFLA_H */
