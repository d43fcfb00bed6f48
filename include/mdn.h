/*
 * mdn.h -- C ABI of libmdn: the Momentum DeltaNet (MDN) chunkwise forward
 * pass and single-token decode step on NVIDIA B200 (sm_100a).
 *
 * The method ("MDN: Parallelizing Stepwise Momentum for Delta Linear
 * Attention", arXiv 2605.05838; paper.rainbus.top summary, steps 1-7;
 * ijyty.com article, sections 3-6).  Per (batch b, head h), with fast weight S
 * and momentum M, both d_k x d_v fp32, and alpha_t = exp(alpha_log_t),
 * mu_t = exp(mu_log_t):
 *
 *     p_t      = alpha_t k_t
 *     vtilde_t = v_t - S_{t-1}^T p_t                   (corrected value)
 *     M_t      = mu_t M_{t-1} - eta_t k_t vtilde_t^T
 *     S_t      = alpha_t S_{t-1} - beta_t M_t
 *     o_t      = S_t^T qhat_t,   qhat_t = q_t - d k_t  (output correction)
 *
 * mdn_chunk_fwd computes o, vtilde and the final (S_T, M_T) for a whole
 * sequence with the chunkwise-parallel form (summary, step 4); mdn_step runs
 * the recurrence for one token (the decoding form, ijyty.com section 6).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates or frees memory; scratch space is passed in explicitly.
 *  - Layouts are dense, row-major, without padding:
 *        q, k, v, o, vtilde : [B, T, H, d]        (mdn_step: [B, H, d])
 *        gates              : [B, T, H] fp32      (mdn_step: [B, H])
 *        S0, M0, S_T, M_T, S, M : [B, H, d_k, d_v] fp32, row index over d_k
 *    q, k, v, o and vtilde use the element type `in_dtype`; everything else
 *    is fp32.  Alignment: mdn_chunk_fwd wants q, k, v, o, vtilde and the
 *    states 16-byte aligned and the workspace 256-byte aligned; mdn_step wants
 *    S and M 16-byte aligned; every other pointer needs only the alignment of
 *    its element type (la, lm, lc, b of mdn_chunk_gate_prep: 8 bytes).
 *  - Work is enqueued on `stream` (NULL = the legacy default stream) and runs
 *    asynchronously; the call returns once the work is enqueued.
 *  - Arguments are validated on the host before anything is enqueued; a call
 *    that fails validation writes nothing.  No entry point aborts or exits.
 *  - Gates are taken as given: the library applies no clamp or activation.
 *  - Calls that share output or scratch buffers must be ordered by the caller.
 */
#ifndef MDN_H
#define MDN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *mdn_stream_t;

typedef enum {
    MDN_OK = 0,
    MDN_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misalignment, bad size  */
    MDN_ERR_UNSUPPORTED = 2,  /* valid but outside what the library supports (d, C, dtype) */
    MDN_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed                 */
    MDN_ERR_NONFINITE = 4,    /* MDN_CHECK_FINITE found a NaN/Inf in an output        */
    MDN_ERR_TIMEOUT = 5       /* a bounded on-device wait ran out (kernel gave up)    */
} mdn_status;

typedef enum {
    MDN_F32 = 0,   /* IEEE fp32 */
    MDN_BF16 = 1   /* bfloat16  */
} mdn_dtype;

/* Flags for mdn_chunk_fwd. */
#define MDN_CHECK_FINITE 0x1  /* after the pass, synchronise `stream` and return
                                 MDN_ERR_NONFINITE if o, vtilde, S_T or M_T holds
                                 a NaN or Inf, and MDN_ERR_TIMEOUT if a kernel
                                 reported a wait that ran out */
#define MDN_FORCE_SIMT   0x2  /* use the fp32 CUDA-core kernels even for bf16 input */
#define MDN_SLICE32      0x4  /* tensor-core path: the inter-chunk kernel gives each CTA
                                 32 columns of d_v (four CTAs per head) */
#define MDN_SLICE64      0x8  /* ... 64 columns (two CTAs per head) */
#define MDN_SLICE128     0x10 /* ... all 128 columns (one CTA per head).  None of the
                                 three: 32 when B*H*4 CTAs fit on the SMs at once,
                                 else 128 (packed sequences: 32 up to four waves, else
                                 64).  At most one; every width computes the same
                                 result; the flags exist for tuning and testing. */
#define MDN_TEST_NO_INTRA 0x100 /* testing the failure path only: the tensor-core
                                 path does not launch its intra-chunk kernel, so the
                                 inter-chunk kernel's wait for each chunk's operands
                                 runs out (after about 1 s), its CTAs stop cleanly,
                                 and with MDN_CHECK_FINITE the call returns
                                 MDN_ERR_TIMEOUT.  The outputs are not written. */

/* Version of this ABI (incremented on any incompatible change). */
int mdn_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *mdn_status_string(mdn_status status);

/*
 * The CUDA error behind the last MDN_ERR_CUDA that a call returned on the
 * calling thread: "<name> (<code>): <description>".  The string belongs to
 * the library and stays valid until the next failing call on this thread.
 * Before any failure it says that no error was recorded.  Never NULL.
 */
const char *mdn_last_cuda_error(void);

/*
 * Bytes of device scratch that mdn_chunk_fwd needs for these sizes with
 * flags = 0, or 0 if the sizes are invalid or unsupported.  Pure host
 * function.  The scratch is sized for the path the call takes: bf16 input
 * with d = 128 runs on the tensor cores and needs about 1 KB per chunk of C
 * tokens of each head (the per-chunk operands of the sequential kernel); every
 * other case runs on CUDA cores and needs about (C + 4 d + 4) x 4 bytes per
 * token and head.
 */
size_t mdn_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int C,
                                    mdn_dtype in_dtype);

/*
 * As mdn_chunk_fwd_workspace_size, for the path that `flags` selects (with
 * MDN_FORCE_SIMT, bf16 d = 128 input takes the CUDA-core path and needs its
 * larger scratch).  A workspace sized for flags = 0 is too small for such a
 * call, which then returns MDN_ERR_INVALID_ARG.  Pure host function.
 */
size_t mdn_chunk_fwd_workspace_size_flags(int B, int T, int H, int dk, int dv, int C,
                                          mdn_dtype in_dtype, int flags);

/*
 * What the kernels of the last mdn_chunk_fwd or mdn_chunk_fwd_varlen call on
 * this workspace recorded on the device, for callers that do not pass
 * MDN_CHECK_FINITE (which makes the pass itself synchronise and report).  Synchronises `stream` (the stream that call used)
 * and returns MDN_OK, MDN_ERR_TIMEOUT (a bounded device wait ran out: the
 * call's outputs are undefined), MDN_ERR_INVALID_ARG (packed sequences only:
 * cu_seqlens broke its rules, every sequence was treated as empty) or
 * MDN_ERR_NONFINITE (only after a call with MDN_CHECK_FINITE).  Every chunk
 * pass clears these words before its kernels run.  (mdn_chunk_fwd_noalloc has
 * no caller workspace; pass it MDN_CHECK_FINITE to have it report.)
 *   workspace   the workspace pointer passed to that call (256-byte aligned).
 * Errors: MDN_ERR_INVALID_ARG (null or unaligned workspace), MDN_ERR_CUDA.
 */
mdn_status mdn_chunk_fwd_status(const void *workspace, mdn_stream_t stream);

/*
 * Chunkwise forward pass over a whole sequence (summary, steps 2-5; the
 * chunk form Vtilde = U - Y S + Z M, U = T V, Y = T Diag(alphabar) P,
 * Z = T Diag(b) P, T = (I + P K^T o Gamma-)^{-1}, with o from the reordered
 * sum (Qhat K^T o Gamma) Vtilde plus the carried-state term).
 *
 *   q, k, v     [B,T,H,d] in_dtype.  d_k = d_v = d.
 *   alpha_log, mu_log, beta, eta  [B,T,H] fp32.
 *   d_corr      the scalar d of qhat = q - d k.
 *   S0, M0      [B,H,d,d] fp32 entering states; either may be NULL (zeros).
 *   C           chunk length; the library supports C = 64.
 *   o, vtilde   [B,T,H,d] in_dtype outputs (vtilde is the materialised Vtilde).
 *   S_T, M_T    [B,H,d,d] fp32 outputs: the states after token T.  They may
 *               alias S0 / M0 (read before written, per head).
 *   workspace   device scratch of at least
 *               mdn_chunk_fwd_workspace_size_flags(..., flags) bytes (for
 *               flags without MDN_FORCE_SIMT, mdn_chunk_fwd_workspace_size),
 *               256-byte aligned; its contents on entry do not matter.
 *   flags       0 or MDN_CHECK_FINITE | MDN_FORCE_SIMT, plus at most one of
 *               MDN_SLICE32 / MDN_SLICE64 / MDN_SLICE128 (and MDN_TEST_NO_INTRA
 *               in tests).
 *
 * Support: d in {64, 128}, C = 64, any T >= 0 (a short last chunk is handled
 * as if padded with steps that leave S and M unchanged), B, H >= 0 with
 * B*H*ceil(T/C) < 2^31.  T = 0 copies S0, M0 (or zeros) to S_T, M_T.
 * Errors: MDN_ERR_INVALID_ARG (null required pointer, negative size,
 * unaligned pointer, too-small workspace), MDN_ERR_UNSUPPORTED (d, C or dtype
 * outside support), MDN_ERR_CUDA (launch failure), and with MDN_CHECK_FINITE
 * also MDN_ERR_NONFINITE / MDN_ERR_TIMEOUT.  Without MDN_CHECK_FINITE an
 * expired device wait (MDN_ERR_TIMEOUT; the outputs are then undefined) is
 * only recorded in the workspace: mdn_chunk_fwd_status reads it.
 *
 * Asynchronous on `stream` (except with MDN_CHECK_FINITE).  Every call first
 * clears the workspace's status words with a small memset.  The bf16 d = 128
 * path then enqueues two kernels, the second
 * launched as the first one's programmatic dependent; the sequence can be
 * captured in a CUDA graph and replayed.  Calls that may run concurrently
 * need separate workspaces.
 */
mdn_status mdn_chunk_fwd(const void *q, const void *k, const void *v, mdn_dtype in_dtype,
                         const float *alpha_log, const float *mu_log,
                         const float *beta, const float *eta, float d_corr,
                         const float *S0, const float *M0,
                         int B, int T, int H, int dk, int dv, int C,
                         void *o, void *vtilde, float *S_T, float *M_T,
                         void *workspace, size_t ws_bytes, int flags,
                         mdn_stream_t stream);

/*
 * Bytes of device scratch that mdn_chunk_bwd needs, or 0 if the sizes are
 * invalid or unsupported.  For bf16 at d = 128 it covers both paths (the
 * tensor-core path needs more than MDN_FORCE_SIMT's).  Pure host function.
 */
size_t mdn_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int C,
                                    mdn_dtype in_dtype);

/*
 * The backward pass of mdn_chunk_fwd: gradients of
 * L = <d_o, o> + <dS_T, S_T> + <dM_T, M_T> with respect to every input.  As
 * the pages train (summary, step 7; article, section 6), it takes the Vtilde
 * that the forward pass saved and rebuilds the chunk-entering states from it,
 * then runs the adjoints of S and M backwards over the chunks and forms every
 * other gradient chunk by chunk.
 *
 *   q .. M0, d_corr   the forward pass's inputs (same layouts and dtypes).
 *   vtilde      [B,T,H,d] in_dtype: the forward pass's vtilde output.
 *   d_o         [B,T,H,d] in_dtype: the cotangent of o.
 *   dS_T, dM_T  [B,H,d,d] fp32 cotangents of S_T, M_T, or NULL (zero).
 *   dq, dk, dv  [B,T,H,d] fp32 outputs.
 *   dalpha_log, dmu_log, dbeta, deta  [B,T,H] fp32 outputs.
 *   dS0, dM0    [B,H,d,d] fp32 outputs (the gradients of the entering states).
 *   workspace   at least mdn_chunk_bwd_workspace_size(...) bytes, 256-byte
 *               aligned (about (4 d^2 + 3 C^2 + 10 C) x 4 bytes per chunk of C
 *               tokens of each head on CUDA cores; on the tensor-core path
 *               the states and adjoints are kept in bf16 (2 d^2 x 2 bytes
 *               less) and the chunk operands add about 260 KB per chunk).
 *   flags       0, or MDN_CHECK_FINITE (synchronise, then report non-finite
 *               outputs or an expired device wait) and/or MDN_FORCE_SIMT (the
 *               CUDA-core kernels for bf16 d = 128 too).
 *
 * bf16 inputs with d = 128 run every product on tcgen05 tensor cores (bf16
 * operands, fp32 accumulation; the reverse chain of the state adjoints as a
 * warp-specialised chain like the forward pass's): seven kernels on `stream`.
 * Every other input combination runs in fp32 on CUDA cores: six kernels, the
 * state rebuild on a side stream of the library that joins back.  Support
 * and errors as mdn_chunk_fwd (T = 0 copies dS_T, dM_T to dS0, dM0).
 * Asynchronous on `stream` (except with MDN_CHECK_FINITE).
 */
mdn_status mdn_chunk_bwd(const void *q, const void *k, const void *v, mdn_dtype in_dtype,
                         const float *alpha_log, const float *mu_log,
                         const float *beta, const float *eta, float d_corr,
                         const float *S0, const float *M0, const void *vtilde,
                         const void *d_o, const float *dS_T, const float *dM_T,
                         int B, int T, int H, int dk, int dv, int C,
                         float *dq, float *dk_out, float *dv_out, float *dalpha_log,
                         float *dmu_log, float *dbeta, float *deta, float *dS0, float *dM0,
                         void *workspace, size_t ws_bytes, int flags, mdn_stream_t stream);

/*
 * Bytes of device scratch that mdn_chunk_fwd_varlen needs, or 0 if the sizes
 * are invalid or unsupported.  Pure host function.
 */
size_t mdn_chunk_fwd_varlen_workspace_size(int N, int total_T, int H, int dk, int dv, int C,
                                           mdn_dtype in_dtype);

/*
 * As mdn_chunk_fwd_varlen_workspace_size, for the path that `flags` selects
 * (see mdn_chunk_fwd_workspace_size_flags).  Pure host function.
 */
size_t mdn_chunk_fwd_varlen_workspace_size_flags(int N, int total_T, int H, int dk, int dv,
                                                 int C, mdn_dtype in_dtype, int flags);

/*
 * mdn_chunk_fwd over N independent sequences of different lengths packed
 * along the token axis.  The pages run one sequence per batch row; this is
 * the plain extension: sequence s is the recurrence above over its own
 * tokens, from its own entering state.
 *
 *   q, k, v, o, vtilde  [total_T,H,d] in_dtype, the sequences back to back.
 *   alpha_log, mu_log, beta, eta  [total_T,H] fp32.
 *   cu_seqlens  DEVICE pointer to N+1 ints: sequence s is tokens
 *               [cu_seqlens[s], cu_seqlens[s+1]); cu_seqlens[0] = 0,
 *               non-decreasing, cu_seqlens[N] = total_T.  Empty sequences
 *               are allowed (their S_T, M_T are S0, M0).
 *   S0, M0      [N,H,d,d] fp32 or NULL (zeros); S_T, M_T  [N,H,d,d] fp32.
 *   workspace   at least mdn_chunk_fwd_varlen_workspace_size(...) bytes,
 *               256-byte aligned.
 *   flags       as mdn_chunk_fwd (without MDN_TEST_NO_INTRA).
 *
 * The inputs are first copied into a chunk-aligned layout (each sequence
 * padded to a whole number of chunks with steps that leave S and M
 * unchanged); the chain kernels write o and vtilde straight back to the
 * packed rows.  cu_seqlens is read on the device only.  If it breaks the
 * rules above, every sequence is treated as empty (S_T = S0, M_T = M0, o and
 * vtilde untouched) and, with MDN_CHECK_FINITE, the call returns
 * MDN_ERR_INVALID_ARG.  Other errors as mdn_chunk_fwd.  Asynchronous on
 * `stream` (except with MDN_CHECK_FINITE).
 */
mdn_status mdn_chunk_fwd_varlen(const void *q, const void *k, const void *v, mdn_dtype in_dtype,
                                const float *alpha_log, const float *mu_log,
                                const float *beta, const float *eta, float d_corr,
                                const int *cu_seqlens, int N, int total_T,
                                const float *S0, const float *M0, int H, int dk, int dv, int C,
                                void *o, void *vtilde, float *S_T, float *M_T,
                                void *workspace, size_t ws_bytes, int flags,
                                mdn_stream_t stream);

/*
 * One decode token for every (b, h): the stepwise recurrence above, applied
 * in place (ijyty.com section 6: decoding runs the recurrence token by token).
 *
 *   q, k, v     [B,H,d] in_dtype;  gates [B,H] fp32;  d_corr as above.
 *   S, M        [B,H,d,d] fp32, read and overwritten with S_t, M_t.
 *   o           [B,H,d] in_dtype output;  vtilde [B,H,d] in_dtype or NULL.
 *
 *   flags       must be 0 (reserved).
 * Support: d in {64, 128}.  Each state element is read once and written once.
 * Errors: MDN_ERR_INVALID_ARG, MDN_ERR_UNSUPPORTED, MDN_ERR_CUDA.
 */
mdn_status mdn_step(const void *q, const void *k, const void *v, mdn_dtype in_dtype,
                    const float *alpha_log, const float *mu_log,
                    const float *beta, const float *eta, float d_corr,
                    float *S, float *M, int B, int H, int dk, int dv,
                    void *o, void *vtilde, int flags, mdn_stream_t stream);

/*
 * mdn_step that also measures how far the fast weight moved:
 *
 *   ds_norm     [B,H] fp32 output: ||S_t - S_{t-1}||_F of each head (the
 *               decoding diagnostic of ijyty.com section 8, which averages it
 *               over steps).  Must not be NULL when B*H > 0.
 *
 * Enqueues a memset of ds_norm, the step (whose blocks add their shares of
 * the squared norm atomically) and an in-place square root.  o, vtilde, S and
 * M come out bit-identical to mdn_step's.  Everything else as mdn_step.
 */
mdn_status mdn_step_delta_norm(const void *q, const void *k, const void *v, mdn_dtype in_dtype,
                               const float *alpha_log, const float *mu_log,
                               const float *beta, const float *eta, float d_corr,
                               float *S, float *M, int B, int H, int dk, int dv,
                               void *o, void *vtilde, float *ds_norm, int flags,
                               mdn_stream_t stream);

/* Activations of eta for mdn_gate_params. */
#define MDN_ETA_TANH     0  /* eta = tanh(x) + 1 (the pages' choice) */
#define MDN_ETA_2SIGMOID 1  /* eta = 2 sigmoid(x) (their ablation, article section 8) */

/*
 * The four gates from raw per-token pre-activations, by the pages' stable
 * parameterisation (summary step 6; ijyty.com sections 5 and 8):
 *
 *   eta       = tanh(x_eta) + 1   (or 2 sigmoid(x_eta), eta_act)
 *   theta     = arctan(eta * s)
 *   alpha_log = log(cos^2(theta) sigmoid(a))
 *   beta      = sin^2(theta) sigmoid(b)
 *   mu_log    = max(log sigmoid(c), mu_log_min)
 *
 *   x_eta, a, b, c   n fp32 pre-activations each (any layout; elementwise).
 *   s                the scale of theta (finite).
 *   mu_log_min       the lower clamp of log mu (finite; the pages use -2, their
 *                    ablations -1.5 .. -1).
 *   alpha_log, mu_log, beta, eta   n fp32 outputs, ready for mdn_chunk_fwd /
 *                    mdn_step.  Outputs may not alias inputs.
 *
 * Pointers 4-byte aligned (16-byte alignment and n % 4 == 0 take a vectorised
 * path).  Errors: MDN_ERR_INVALID_ARG (n < 0, null or unaligned pointer,
 * unknown eta_act, non-finite s or clamp), MDN_ERR_CUDA.
 */
mdn_status mdn_gate_params(const float *x_eta, const float *a, const float *b, const float *c,
                           long long n, float s, float mu_log_min, int eta_act,
                           float *alpha_log, float *mu_log, float *beta, float *eta,
                           mdn_stream_t stream);

/*
 * mdn_chunk_fwd with the gate parameterisation fused into the pass: the four
 * gates are computed from their raw per-token pre-activations (the stable
 * gating of summary step 6 and ijyty.com sections 5 and 8, exactly as
 * mdn_gate_params computes them) inside the kernels that read them, so no
 * gate array is written or read back.
 *
 *   x_eta, a_pre, b_pre, c_pre   [B,T,H] fp32 pre-activations of eta, alpha,
 *                beta and mu (4-byte aligned).
 *   s, mu_log_min, eta_act       as mdn_gate_params (s and the clamp finite;
 *                eta_act MDN_ETA_TANH or MDN_ETA_2SIGMOID).
 * Every other argument, the workspace size (mdn_chunk_fwd_workspace_size...),
 * the support and the errors are those of mdn_chunk_fwd (plus
 * MDN_ERR_INVALID_ARG for a bad eta_act, s or clamp).  The result equals
 * mdn_gate_params followed by mdn_chunk_fwd up to the rounding of the gates.
 */
mdn_status mdn_chunk_fwd_preact(const void *q, const void *k, const void *v, mdn_dtype in_dtype,
                                const float *x_eta, const float *a_pre, const float *b_pre,
                                const float *c_pre, float s, float mu_log_min, int eta_act,
                                float d_corr, const float *S0, const float *M0,
                                int B, int T, int H, int dk, int dv, int C,
                                void *o, void *vtilde, float *S_T, float *M_T,
                                void *workspace, size_t ws_bytes, int flags,
                                mdn_stream_t stream);

/*
 * The chunk coefficients alone (the gate-preparation stage of mdn_chunk_fwd;
 * summary step 5), each cumulative quantity restarting at every chunk start:
 *
 *   la_r = sum_{j<=r} alpha_log_j            lm_r = sum_{j<=r} mu_log_j
 *   lc_r = logcumsumexp_{j<=r}(log beta_j + lm_j - la_j)     (-inf if all beta = 0)
 *   b_r  = exp(la_r + lc_r)                   (= alphabar_r c_r)
 *   gamma_{r,i} = eta_i (alphabar_r / mubar_i)(c_r - c_{i-1})  for i <= r, else 0
 *
 *   la, lm, lc, b   [B,H,NT*C] fp32 outputs, NT = ceil(T/C); positions past T
 *                   hold the values of steps that leave the state unchanged.
 *   gamma           [B,H,NT,C,C] fp32 output, or NULL to skip it.
 * Support: C = 64.  Errors: MDN_ERR_INVALID_ARG, MDN_ERR_UNSUPPORTED, MDN_ERR_CUDA.
 */
mdn_status mdn_chunk_gate_prep(const float *alpha_log, const float *mu_log,
                               const float *beta, const float *eta,
                               int B, int T, int H, int C,
                               float *la, float *lm, float *lc, float *b, float *gamma,
                               mdn_stream_t stream);

/*
 * mdn_chunk_fwd without a caller-supplied workspace.  The paper has no
 * counterpart: this is a deployment aid of this library.
 *
 * Some callers cannot call cudaMalloc or hand out scratch memory: for example
 * a plug-in that runs inside another runtime's execution phase, where that
 * runtime owns all device memory and forbids allocation there, or a
 * latency-critical loop that cannot afford cudaMalloc's implicit device-wide
 * synchronisation.  Such callers still own and pass q, k, v, the gates, the
 * states and the outputs; only the scratch space comes from the library.
 *
 * The scratch is one fixed array of 64 MiB in device memory per GPU, created
 * when the library is loaded on that GPU and held until the process exits.
 * Arguments and results are exactly those of mdn_chunk_fwd (minus workspace
 * and ws_bytes).  Sizes whose scratch need,
 * mdn_chunk_fwd_workspace_size_flags(..., flags), exceeds 64 MiB are rejected
 * with MDN_ERR_UNSUPPORTED before anything runs (on the tensor-core path that
 * is about 63,000 chunks of 64 tokens, e.g. B*H = 32 heads of T = 120,000);
 * invalid or unsupported arguments get mdn_chunk_fwd's own error, also
 * before any device work.
 *
 * - The scratch of the CURRENT device is used; `stream` must belong to it.
 * - The first call on a device looks up the array's device address (a
 *   one-time set-up, no allocation); make that first call before any stream
 *   capture is begun on the device.
 * - All calls on a device share the one array and it keeps the last call's
 *   contents.  The pass never relies on them, but calls that overlap on the
 *   GPU (e.g. on two unordered streams) race on the array and corrupt each
 *   other's results: order such calls on one stream or with events.
 * - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
mdn_status mdn_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                 mdn_dtype in_dtype, const float *alpha_log,
                                 const float *mu_log, const float *beta, const float *eta,
                                 float d_corr, const float *S0, const float *M0,
                                 int B, int T, int H, int dk, int dv, int C,
                                 void *o, void *vtilde, float *S_T, float *M_T,
                                 int flags, mdn_stream_t stream);

/*
 * Optional per-kernel timing (no counterpart in the method; a measurement aid).
 * mdn_profile_enable(1) makes every later kernel launch of the library record a
 * CUDA event pair on its launch stream (the events are created on the first
 * enable, so that call needs a current CUDA device); mdn_profile_enable(0)
 * stops recording.  Returns the previous state, or -1 if events could not be
 * created.
 * mdn_profile_read synchronises the recorded events and writes, for up to
 * `capacity` kernel names, the name (static string), total device time in ms
 * and launch count since the last reset; returns the number written, or -1 on
 * a CUDA error.  `reset` != 0 clears the totals afterwards.  Any output array
 * may be NULL.
 */
int mdn_profile_enable(int on);
int mdn_profile_read(int reset, const char **names, double *total_ms,
                     long long *launches, int capacity);

#ifdef __cplusplus
}
#endif
#endif /* MDN_H */
