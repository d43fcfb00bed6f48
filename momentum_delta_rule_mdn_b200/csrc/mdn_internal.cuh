// Internal declarations shared by the libmdn translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gate_math.cuh"
#include "mdn.h"

namespace mdn {

constexpr int kChunk = 64;  // the chunk length C the kernels support

// Element loads/stores in the input dtype, computed in fp32.
__device__ __forceinline__ float ld_elem(const float* p) { return *p; }
__device__ __forceinline__ float ld_elem(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_elem(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_elem(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// log(exp(a) + exp(b)) with -inf handled.
__device__ __forceinline__ float log_add_exp(float a, float b) {
    const float m = fmaxf(a, b);
    if (m == -INFINITY) return -INFINITY;
    return m + log1pf(expf(-fabsf(a - b)));
}

// Inclusive warp scans (lane order) of a sum and of a log-sum-exp.
__device__ __forceinline__ float warp_incl_sum(float x, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    return x;
}
__device__ __forceinline__ float warp_incl_lse(float x, int lane) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x = log_add_exp(x, y);
    }
    return x;
}

// Log-domain coefficients of one chunk of 64 positions, computed by one warp
// (lane owns positions 2*lane and 2*lane+1): from alpha_log, mu_log, beta in
// a[], m[], be[], the chunk-local prefix sums la, lm and lc = logcumsumexp of
// (log beta + lm - la), lc = -inf while every beta so far is 0.
__device__ __forceinline__ void chunk_log_coeffs(const float (&a)[2], const float (&m)[2],
                                                 const float (&be)[2], int lane, float (&la)[2],
                                                 float (&lm)[2], float (&lc)[2]) {
    const float sa = warp_incl_sum(a[0] + a[1], lane);
    const float sm = warp_incl_sum(m[0] + m[1], lane);
    float pa = __shfl_up_sync(0xffffffffu, sa, 1), pm = __shfl_up_sync(0xffffffffu, sm, 1);
    if (lane == 0) pa = pm = 0.f;
    la[0] = pa + a[0];
    la[1] = la[0] + a[1];
    lm[0] = pm + m[0];
    lm[1] = lm[0] + m[1];
    float x[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) x[e] = (be[e] > 0.f) ? logf(be[e]) + lm[e] - la[e] : -INFINITY;
    const float sx = warp_incl_lse(log_add_exp(x[0], x[1]), lane);
    float px = __shfl_up_sync(0xffffffffu, sx, 1);
    if (lane == 0) px = -INFINITY;
    lc[0] = log_add_exp(px, x[0]);
    lc[1] = log_add_exp(lc[0], x[1]);
}

// The gates a chunk pass reads: the four gate arrays [B, T, H]
// (alpha_log, mu_log, beta, eta), or, with pre != 0, four pre-activation
// arrays of the same layout (x_eta, a, b, c) from which every kernel that
// needs a gate computes it as it reads it (the stable parameterisation of
// gate_math.cuh; pre = 1 + the eta activation, s and mu_min its constants).
struct GateSrc {
    const float* g[4];
    int pre;
    float s, mu_min;
};
__device__ __forceinline__ void gates_at(const GateSrc& G, size_t i, float& al, float& ml,
                                         float& be, float& et)
{
    if (G.pre == 0) {
        al = G.g[0][i];
        ml = G.g[1][i];
        be = G.g[2][i];
        et = G.g[3][i];
    } else {
        gate::gate_one_rt(G.pre - 1, G.g[0][i], G.g[1][i], G.g[2][i], G.g[3][i], G.s, G.mu_min,
                          al, ml, be, et);
    }
}

// Everything one mdn_chunk_fwd call needs, with the workspace already carved.
struct ChunkArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha_log;
    const float* mu_log;
    const float* beta;
    const float* eta;
    float dcorr;
    const float* S0;  // may be null
    const float* M0;  // may be null
    int B, T, H, D, NT;  // D = d_k = d_v; NT = ceil(T / C)
    void* o;
    void* vt;
    float* S_T;
    float* M_T;
    // scratch (workspace)
    unsigned* status;  // [0]: non-finite flag, [1]: timeout flag, [2]: bad cu_seqlens
    float* la;         // [B*H, NT*C]
    float* lm;
    float* lc;
    float* bco;
    float* gamma;      // [B*H*NT, C, C]
    float* U;          // [B*H*NT, C, D]
    float* Y;
    float* Z;
    float* Oi;         // [B*H, NT*C, D]  carried-state part of o
    // operands the intra-chunk kernel prepares for the inter-chunk kernel (bf16, per chunk)
    __nv_bfloat16* qhat;  // [B*H*NT, C, D]      qhat = q - d k
    __nv_bfloat16* tat;   // [B*H*NT, 2C, C]     [T; Att T]
    __nv_bfloat16* a2t;   // [B*H*NT, 2D, C]     [K^T Diag(Gamma_C) T; -K^T Diag(w) T]
    unsigned* ready;      // [B*H*NT + 1] chunk operands written (tensor-core path), then the
                          // intra-chunk kernel's work counter; zeroed per call
    float* crec;          // [B*H*NT, 256]       alphabar_r, alpha_r b_{r-1}, b_r, then
                          //                     alphabar_C, b_C, mubar_C
    bool test_no_intra = false;  // failure-path test: skip the intra-chunk kernel
    float* dbg = nullptr;  // diagnostics: if set, CTA 0 dumps its first chunk's intermediates
    // Variable-length mode (cu_chunks != null).  q, k, v and the gates are then
    // the chunk-aligned padded copy, seen as one batch row (B = 1, T = NT*C):
    // sequence s owns padded chunks [cu_chunks[s], cu_chunks[s+1]) and packed
    // tokens [cu_seqlens[s], cu_seqlens[s+1]) of o and vt; S0 .. M_T are
    // [nseq, H, D, D].
    const int* cu_seqlens = nullptr;
    const int* cu_chunks = nullptr;
    int nseq = 0;
    // Work order in variable-length mode: seq_order lists the sequences by
    // decreasing chunk count (chain CTA sh takes sequence seq_order[sh / H]),
    // chunk_order the padded chunks with the longest sequence's first (the
    // intra-chunk kernel's q-th chunk index), so that the longest chain, the
    // pass's critical path, starts first and is fed first.
    const int* seq_order = nullptr;
    const int* chunk_order = nullptr;
    // Fused gate parameterisation: with gate_pre != 0, alpha_log, mu_log,
    // beta and eta above hold the pre-activations x_eta, a, b, c (see GateSrc).
    int gate_pre = 0;
    float gate_s = 1.f, gate_mu_min = -2.f;
    __host__ __device__ GateSrc gates() const {
        return GateSrc{{alpha_log, mu_log, beta, eta}, gate_pre, gate_s, gate_mu_min};
    }
};

// Everything one mdn_chunk_bwd call needs, with the workspace carved.
constexpr int kBwdRec = 6 * kChunk;  // floats of the per-chunk coefficient-adjoint record

// "Chain order" of a 128 x 128 per-chunk matrix on the backward tensor-core
// path (the reverse chain's operands E, F and its results, the adjoints
// leaving each chunk; the state rebuild's increments and the entering
// states): column quarters (4 columns) outermost, then rows, then the 4
// columns of the quarter.  The reverse chain's threads hold one row and
// whole quarters each, 32 consecutive rows per warp, so a warp's float4
// access at one quarter is 512 contiguous bytes.
__device__ __forceinline__ int chain_off(int i, int j) { return (((j >> 2) * 128 + i) << 2) | (j & 3); }
// The row i and column j of the element at chain-order offset o.
__device__ __forceinline__ void chain_ij(int o, int& i, int& j) {
    i = (o >> 2) & 127;
    j = ((o >> 9) << 2) | (o & 3);
}
// A pair of d x d states [X | Y] (d = 128) in bf16 as one 64 KB image: 256
// rows (X's rows, then Y's), K-major, two 64-column panels of 256 rows x 128 B
// with the 128-byte swizzle.  It is the shared-memory form of the B operand
// of products by X^T and Y^T, so a plain bulk copy moves it in.  Byte offset
// of the 16-byte piece holding columns 8g .. 8g + 7 of row `row`:
constexpr uint32_t kStateImgBytes = 2u * 128u * 128u * 2u;
__device__ __forceinline__ uint32_t state_img_off(int row, int g) {
    return (uint32_t)(g >> 3) * 32768u + (uint32_t)row * 128u + ((uint32_t)((g ^ row) & 7) << 4);
}
// The 64 x 128 bf16 rows of one chunk (d = 128) as a K-major operand image:
// two 64-column panels of 64 rows x 128 B, 128-byte swizzle (row r, columns
// 8g .. 8g + 7 at (g >> 3) * 8192 + sw128 offset of (r, g & 7)).
constexpr uint32_t kDyImgBytes = 2u * 64u * 128u;
struct BwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const void* vt;    // Vtilde saved by the forward pass
    const void* dout;  // cotangent of o
    const float* alpha_log;
    const float* mu_log;
    const float* beta;
    const float* eta;
    float dcorr;
    const float* S0;    // may be null
    const float* M0;
    const float* dS_T;  // cotangents of S_T, M_T; may be null
    const float* dM_T;
    int B, T, H, D, NT;
    // scratch
    unsigned* status;  // [0]: non-finite flag, [1]: timeout flag
    float* la;       // [B*H, NT*C] chunk coefficients (gate preparation)
    float* lm;
    float* lc;
    float* bco;
    float* gamma;    // [B*H*NT, C, C]
    float* att;      // [B*H*NT, C, C]  (Qhat K^T) o Gamma (tensor-core path: bf16 in the same place)
    float* tmat;     // [B*H*NT, C, C]  T = (I + A)^{-1} (CUDA-core path; the tensor-core path
                     // keeps T in bf16 in bc_tt)
    float* SS;       // [B*H*NT, 2, D, D]  S, M entering each chunk (CUDA-core path)
    float* dSS;      // [B*H*NT, 2, D, D]  adjoints of S, M leaving each chunk (CUDA-core path)
    // tensor-core path (null otherwise): the same states and adjoints as bf16,
    // each chunk's [S | M] and [dS | dM] as the 64 KB shared-memory image of
    // the state products' B operand (see state_img_off)
    uint8_t* ss_img;   // [B*H*NT][kStateImgBytes]
    uint8_t* dss_img;  // [B*H*NT][kStateImgBytes]
    uint8_t* dy_img;   // [B*H*NT][kDyImgBytes]  dv of each chunk in bf16 (tensor-core path)
    float* crec_bw;  // [B*H*NT, kBwdRec]  coefficient adjoints from the state products
    // chunk-only operands of the tensor-core reverse chain (null on the CUDA-core path)
    __nv_bfloat16* bc_u;   // [B*H*NT, 256, 64]  [-K^T Diag(alphabar) T^T; K^T Diag(D2) T^T]
    __nv_bfloat16* bc_tt;  // [B*H*NT, 64, 64]  T, row-major (the MN-major form of T^T)
    __nv_bfloat16* bc_p;   // [B*H*NT, D/32, 64, 32]  Att^T dO, by 32-column slice (bf16: the
                           // chain rounds dVtilde, of which it is a term, to bf16 anyway)
    __nv_bfloat16* bc_qh;  // [B*H*NT, C, D]  Qhat = Q - d K (bf16, rows of the chunk)
    uint8_t* bc_eo;        // [B*H*NT, D/32, 2, 4096 B]  Diag(alphabar) dO and -Diag(b) dO by
                           // 32-column slice, bf16, each the shared-memory image of the reverse
                           // chain's B operand (MN-major, 64-byte swizzle); with Qhat^T they
                           // give E and F inside the chain
    float* bc_rec;         // [B*H*NT, 256]  Gamma_C, w, then alphabar_C, b_C, mubar_C
    __nv_bfloat16* bc_d;   // [B*H*NT, 2, D, D]  K^T Diag(Gamma_C) Vtilde, K^T Diag(w) Vtilde (chain
                           // order, bf16: increments of the fp32 rebuild)
    // outputs (fp32)
    float* dq;
    float* dk;
    float* dv;
    float* dalpha_log;
    float* dmu_log;
    float* dbeta;
    float* deta;
    float* dS0;
    float* dM0;
};

// One chain of the sequential pass: a state head and its run of chunks.
struct Chain {
    long long sh;      // state head (index into S0 .. M_T, in units of D*D)
    int b, h;          // batch row and head of the inputs
    long long chunk0;  // its first chunk in the per-chunk buffers
    int n0;            // its first chunk in the input rows (token row n0*C of batch row b)
    int nt;            // chunks in the chain
    long long out0;    // token row (of o, vt) of its first token
    int len;           // tokens of the chain written to o, vt
};

// A: ChunkArgs or a kernel's own argument block with the same fields.
template <class A>
__device__ __forceinline__ Chain chain_of(const A& a, long long sh)
{
    Chain c;
    c.sh = sh;
    c.h = (int)(sh % a.H);
    if (a.cu_chunks) {
        const int seq = a.seq_order ? a.seq_order[sh / a.H] : (int)(sh / a.H);
        const int c0 = a.cu_chunks[seq];
        c.sh = (long long)seq * a.H + c.h;  // states are [nseq, H, D, D] in sequence order
        c.b = 0;
        c.chunk0 = (long long)c.h * a.NT + c0;
        c.n0 = c0;
        c.nt = a.cu_chunks[seq + 1] - c0;
        c.out0 = a.cu_seqlens[seq];
        c.len = a.cu_seqlens[seq + 1] - a.cu_seqlens[seq];
    } else {
        c.b = (int)(sh / a.H);
        c.chunk0 = sh * a.NT;
        c.n0 = 0;
        c.nt = a.NT;
        c.out0 = (long long)c.b * a.T;
        c.len = a.T;
    }
    return c;
}

// The sequence that owns padded chunk n (variable-length mode), or -1 for
// the unused chunks past the last sequence.  Empty sequences own no chunk.
__device__ __forceinline__ int varlen_seq_of_chunk(const int* cu_chunks, int nseq, int n)
{
    if (n >= cu_chunks[nseq]) return -1;
    int lo = 0, hi = nseq - 1;  // the last s with cu_chunks[s] <= n
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu_chunks[mid] <= n) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Output rows of input chunk n of batch row b: row r (< valid) of the chunk
// is token row row0 + r of o and vt.
struct ChunkOut {
    long long row0;
    int valid;
};

__device__ __forceinline__ ChunkOut chunk_out(const ChunkArgs& a, int b, int n)
{
    ChunkOut o;
    int rest;
    if (a.cu_chunks) {
        const int seq = varlen_seq_of_chunk(a.cu_chunks, a.nseq, n);
        if (seq < 0) return ChunkOut{0, 0};
        const int local0 = (n - a.cu_chunks[seq]) * kChunk;
        o.row0 = (long long)a.cu_seqlens[seq] + local0;
        rest = a.cu_seqlens[seq + 1] - a.cu_seqlens[seq] - local0;
    } else {
        o.row0 = (long long)b * a.T + (long long)n * kChunk;
        rest = a.T - n * kChunk;
    }
    o.valid = rest < 0 ? 0 : (rest > kChunk ? kChunk : rest);
    return o;
}

// Kernel kinds known to the optional timing facility (profile.cu).
enum KernelKind {
    kGatePrep = 0, kIntraSimt, kInterSimt, kOutputSimt, kStep, kFiniteCheck,
    kChunkTc, kIntraTc, kInterTc, kOutputTc, kGateParams, kVarlen, kBwdPrep, kBwdStates,
    kBwdChain, kBwdStateGrads, kBwdLocal, kBwdChainPrep, kKernelKinds
};
// Record a start event for a launch of kind k on s (returns a slot, or -1 when
// timing is off); prof_end records the matching stop event.
int prof_begin(KernelKind k, cudaStream_t s);
void prof_end(int slot, cudaStream_t s);
struct ProfScope {
    int slot;
    cudaStream_t s;
    ProfScope(KernelKind k, cudaStream_t s_) : slot(prof_begin(k, s_)), s(s_) {}
    ~ProfScope() { prof_end(slot, s); }
};

// Launchers (each returns the launch's cudaGetLastError()).
cudaError_t launch_gate_prep(const GateSrc& g, int B, int T, int H, float* la, float* lm,
                             float* lc, float* bco, float* gamma, cudaStream_t s);
cudaError_t launch_chunk_simt(const ChunkArgs& a, mdn_dtype dt, cudaStream_t s);
// The backward pass (fp32, CUDA cores); K-1's outputs must already be in a's scratch.
cudaError_t launch_chunk_bwd_simt(const BwdArgs& a, mdn_dtype dt, cudaStream_t s);
// B-3a of the backward pass on tcgen05 (bf16 inputs, d = 128).
cudaError_t launch_bwd_state_grads_tc(const BwdArgs& a, cudaStream_t s);
// B-3b of the backward pass on tcgen05 (bf16 inputs, d = 128).
cudaError_t launch_bwd_local_grads_tc(const BwdArgs& a, cudaStream_t s);
// The tensor-core reverse chain (bf16, d = 128).
cudaError_t launch_bwd_chain_tc(const BwdArgs& a, cudaStream_t s);
// tcgen05 version of the chain's operands plus the rebuilt entering states (a scan).
cudaError_t launch_bwd_chain_prep_tc(const BwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_prep_tc(const BwdArgs& a, cudaStream_t s);
// Tensor-core (tcgen05) path: bf16 q, k, v with d = 128.  Returns cudaErrorNotSupported
// when the arguments are outside what it handles.
// Records e as this thread's last CUDA error (mdn_last_cuda_error) and
// returns MDN_ERR_CUDA.
mdn_status cuda_fail(cudaError_t e);
// ns: columns of d_v per inter-chunk CTA (32 or 64), 0 = choose by batch size
cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t s, int ns);
cudaError_t launch_inter_head(const ChunkArgs& a, cudaStream_t s);
cudaError_t launch_chunk_intra_tc(const ChunkArgs& a, cudaStream_t s, int reserve, int limit);
// ds_norm (nullable, [B*H]): receives ||S_t - S_{t-1}||_F of each head.
cudaError_t launch_step(const void* q, const void* k, const void* v, mdn_dtype dt,
                        const float* alpha_log, const float* mu_log, const float* beta,
                        const float* eta, float dcorr, float* S, float* M, int B, int H,
                        int D, void* o, void* vt, float* ds_norm, cudaStream_t s);
// Gates from pre-activations (K-0), n elements; eta_act 0 = tanh + 1, 1 = 2 sigmoid.
cudaError_t launch_gate_params(const float* x_eta, const float* a, const float* b, const float* c,
                               long long n, float s_scale, float mu_log_min, int eta_act,
                               float* alpha_log, float* mu_log, float* beta, float* eta,
                               cudaStream_t s);
cudaError_t launch_finite_check(const void* x, size_t n, bool bf16, unsigned* flag,
                                cudaStream_t s);
// Variable-length mode.  Setup: checks cu_seqlens (N+1 device ints: 0, non-
// decreasing, ending at total_T), writes the checked copy to cu_s and the
// chunk offsets to cu_c (N+1 each); an invalid cu_seqlens sets *bad and
// makes every sequence empty.  Gather: the chunk-aligned padded inputs
// (NT*C rows; padding rows are steps that change nothing: k = v = q = 0,
// alpha = mu = 1, beta = eta = 0).
cudaError_t launch_varlen_setup(const int* cu_seqlens, int N, int total_T, int NT, int* cu_s,
                                int* cu_c, int* seq_order, int* chunk_order, unsigned* bad,
                                cudaStream_t s);
cudaError_t launch_varlen_gather(const void* q, const void* k, const void* v, size_t elt,
                                 const float* alpha_log, const float* mu_log, const float* beta,
                                 const float* eta, const int* cu_s, const int* cu_c, int N, int H,
                                 int D, int NT, void* qp, void* kp, void* vp, float* alp,
                                 float* mlp, float* bep, float* etp, cudaStream_t s);

}  // namespace mdn
