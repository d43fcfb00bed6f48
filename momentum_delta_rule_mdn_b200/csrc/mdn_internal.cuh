// Internal declarations shared by the libmdn translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "mdn.h"

namespace mdn {

constexpr int kChunk = 64;  // chunk length C supported by this build

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
    unsigned* status;  // [0]: non-finite flag, [1]: timeout flag
    float* la;         // [B*H, NT*C]
    float* lm;
    float* lc;
    float* bco;
    float* gamma;      // [B*H*NT, C, C]
    float* U;          // [B*H*NT, C, D]
    float* Y;
    float* Z;
    float* Oi;         // [B*H, NT*C, D]  carried-state part of o
    float* rec;        // [B*H*NT, 7, C]  packed coefficients (tensor-core path)
    // operands the intra-chunk kernel prepares for the inter-chunk kernel (bf16, per chunk)
    __nv_bfloat16* qhat;  // [B*H*NT, C, D]      qhat = q - d k
    __nv_bfloat16* tat;   // [B*H*NT, 2C, C]     [T; Att T]
    __nv_bfloat16* a2t;   // [B*H*NT, 2D, C]     [K^T Diag(Gamma_C) T; -K^T Diag(w) T]
    float* crec;          // [B*H*NT, 256]       alphabar_r, alpha_r b_{r-1}, b_r, then
                          //                     alphabar_C, b_C, mubar_C
    float* dbg = nullptr;  // diagnostics: if set, CTA 0 dumps its first chunk's intermediates
};

// Kernel kinds known to the optional timing facility (profile.cu).
enum KernelKind {
    kGatePrep = 0, kIntraSimt, kInterSimt, kOutputSimt, kStep, kFiniteCheck,
    kChunkTc, kIntraTc, kInterTc, kOutputTc, kKernelKinds
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
cudaError_t launch_gate_prep(const float* alpha_log, const float* mu_log, const float* beta,
                             const float* eta, int B, int T, int H, float* la, float* lm,
                             float* lc, float* bco, float* gamma, cudaStream_t s);
cudaError_t launch_gate_pack(const float* alpha_log, const float* mu_log, const float* beta,
                             const float* eta, int B, int T, int H, float* rec, cudaStream_t s);
cudaError_t launch_chunk_simt(const ChunkArgs& a, mdn_dtype dt, cudaStream_t s);
// Tensor-core (tcgen05) path: bf16 q, k, v with d = 128.  Returns cudaErrorNotSupported
// when the arguments are outside what it handles.
cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t s);
cudaError_t launch_chunk_intra_tc(const ChunkArgs& a, cudaStream_t s);
cudaError_t launch_chunk_inter_tc(const ChunkArgs& a, cudaStream_t s);
cudaError_t launch_step(const void* q, const void* k, const void* v, mdn_dtype dt,
                        const float* alpha_log, const float* mu_log, const float* beta,
                        const float* eta, float dcorr, float* S, float* M, int B, int H,
                        int D, void* o, void* vt, cudaStream_t s);
cudaError_t launch_finite_check(const void* x, size_t n, bool bf16, unsigned* flag,
                                cudaStream_t s);

}  // namespace mdn
