// The C ABI of libmdn (see include/mdn.h): argument validation, workspace
// layout and kernel dispatch.  Nothing here allocates device memory.
#include <stdint.h>
#include <string.h>

#include <cmath>
#include <cstdio>

#include "mdn_internal.cuh"

using namespace mdn;

namespace {

constexpr int kAbiVersion = 1;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
constexpr int kSliceFlags = MDN_SLICE32 | MDN_SLICE64 | MDN_SLICE128;
// At most one chain-width flag.
bool one_slice_flag(int flags)
{
    const int f = flags & kSliceFlags;
    return (f & (f - 1)) == 0;
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool aligned_elem(const void* p, mdn_dtype dt) {
    return (reinterpret_cast<uintptr_t>(p) & (dt == MDN_F32 ? 3u : 1u)) == 0;
}

struct WsLayout {
    size_t status, ready, la, lm, lc, bco, gamma, U, Y, Z, Oi, qhat, tat, a2t, crec, total;
    size_t head;  // bytes from the start that every call zeroes: status words and ready flags
};

// Whether a chunk pass with these arguments runs on the tensor cores.
bool uses_tensor_cores(mdn_dtype dt, int D, int flags)
{
    return dt == MDN_BF16 && D == 128 && !(flags & MDN_FORCE_SIMT);
}

// Byte offsets of the scratch regions of the path that will run (tc: the
// tensor-core path; else the CUDA-core path).  The status words and the
// ready flags sit together at the start so that one memset clears both.
WsLayout ws_layout(long long BH, int NT, int D, bool tc)
{
    const size_t chunks = (size_t)BH * NT;
    const size_t rows = chunks * kChunk;  // positions, padded to whole chunks
    WsLayout w = {};
    size_t off = 0;
    w.status = off; off += 64;
    w.ready = off;  off += (chunks + 1) * sizeof(unsigned);
    w.head = off;
    off = align_up(off);
    if (tc) {
        w.qhat = off;   off += align_up(rows * D * 2);
        w.tat = off;    off += align_up(rows * 2 * kChunk * 2);
        w.a2t = off;    off += align_up(rows * 2 * D * 2);
        w.crec = off;   off += align_up(rows * 4 * sizeof(float));
    } else {
        w.la = off;     off += align_up(rows * sizeof(float));
        w.lm = off;     off += align_up(rows * sizeof(float));
        w.lc = off;     off += align_up(rows * sizeof(float));
        w.bco = off;    off += align_up(rows * sizeof(float));
        w.gamma = off;  off += align_up(rows * kChunk * sizeof(float));
        w.U = off;      off += align_up(rows * D * sizeof(float));
        w.Y = off;      off += align_up(rows * D * sizeof(float));
        w.Z = off;      off += align_up(rows * D * sizeof(float));
        w.Oi = off;     off += align_up(rows * D * sizeof(float));
    }
    w.total = off;
    return w;
}

mdn_status check_sizes(int B, int T, int H, int dk, int dv, int C, mdn_dtype dt)
{
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0 || C <= 0) return MDN_ERR_INVALID_ARG;
    if (dt != MDN_F32 && dt != MDN_BF16) return MDN_ERR_UNSUPPORTED;
    if (dk != dv) return MDN_ERR_UNSUPPORTED;
    if (dk != 64 && dk != 128) return MDN_ERR_UNSUPPORTED;
    if (C != kChunk) return MDN_ERR_UNSUPPORTED;
    const long long NT = ((long long)T + C - 1) / C;
    if ((long long)B * H * NT >= (1LL << 31) || (long long)B * H >= (1LL << 31) / 2)
        return MDN_ERR_UNSUPPORTED;
    return MDN_OK;
}

mdn_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MDN_OK : mdn::cuda_fail(e); }

// Points the scratch members of a at their regions of ws (null for the
// regions the other path uses).
void carve(ChunkArgs& a, char* ws, const WsLayout& w)
{
    auto at = [ws](size_t off) -> char* { return off ? ws + off : nullptr; };
    a.status = reinterpret_cast<unsigned*>(ws + w.status);
    a.ready = reinterpret_cast<unsigned*>(ws + w.ready);
    a.la = reinterpret_cast<float*>(at(w.la));
    a.lm = reinterpret_cast<float*>(at(w.lm));
    a.lc = reinterpret_cast<float*>(at(w.lc));
    a.bco = reinterpret_cast<float*>(at(w.bco));
    a.gamma = reinterpret_cast<float*>(at(w.gamma));
    a.U = reinterpret_cast<float*>(at(w.U));
    a.Y = reinterpret_cast<float*>(at(w.Y));
    a.Z = reinterpret_cast<float*>(at(w.Z));
    a.Oi = reinterpret_cast<float*>(at(w.Oi));
    a.qhat = reinterpret_cast<__nv_bfloat16*>(at(w.qhat));
    a.tat = reinterpret_cast<__nv_bfloat16*>(at(w.tat));
    a.a2t = reinterpret_cast<__nv_bfloat16*>(at(w.a2t));
    a.crec = reinterpret_cast<float*>(at(w.crec));
}

// The chunk pass over a (scratch carved from layout w).  The status words
// and ready flags are zeroed first on every call, so that
// mdn_chunk_fwd_status can report what this call's kernels recorded.
// ntok: elements of o and of vt; nstate: heads of S_T and M_T.
// zero_head: false when the caller has already zeroed the head (packed
// sequences zero it before their offset check writes status[2]).
mdn_status run_pass(ChunkArgs& a, const WsLayout& w, mdn_dtype in_dtype, int flags,
                    cudaStream_t s, size_t ntok, size_t nstate, bool zero_head = true)
{
    cudaError_t e;
    const int D = a.D;
    if (zero_head && (e = cudaMemsetAsync(a.status, 0, w.head, s))) return mdn::cuda_fail(e);
    if (uses_tensor_cores(in_dtype, D, flags)) {
        const int ns = (flags & MDN_SLICE32) ? 32 : (flags & MDN_SLICE64) ? 64
                     : (flags & MDN_SLICE128) ? 128 : 0;
        a.test_no_intra = (flags & MDN_TEST_NO_INTRA) != 0;
        if ((e = launch_chunk_tc(a, s, ns))) return mdn::cuda_fail(e);
    } else {
        if ((e = launch_gate_prep(a.gates(), a.B, a.T, a.H, a.la, a.lm, a.lc, a.bco, a.gamma, s)))
            return mdn::cuda_fail(e);
        if ((e = launch_chunk_simt(a, in_dtype, s))) return mdn::cuda_fail(e);
    }
    if (!(flags & MDN_CHECK_FINITE)) return MDN_OK;

    const bool bf = in_dtype == MDN_BF16;
    const size_t nst = nstate * D * D;
    if ((e = launch_finite_check(a.o, ntok, bf, a.status, s))) return mdn::cuda_fail(e);
    if ((e = launch_finite_check(a.vt, ntok, bf, a.status, s))) return mdn::cuda_fail(e);
    if ((e = launch_finite_check(a.S_T, nst, false, a.status, s))) return mdn::cuda_fail(e);
    if ((e = launch_finite_check(a.M_T, nst, false, a.status, s))) return mdn::cuda_fail(e);
    unsigned host_status[3] = {0, 0, 0};
    if ((e = cudaMemcpyAsync(host_status, a.status, sizeof(host_status), cudaMemcpyDeviceToHost, s)))
        return mdn::cuda_fail(e);
    if ((e = cudaStreamSynchronize(s))) return mdn::cuda_fail(e);
    if (host_status[2]) return MDN_ERR_INVALID_ARG;
    if (host_status[1]) return MDN_ERR_TIMEOUT;
    if (host_status[0]) return MDN_ERR_NONFINITE;
    return MDN_OK;
}

}  // namespace

// ---------------------------------------------------------------- CUDA errors
namespace mdn {
namespace {
thread_local cudaError_t t_last_cuda_error = cudaSuccess;
thread_local char t_last_cuda_text[160] = "no CUDA error recorded on this thread";
}  // namespace
mdn_status cuda_fail(cudaError_t e)
{
    t_last_cuda_error = e;
    snprintf(t_last_cuda_text, sizeof(t_last_cuda_text), "%s (%d): %s", cudaGetErrorName(e),
             (int)e, cudaGetErrorString(e));
    return MDN_ERR_CUDA;
}
}  // namespace mdn

extern "C" const char* mdn_last_cuda_error(void) { return mdn::t_last_cuda_text; }

// ---------------------------------------------------------------- finite check
namespace mdn {
namespace {
__global__ void finite_check_kernel(const void* x, size_t n, bool bf16, unsigned* flag)
{
    unsigned bad = 0;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        if (bf16) {
            const unsigned short u = static_cast<const unsigned short*>(x)[i];
            bad |= ((u & 0x7f80u) == 0x7f80u);
        } else {
            bad |= !isfinite(static_cast<const float*>(x)[i]);
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(flag, 1u);
}
}  // namespace

cudaError_t launch_finite_check(const void* x, size_t n, bool bf16, unsigned* flag,
                                cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    size_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    ProfScope ps(kFiniteCheck, s);
    finite_check_kernel<<<(unsigned)blocks, 256, 0, s>>>(x, n, bf16, flag);
    return cudaGetLastError();
}
}  // namespace mdn

// ---------------------------------------------------------------- exports
extern "C" {

int mdn_abi_version(void) { return kAbiVersion; }

const char* mdn_status_string(mdn_status s)
{
    switch (s) {
        case MDN_OK: return "MDN_OK";
        case MDN_ERR_INVALID_ARG: return "MDN_ERR_INVALID_ARG: invalid argument";
        case MDN_ERR_UNSUPPORTED: return "MDN_ERR_UNSUPPORTED: sizes or dtype outside the library's support";
        case MDN_ERR_CUDA: return "MDN_ERR_CUDA: a CUDA launch or runtime call failed";
        case MDN_ERR_NONFINITE: return "MDN_ERR_NONFINITE: an output holds NaN or Inf";
        case MDN_ERR_TIMEOUT: return "MDN_ERR_TIMEOUT: a bounded device wait ran out";
    }
    return "unknown mdn_status";
}

size_t mdn_chunk_fwd_workspace_size_flags(int B, int T, int H, int dk, int dv, int C,
                                          mdn_dtype in_dtype, int flags)
{
    if (check_sizes(B, T, H, dk, dv, C, in_dtype) != MDN_OK) return 0;
    const int NT = (T + C - 1) / C;
    return ws_layout((long long)B * H, NT, dk, uses_tensor_cores(in_dtype, dk, flags)).total;
}

size_t mdn_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int C,
                                    mdn_dtype in_dtype)
{
    return mdn_chunk_fwd_workspace_size_flags(B, T, H, dk, dv, C, in_dtype, 0);
}

mdn_status mdn_chunk_fwd_status(const void* workspace, mdn_stream_t stream)
{
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % kAlign) return MDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned host_status[3] = {0, 0, 0};
    cudaError_t e = cudaMemcpyAsync(host_status, workspace, sizeof(host_status),
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return mdn::cuda_fail(e);
    if (host_status[2]) return MDN_ERR_INVALID_ARG;
    if (host_status[1]) return MDN_ERR_TIMEOUT;
    if (host_status[0]) return MDN_ERR_NONFINITE;
    return MDN_OK;
}

namespace {
// mdn_chunk_fwd with the gates from `g` (the gate arrays, or pre-activations).
mdn_status chunk_fwd_impl(const void* q, const void* k, const void* v, mdn_dtype in_dtype,
                          const GateSrc& g, float d_corr, const float* S0, const float* M0,
                          int B, int T, int H, int dk, int dv, int C, void* o, void* vtilde,
                          float* S_T, float* M_T, void* workspace, size_t ws_bytes, int flags,
                          mdn_stream_t stream)
{
    mdn_status st = check_sizes(B, T, H, dk, dv, C, in_dtype);
    if (st != MDN_OK) return st;
    if (flags & ~(MDN_CHECK_FINITE | MDN_FORCE_SIMT | kSliceFlags | MDN_TEST_NO_INTRA))
        return MDN_ERR_INVALID_ARG;
    if (!one_slice_flag(flags)) return MDN_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return MDN_OK;
    if (!S_T || !M_T || !aligned16(S_T) || !aligned16(M_T)) return MDN_ERR_INVALID_ARG;
    if ((S0 && !aligned16(S0)) || (M0 && !aligned16(M0))) return MDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = dk;
    const size_t state_bytes = (size_t)B * H * D * D * sizeof(float);
    if (T == 0) {
        cudaError_t e = cudaSuccess;
        if (S0) { if (S0 != S_T) e = cudaMemcpyAsync(S_T, S0, state_bytes, cudaMemcpyDeviceToDevice, s); }
        else e = cudaMemsetAsync(S_T, 0, state_bytes, s);
        if (e == cudaSuccess) {
            if (M0) { if (M0 != M_T) e = cudaMemcpyAsync(M_T, M0, state_bytes, cudaMemcpyDeviceToDevice, s); }
            else e = cudaMemsetAsync(M_T, 0, state_bytes, s);
        }
        return cuda_status(e);
    }
    const void* tok[] = {q, k, v, o, vtilde};
    for (const void* p : tok)
        if (!p || !aligned16(p)) return MDN_ERR_INVALID_ARG;
    for (const void* p : g.g)
        if (!p || !aligned4(p)) return MDN_ERR_INVALID_ARG;
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % kAlign) return MDN_ERR_INVALID_ARG;
    const int NT = (T + C - 1) / C;
    const WsLayout w = ws_layout((long long)B * H, NT, D, uses_tensor_cores(in_dtype, D, flags));
    if (ws_bytes < w.total) return MDN_ERR_INVALID_ARG;

    ChunkArgs a;
    a.q = q; a.k = k; a.v = v;
    a.alpha_log = g.g[0]; a.mu_log = g.g[1]; a.beta = g.g[2]; a.eta = g.g[3];
    a.gate_pre = g.pre; a.gate_s = g.s; a.gate_mu_min = g.mu_min;
    a.dcorr = d_corr; a.S0 = S0; a.M0 = M0;
    a.B = B; a.T = T; a.H = H; a.D = D; a.NT = NT;
    a.o = o; a.vt = vtilde; a.S_T = S_T; a.M_T = M_T;
    carve(a, static_cast<char*>(workspace), w);
    return run_pass(a, w, in_dtype, flags, s, (size_t)B * T * H * D, (size_t)B * H);
}
}  // namespace

mdn_status mdn_chunk_fwd(const void* q, const void* k, const void* v, mdn_dtype in_dtype,
                         const float* alpha_log, const float* mu_log, const float* beta,
                         const float* eta, float d_corr, const float* S0, const float* M0,
                         int B, int T, int H, int dk, int dv, int C, void* o, void* vtilde,
                         float* S_T, float* M_T, void* workspace, size_t ws_bytes, int flags,
                         mdn_stream_t stream)
{
    return chunk_fwd_impl(q, k, v, in_dtype, GateSrc{{alpha_log, mu_log, beta, eta}, 0, 1.f, 0.f},
                          d_corr, S0, M0, B, T, H, dk, dv, C, o, vtilde, S_T, M_T, workspace,
                          ws_bytes, flags, stream);
}

mdn_status mdn_chunk_fwd_preact(const void* q, const void* k, const void* v, mdn_dtype in_dtype,
                                const float* x_eta, const float* a_pre, const float* b_pre,
                                const float* c_pre, float s, float mu_log_min, int eta_act,
                                float d_corr, const float* S0, const float* M0, int B, int T,
                                int H, int dk, int dv, int C, void* o, void* vtilde, float* S_T,
                                float* M_T, void* workspace, size_t ws_bytes, int flags,
                                mdn_stream_t stream)
{
    if (eta_act != MDN_ETA_TANH && eta_act != MDN_ETA_2SIGMOID) return MDN_ERR_INVALID_ARG;
    if (!std::isfinite(s) || !std::isfinite(mu_log_min)) return MDN_ERR_INVALID_ARG;
    return chunk_fwd_impl(q, k, v, in_dtype,
                          GateSrc{{x_eta, a_pre, b_pre, c_pre}, 1 + eta_act, s, mu_log_min},
                          d_corr, S0, M0, B, T, H, dk, dv, C, o, vtilde, S_T, M_T, workspace,
                          ws_bytes, flags, stream);
}

// ---------------------------------------------------------------- backward
namespace {

struct BwdLayout {
    size_t status, la, lm, lc, bco, gamma, att, tmat, SS, dSS, rec;
    size_t bc_u, bc_tt, bc_p, bc_qh, bc_eo, bc_rec, bc_d, dy;  // tensor-core path (bf16, d = 128)
    size_t total;
};

// tc: the tensor-core path (bf16 state images instead of fp32 states, and the
// reverse chain's chunk operands).  For bf16 at d = 128 its total is the
// larger of the two paths'.
BwdLayout bwd_layout(long long BH, int NT, int D, bool tc)
{
    const size_t chunks = (size_t)BH * NT, rows = chunks * kChunk;
    BwdLayout w;
    size_t off = 0;
    w.status = off; off += align_up(64);
    w.la = off;    off += align_up(rows * sizeof(float));
    w.lm = off;    off += align_up(rows * sizeof(float));
    w.lc = off;    off += align_up(rows * sizeof(float));
    w.bco = off;   off += align_up(rows * sizeof(float));
    w.gamma = off; off += align_up(rows * kChunk * sizeof(float));
    w.att = off;   off += align_up(rows * kChunk * sizeof(float));
    w.tmat = off;  off += align_up(rows * kChunk * sizeof(float));
    const size_t state_bytes = tc ? (size_t)kStateImgBytes : 2 * D * D * sizeof(float);
    w.SS = off;    off += align_up(chunks * state_bytes);
    w.dSS = off;   off += align_up(chunks * state_bytes);
    w.rec = off;   off += align_up(chunks * kBwdRec * sizeof(float));
    w.bc_u = w.bc_tt = w.bc_p = w.bc_qh = w.bc_eo = w.bc_rec = w.bc_d = w.dy = 0;
    if (tc) {
        w.bc_u = off;   off += align_up(chunks * 256 * 64 * 2);
        w.bc_tt = off;  off += align_up(chunks * 64 * 64 * 2);
        w.bc_p = off;   off += align_up(chunks * kChunk * D * 2);
        w.bc_qh = off;  off += align_up(chunks * kChunk * D * 2);
        w.bc_eo = off;  off += align_up(chunks * (D / 32) * 2 * 4096);
        w.bc_rec = off; off += align_up(chunks * 256 * sizeof(float));
        w.bc_d = off;   off += align_up(chunks * 2 * D * D * 2);
        w.dy = off;     off += align_up(chunks * kDyImgBytes);
    }
    w.total = off;
    return w;
}

}  // namespace

size_t mdn_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int C,
                                    mdn_dtype in_dtype)
{
    if (check_sizes(B, T, H, dk, dv, C, in_dtype) != MDN_OK) return 0;
    return bwd_layout((long long)B * H, (T + C - 1) / C, dk, in_dtype == MDN_BF16 && dk == 128).total;
}

mdn_status mdn_chunk_bwd(const void* q, const void* k, const void* v, mdn_dtype in_dtype,
                         const float* alpha_log, const float* mu_log, const float* beta,
                         const float* eta, float d_corr, const float* S0, const float* M0,
                         const void* vtilde, const void* d_o, const float* dS_T,
                         const float* dM_T, int B, int T, int H, int dk, int dv, int C,
                         float* dq, float* dk_out, float* dv_out, float* dalpha_log,
                         float* dmu_log, float* dbeta, float* deta, float* dS0, float* dM0,
                         void* workspace, size_t ws_bytes, int flags, mdn_stream_t stream)
{
    mdn_status st = check_sizes(B, T, H, dk, dv, C, in_dtype);
    if (st != MDN_OK) return st;
    if (flags & ~(MDN_CHECK_FINITE | MDN_FORCE_SIMT)) return MDN_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return MDN_OK;
    if (!dS0 || !dM0 || !aligned16(dS0) || !aligned16(dM0)) return MDN_ERR_INVALID_ARG;
    const void* opt[] = {S0, M0, dS_T, dM_T};
    for (const void* p : opt)
        if (p && !aligned16(p)) return MDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = dk;
    if (T > 0) {
        const void* tok[] = {q, k, v, vtilde, d_o, dq, dk_out, dv_out};
        for (const void* p : tok)
            if (!p || !aligned16(p)) return MDN_ERR_INVALID_ARG;
        const void* g[] = {alpha_log, mu_log, beta, eta, dalpha_log, dmu_log, dbeta, deta};
        for (const void* p : g)
            if (!p || !aligned4(p)) return MDN_ERR_INVALID_ARG;
    }
    const int NT = (T + C - 1) / C;
    const bool tc = in_dtype == MDN_BF16 && D == 128 && !(flags & MDN_FORCE_SIMT);
    const BwdLayout w = bwd_layout((long long)B * H, NT, D, tc);
    if (T > 0 && (!workspace || reinterpret_cast<uintptr_t>(workspace) % kAlign))
        return MDN_ERR_INVALID_ARG;
    if (T > 0 && ws_bytes < w.total) return MDN_ERR_INVALID_ARG;
    const size_t state_bytes = (size_t)B * H * D * D * sizeof(float);
    cudaError_t e;
    if (T == 0) {  // S_T = S0, M_T = M0: the adjoints pass straight through
        if (dS_T) e = cudaMemcpyAsync(dS0, dS_T, state_bytes, cudaMemcpyDeviceToDevice, s);
        else e = cudaMemsetAsync(dS0, 0, state_bytes, s);
        if (e == cudaSuccess) {
            if (dM_T) e = cudaMemcpyAsync(dM0, dM_T, state_bytes, cudaMemcpyDeviceToDevice, s);
            else e = cudaMemsetAsync(dM0, 0, state_bytes, s);
        }
        return cuda_status(e);
    }
    char* ws = static_cast<char*>(workspace);
    BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.vt = vtilde; a.dout = d_o;
    a.alpha_log = alpha_log; a.mu_log = mu_log; a.beta = beta; a.eta = eta;
    a.dcorr = d_corr; a.S0 = S0; a.M0 = M0; a.dS_T = dS_T; a.dM_T = dM_T;
    a.B = B; a.T = T; a.H = H; a.D = D; a.NT = NT;
    a.status = reinterpret_cast<unsigned*>(ws + w.status);
    a.la = reinterpret_cast<float*>(ws + w.la);
    a.lm = reinterpret_cast<float*>(ws + w.lm);
    a.lc = reinterpret_cast<float*>(ws + w.lc);
    a.bco = reinterpret_cast<float*>(ws + w.bco);
    a.gamma = reinterpret_cast<float*>(ws + w.gamma);
    a.att = reinterpret_cast<float*>(ws + w.att);
    a.tmat = reinterpret_cast<float*>(ws + w.tmat);
    a.SS = tc ? nullptr : reinterpret_cast<float*>(ws + w.SS);
    a.dSS = tc ? nullptr : reinterpret_cast<float*>(ws + w.dSS);
    a.ss_img = tc ? reinterpret_cast<uint8_t*>(ws + w.SS) : nullptr;
    a.dss_img = tc ? reinterpret_cast<uint8_t*>(ws + w.dSS) : nullptr;
    a.crec_bw = reinterpret_cast<float*>(ws + w.rec);
    a.bc_u = tc ? reinterpret_cast<__nv_bfloat16*>(ws + w.bc_u) : nullptr;
    a.bc_tt = tc ? reinterpret_cast<__nv_bfloat16*>(ws + w.bc_tt) : nullptr;
    a.bc_p = tc ? reinterpret_cast<__nv_bfloat16*>(ws + w.bc_p) : nullptr;
    a.bc_qh = tc ? reinterpret_cast<__nv_bfloat16*>(ws + w.bc_qh) : nullptr;
    a.bc_eo = tc ? reinterpret_cast<uint8_t*>(ws + w.bc_eo) : nullptr;
    a.bc_rec = tc ? reinterpret_cast<float*>(ws + w.bc_rec) : nullptr;
    a.bc_d = tc ? reinterpret_cast<__nv_bfloat16*>(ws + w.bc_d) : nullptr;
    a.dy_img = tc ? reinterpret_cast<uint8_t*>(ws + w.dy) : nullptr;
    a.dq = dq; a.dk = dk_out; a.dv = dv_out;
    a.dalpha_log = dalpha_log; a.dmu_log = dmu_log; a.dbeta = dbeta; a.deta = deta;
    a.dS0 = dS0; a.dM0 = dM0;
    const bool check = flags & MDN_CHECK_FINITE;
    if (check && (e = cudaMemsetAsync(a.status, 0, 64, s))) return mdn::cuda_fail(e);
    if ((e = launch_gate_prep(GateSrc{{alpha_log, mu_log, beta, eta}, 0, 1.f, 0.f}, B, T, H,
                              a.la, a.lm, a.lc, a.bco,
                              a.gamma, s)))
        return mdn::cuda_fail(e);
    if ((e = launch_chunk_bwd_simt(a, in_dtype, s))) return mdn::cuda_fail(e);
    if (!check) return MDN_OK;
    const size_t ntok = (size_t)B * T * H * D, ngate = (size_t)B * T * H;
    const float* outs[] = {dq, dk_out, dv_out};
    for (const float* p : outs)
        if ((e = launch_finite_check(p, ntok, false, a.status, s))) return mdn::cuda_fail(e);
    const float* gouts[] = {dalpha_log, dmu_log, dbeta, deta};
    for (const float* p : gouts)
        if ((e = launch_finite_check(p, ngate, false, a.status, s))) return mdn::cuda_fail(e);
    if ((e = launch_finite_check(dS0, (size_t)B * H * D * D, false, a.status, s)) ||
        (e = launch_finite_check(dM0, (size_t)B * H * D * D, false, a.status, s)))
        return mdn::cuda_fail(e);
    unsigned host_status[2] = {0, 0};
    if ((e = cudaMemcpyAsync(host_status, a.status, sizeof(host_status), cudaMemcpyDeviceToHost, s)))
        return mdn::cuda_fail(e);
    if ((e = cudaStreamSynchronize(s))) return mdn::cuda_fail(e);
    if (host_status[1]) return MDN_ERR_TIMEOUT;
    if (host_status[0]) return MDN_ERR_NONFINITE;
    return MDN_OK;
}

// ---------------------------------------------------------------- variable length
namespace {

struct VarlenLayout {
    size_t cu_s, cu_c, seq_order, chunk_order, q, k, v, al, ml, be, et, total;
    WsLayout chunk;  // the chunk pass's scratch, at the start of the workspace
    int NT;          // padded chunks (an upper bound on the sequences' chunk count)
};

// NT = floor(total_T / C) + N bounds sum_s ceil(len_s / C) for any split of
// total_T tokens into N sequences.
mdn_status varlen_layout(int N, int total_T, int H, int dk, int dv, int C, mdn_dtype dt,
                         int flags, VarlenLayout& v)
{
    if (N < 0 || total_T < 0 || C <= 0) return MDN_ERR_INVALID_ARG;
    const long long NT = (long long)total_T / (C > 0 ? C : 1) + N;
    if (NT * C >= (1LL << 31)) return MDN_ERR_UNSUPPORTED;
    mdn_status st = check_sizes(1, (int)(NT * C), H, dk, dv, C, dt);
    if (st != MDN_OK) return st;
    if ((long long)N * H >= (1LL << 31) / 2) return MDN_ERR_UNSUPPORTED;
    const size_t rows = (size_t)NT * C * H;  // padded token-heads
    const size_t elt = dt == MDN_F32 ? 4 : 2;
    v.NT = (int)NT;
    v.chunk = ws_layout(H, v.NT, dk, uses_tensor_cores(dt, dk, flags));
    size_t off = v.chunk.total;
    v.cu_s = off; off += align_up((size_t)(N + 1) * sizeof(int));
    v.cu_c = off; off += align_up((size_t)(N + 1) * sizeof(int));
    v.seq_order = off;   off += align_up((size_t)N * sizeof(int));
    v.chunk_order = off; off += align_up((size_t)NT * sizeof(int));
    v.q = off;    off += align_up(rows * dk * elt);
    v.k = off;    off += align_up(rows * dk * elt);
    v.v = off;    off += align_up(rows * dv * elt);
    v.al = off;   off += align_up(rows * sizeof(float));
    v.ml = off;   off += align_up(rows * sizeof(float));
    v.be = off;   off += align_up(rows * sizeof(float));
    v.et = off;   off += align_up(rows * sizeof(float));
    v.total = off;
    return MDN_OK;
}

}  // namespace

size_t mdn_chunk_fwd_varlen_workspace_size_flags(int N, int total_T, int H, int dk, int dv,
                                                 int C, mdn_dtype in_dtype, int flags)
{
    VarlenLayout v;
    if (varlen_layout(N, total_T, H, dk, dv, C, in_dtype, flags, v) != MDN_OK) return 0;
    return v.total;
}

size_t mdn_chunk_fwd_varlen_workspace_size(int N, int total_T, int H, int dk, int dv, int C,
                                           mdn_dtype in_dtype)
{
    return mdn_chunk_fwd_varlen_workspace_size_flags(N, total_T, H, dk, dv, C, in_dtype, 0);
}

mdn_status mdn_chunk_fwd_varlen(const void* q, const void* k, const void* v, mdn_dtype in_dtype,
                                const float* alpha_log, const float* mu_log, const float* beta,
                                const float* eta, float d_corr, const int* cu_seqlens, int N,
                                int total_T, const float* S0, const float* M0, int H, int dk,
                                int dv, int C, void* o, void* vtilde, float* S_T, float* M_T,
                                void* workspace, size_t ws_bytes, int flags, mdn_stream_t stream)
{
    VarlenLayout L;
    mdn_status st = varlen_layout(N, total_T, H, dk, dv, C, in_dtype, flags, L);
    if (st != MDN_OK) return st;
    if (flags & ~(MDN_CHECK_FINITE | MDN_FORCE_SIMT | kSliceFlags)) return MDN_ERR_INVALID_ARG;
    if (!one_slice_flag(flags)) return MDN_ERR_INVALID_ARG;
    if (N == 0 || H == 0) return MDN_OK;
    if (!cu_seqlens || !aligned4(cu_seqlens)) return MDN_ERR_INVALID_ARG;
    if (!S_T || !M_T || !aligned16(S_T) || !aligned16(M_T)) return MDN_ERR_INVALID_ARG;
    if ((S0 && !aligned16(S0)) || (M0 && !aligned16(M0))) return MDN_ERR_INVALID_ARG;
    if (total_T > 0) {
        const void* tok[] = {q, k, v, o, vtilde};
        for (const void* p : tok)
            if (!p || !aligned16(p)) return MDN_ERR_INVALID_ARG;
        const void* gates[] = {alpha_log, mu_log, beta, eta};
        for (const void* p : gates)
            if (!p || !aligned4(p)) return MDN_ERR_INVALID_ARG;
    }
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % kAlign) return MDN_ERR_INVALID_ARG;
    if (ws_bytes < L.total) return MDN_ERR_INVALID_ARG;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int D = dk;
    char* ws = static_cast<char*>(workspace);
    int* cu_s = reinterpret_cast<int*>(ws + L.cu_s);
    int* cu_c = reinterpret_cast<int*>(ws + L.cu_c);
    ChunkArgs a;
    a.q = ws + L.q; a.k = ws + L.k; a.v = ws + L.v;
    a.alpha_log = reinterpret_cast<float*>(ws + L.al);
    a.mu_log = reinterpret_cast<float*>(ws + L.ml);
    a.beta = reinterpret_cast<float*>(ws + L.be);
    a.eta = reinterpret_cast<float*>(ws + L.et);
    a.dcorr = d_corr; a.S0 = S0; a.M0 = M0;
    a.B = 1; a.T = L.NT * C; a.H = H; a.D = D; a.NT = L.NT;
    a.o = o; a.vt = vtilde; a.S_T = S_T; a.M_T = M_T;
    a.cu_seqlens = cu_s; a.cu_chunks = cu_c; a.nseq = N;
    int* seq_order = reinterpret_cast<int*>(ws + L.seq_order);
    int* chunk_order = reinterpret_cast<int*>(ws + L.chunk_order);
    a.seq_order = seq_order; a.chunk_order = chunk_order;
    carve(a, ws, L.chunk);

    cudaError_t e;
    if ((e = cudaMemsetAsync(a.status, 0, L.chunk.head, s))) return mdn::cuda_fail(e);
    if ((e = launch_varlen_setup(cu_seqlens, N, total_T, L.NT, cu_s, cu_c, seq_order, chunk_order,
                                 a.status + 2, s)))
        return mdn::cuda_fail(e);
    const size_t elt = in_dtype == MDN_F32 ? 4 : 2;
    if ((e = launch_varlen_gather(q, k, v, elt, alpha_log, mu_log, beta, eta, cu_s, cu_c, N, H, D,
                                  L.NT, const_cast<void*>(a.q), const_cast<void*>(a.k),
                                  const_cast<void*>(a.v), const_cast<float*>(a.alpha_log),
                                  const_cast<float*>(a.mu_log), const_cast<float*>(a.beta),
                                  const_cast<float*>(a.eta), s)))
        return mdn::cuda_fail(e);
    return run_pass(a, L.chunk, in_dtype, flags, s, (size_t)total_T * H * D, (size_t)N * H,
                    /*zero_head=*/false);
}

namespace {
mdn_status step_impl(const void* q, const void* k, const void* v, mdn_dtype in_dtype,
                     const float* alpha_log, const float* mu_log, const float* beta,
                     const float* eta, float d_corr, float* S, float* M, int B, int H, int dk,
                     int dv, void* o, void* vtilde, float* ds_norm, int flags,
                     mdn_stream_t stream)
{
    mdn_status st = check_sizes(B, 1, H, dk, dv, kChunk, in_dtype);
    if (st != MDN_OK) return st;
    if (flags != 0) return MDN_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return MDN_OK;
    const void* tok[] = {q, k, v, o};
    for (const void* p : tok)
        if (!p || !aligned_elem(p, in_dtype)) return MDN_ERR_INVALID_ARG;
    if (vtilde && !aligned_elem(vtilde, in_dtype)) return MDN_ERR_INVALID_ARG;
    const void* gates[] = {alpha_log, mu_log, beta, eta};
    for (const void* p : gates)
        if (!p || !aligned4(p)) return MDN_ERR_INVALID_ARG;
    if (!S || !M || !aligned16(S) || !aligned16(M)) return MDN_ERR_INVALID_ARG;
    if (ds_norm && !aligned4(ds_norm)) return MDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(launch_step(q, k, v, in_dtype, alpha_log, mu_log, beta, eta, d_corr, S,
                                   M, B, H, dk, o, vtilde, ds_norm, s));
}
}  // namespace

mdn_status mdn_step(const void* q, const void* k, const void* v, mdn_dtype in_dtype,
                    const float* alpha_log, const float* mu_log, const float* beta,
                    const float* eta, float d_corr, float* S, float* M, int B, int H, int dk,
                    int dv, void* o, void* vtilde, int flags, mdn_stream_t stream)
{
    return step_impl(q, k, v, in_dtype, alpha_log, mu_log, beta, eta, d_corr, S, M, B, H, dk,
                     dv, o, vtilde, nullptr, flags, stream);
}

mdn_status mdn_step_delta_norm(const void* q, const void* k, const void* v, mdn_dtype in_dtype,
                               const float* alpha_log, const float* mu_log, const float* beta,
                               const float* eta, float d_corr, float* S, float* M, int B, int H,
                               int dk, int dv, void* o, void* vtilde, float* ds_norm, int flags,
                               mdn_stream_t stream)
{
    if (!ds_norm && B > 0 && H > 0) return MDN_ERR_INVALID_ARG;
    return step_impl(q, k, v, in_dtype, alpha_log, mu_log, beta, eta, d_corr, S, M, B, H, dk,
                     dv, o, vtilde, ds_norm, flags, stream);
}

mdn_status mdn_gate_params(const float* x_eta, const float* a, const float* b, const float* c,
                           long long n, float s, float mu_log_min, int eta_act,
                           float* alpha_log, float* mu_log, float* beta, float* eta,
                           mdn_stream_t stream)
{
    if (n < 0) return MDN_ERR_INVALID_ARG;
    if (eta_act != MDN_ETA_TANH && eta_act != MDN_ETA_2SIGMOID) return MDN_ERR_INVALID_ARG;
    if (!std::isfinite(s) || !std::isfinite(mu_log_min)) return MDN_ERR_INVALID_ARG;
    if (n == 0) return MDN_OK;
    const void* ptrs[] = {x_eta, a, b, c, alpha_log, mu_log, beta, eta};
    for (const void* p : ptrs)
        if (!p || !aligned4(p)) return MDN_ERR_INVALID_ARG;
    return cuda_status(launch_gate_params(x_eta, a, b, c, n, s, mu_log_min, eta_act, alpha_log,
                                          mu_log, beta, eta,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

mdn_status mdn_chunk_gate_prep(const float* alpha_log, const float* mu_log, const float* beta,
                               const float* eta, int B, int T, int H, int C, float* la,
                               float* lm, float* lc, float* b, float* gamma,
                               mdn_stream_t stream)
{
    mdn_status st = check_sizes(B, T, H, 64, 64, C, MDN_F32);
    if (st != MDN_OK) return st;
    if (B == 0 || H == 0 || T == 0) return MDN_OK;
    const void* gates[] = {alpha_log, mu_log, beta, eta};
    for (const void* p : gates)
        if (!p || !aligned4(p)) return MDN_ERR_INVALID_ARG;
    const void* outs[] = {la, lm, lc, b};
    for (const void* p : outs)
        if (!p || (reinterpret_cast<uintptr_t>(p) & 7u)) return MDN_ERR_INVALID_ARG;
    if (gamma && !aligned4(gamma)) return MDN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(launch_gate_prep(GateSrc{{alpha_log, mu_log, beta, eta}, 0, 1.f, 0.f},
                                        B, T, H, la, lm, lc, b,
                                        gamma, s));
}

}  // extern "C"
