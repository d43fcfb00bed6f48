// The backward pass of the chunkwise forward pass, on CUDA cores in fp32.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 7; ijyty.com article, section 6: training
// keeps the corrected values Vtilde from the forward pass and rebuilds S and M
// from them in the backward pass.  Per chunk (C = 64; S, M the states entering
// it; dS, dM the adjoints of the states leaving it; the coefficients of the
// forward chunk form: alphabar, b, Gamma, w_r = eta_r mubar_C / mubar_r,
// D1 = alphabar, D2_r = b_{r-1} alpha_r, Att = (Qhat K^T) o Gamma):
//
//   rebuild   S' = alphabar_C S - b_C M + K^T Diag(Gamma_C) Vtilde
//             M' = mubar_C M - K^T Diag(w) Vtilde
//   reverse   dVtilde = Att^T dO + Diag(Gamma_C) K dS - Diag(w) K dM
//   chain     dY = T^T dVtilde                       (= dV)
//             dS <- alphabar_C dS + Qhat^T Diag(alphabar) dO - K^T Diag(D1) dY
//             dM <- -b_C dS + mubar_C dM - Qhat^T Diag(b) dO + K^T Diag(D2) dY
//   local     dQhat = Diag(alphabar) dO S^T - Diag(b) dO M^T + ((dO Vtilde^T) o Gamma) K
//             dK = Diag(Gamma_C) Vtilde dS^T - Diag(w) Vtilde dM^T - Diag(D1) dY S^T
//                  + Diag(D2) dY M^T + ((dO Vtilde^T) o Gamma)^T Qhat
//                  + dPK^T P + Diag(alpha) dPK K,  dPK = -(dY Vtilde^T) o Gamma-
//             dq = dQhat,  dk = dK - d dQhat
//   gates     through the adjoints of alphabar, b, Gamma, w and the chunk-end
//             scalars, by the definitions of those coefficients (below).
//
// Kernels: B-0 T and Att per chunk; B-1 the rebuilt entering states (chain over
// chunks, d_v split in slices); B-2 the reverse chain of (dS, dM); B-3a the
// products with the states (dO S^T, ..., per chunk); B-3b the chunk-local
// products and the gate gradients.  All outputs are fp32.
#include <type_traits>

#include "bwd_common.cuh"
#include "mdn_internal.cuh"

namespace mdn {
namespace {

constexpr int C = kChunk;
constexpr int NSB = 32;  // d_v columns per chain CTA

template <typename Tin>
__device__ __forceinline__ float ldt(const void* base, size_t idx) {
    return ld_elem(static_cast<const Tin*>(base) + idx);
}

__device__ __forceinline__ size_t tok_idx(const BwdArgs& a, int b, int t, int h) {
    return ((size_t)b * a.T + t) * a.H + h;
}

// ------------------------------------------------------------------ B-0
// T = (I + A)^{-1}, A = (P K^T) o Gamma-, and Att = (Qhat K^T) o Gamma.
template <typename Tin, int D>
__global__ void __launch_bounds__(256)
bwd_prep_kernel(BwdArgs a)
{
    constexpr int KS = D + 1, AS = C + 1;
    extern __shared__ float smem[];
    float* Ks = smem;              // [C][D+1]
    float* Qs = Ks + C * KS;       // [C][D+1]  qhat
    float* As = Qs + C * KS;       // [C][C+1]  A
    float* Ts = As + C * AS;       // [C][C+1]  T
    float* alpha_s = Ts + C * AS;  // [C]
    const int tid = threadIdx.x;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const size_t chunk = blockIdx.x;
    // K, Qhat: 8-element vector loads, all issued before the shared-memory stores
    {
        constexpr int PER = C * D / 8 / 256;  // vectors per thread and tensor
        float kx[PER][8], qx[PER][8];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int idx = tid + 256 * u, r = idx / (D / 8), c8 = idx % (D / 8), t = n * C + r;
            if (t < a.T) {
                const size_t g = tok_idx(a, b, t, h) * D + 8 * c8;
                ld8<Tin>(a.k, g, kx[u]);
                ld8<Tin>(a.q, g, qx[u]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) kx[u][e] = qx[u][e] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int idx = tid + 256 * u, r = idx / (D / 8), c8 = idx % (D / 8);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                Ks[r * KS + 8 * c8 + e] = kx[u][e];
                Qs[r * KS + 8 * c8 + e] = qx[u][e] - a.dcorr * kx[u][e];
            }
        }
    }
    if (tid < C) {
        const int t = n * C + tid;
        alpha_s[tid] = t < a.T ? expf(a.alpha_log[tok_idx(a, b, t, h)]) : 1.f;
    }
    const float* G = a.gamma + chunk * C * C;
    float* att = a.att + chunk * C * C;
    // Gamma at this thread's tile (rows r and r - 1), loaded before the products
    const int rg = tid >> 4, ig = tid & 15;
    float g_r[4][4], g_m[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int r = rg + 16 * u, i = ig + 16 * v;
            g_r[u][v] = i <= r ? __ldg(G + r * C + i) : 0.f;
            g_m[u][v] = i < r ? __ldg(G + (r - 1) * C + i) : 0.f;
        }
    __syncthreads();
    {
        // K K^T and Qhat K^T over 4 x 4 register tiles: rows rg + 16 u, columns ig + 16 v
        float kk[4][4], qk[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) kk[u][v] = qk[u][v] = 0.f;
        for (int c = 0; c < D; ++c) {
            float rk[4], rq[4], ik[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                rk[u] = Ks[(rg + 16 * u) * KS + c];
                rq[u] = Qs[(rg + 16 * u) * KS + c];
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) ik[v] = Ks[(ig + 16 * v) * KS + c];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    kk[u][v] = fmaf(rk[u], ik[v], kk[u][v]);
                    qk[u][v] = fmaf(rq[u], ik[v], qk[u][v]);
                }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int r = rg + 16 * u, i = ig + 16 * v;
                float av = 0.f, tv = 0.f;
                if (i <= r) {
                    tv = qk[u][v] * g_r[u][v];
                    if (i < r) av = alpha_s[r] * kk[u][v] * g_m[u][v];
                }
                As[r * AS + i] = av;
                att[r * C + i] = tv;
            }
    }
    __syncthreads();
    // unit lower-triangular inverse by forward substitution: column c on the
    // four lanes 4c .. 4c + 3, each summing every fourth term
    bwd_unit_lower_inverse(As, Ts, tid);
    __syncthreads();
    float* Tm = a.tmat + chunk * C * C;
    for (int idx = tid; idx < C * C; idx += 256) Tm[idx] = Ts[(idx / C) * AS + idx % C];
}

// ------------------------------------------------------------------ B-1
// The states entering every chunk, rebuilt from Vtilde.
template <typename Tin, int D>
__global__ void __launch_bounds__(256)
bwd_states_kernel(BwdArgs a)
{
    // a thread owns rows rg + 16 e and the column pair 2 j2, 2 j2 + 1 of the slice
    constexpr int NS = NSB, KS = D + 1, VS = NS + 2;
    constexpr int EP = D / 16;     // rows per thread
    extern __shared__ float smem[];
    float* Ss = smem;              // [D][NS]
    float* Ms = Ss + D * NS;
    float* Ks = Ms + D * NS;       // [C][D+1]
    float* Vs = Ks + C * KS;       // [C][NS+2] (8-byte aligned rows)
    float* gl = Vs + C * VS;       // [C] Gamma_{C,r}
    float* wv = gl + C;            // [C] w_r
    float* scal = wv + C;          // alphabar_C, b_C, mubar_C
    const int tid = threadIdx.x;
    const int slice = blockIdx.x % (D / NS);
    const long long bh = blockIdx.x / (D / NS);
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const int j0 = slice * NS, j2 = tid & 15, rg = tid >> 4, jc = 2 * j2;
    const size_t st = (size_t)bh * D * D;
    for (int e = 0; e < EP; ++e) {
        const int i = rg + 16 * e;
        const size_t g = st + (size_t)i * D + j0 + jc;
        *reinterpret_cast<float2*>(Ss + i * NS + jc) =
            a.S0 ? make_float2(a.S0[g], a.S0[g + 1]) : make_float2(0.f, 0.f);
        *reinterpret_cast<float2*>(Ms + i * NS + jc) =
            a.M0 ? make_float2(a.M0[g], a.M0[g + 1]) : make_float2(0.f, 0.f);
    }
    for (int n = 0; n < a.NT; ++n) {
        const size_t chunk = (size_t)bh * a.NT + n;
        const size_t crow = chunk * C;
        float* SSn = a.SS + chunk * 2 * D * D;
        __syncthreads();
        for (int e = 0; e < EP; ++e) {
            const int i = rg + 16 * e;
            const float2 sv = *reinterpret_cast<const float2*>(Ss + i * NS + jc);
            const float2 mv = *reinterpret_cast<const float2*>(Ms + i * NS + jc);
            SSn[(size_t)i * D + j0 + jc] = sv.x;
            SSn[(size_t)i * D + j0 + jc + 1] = sv.y;
            SSn[(size_t)D * D + (size_t)i * D + j0 + jc] = mv.x;
            SSn[(size_t)D * D + (size_t)i * D + j0 + jc + 1] = mv.y;
        }
        {   // K (C x D) and the Vtilde slice (C x NS), eight elements per load,
            // every load of a thread issued before its stores
            constexpr int KU = C * D / 8 / 256, VU = C * NS / 8 / 256;
            float kx[KU][8], vx[VU > 0 ? VU : 1][8];
#pragma unroll
            for (int u = 0; u < KU; ++u) {
                const int idx = (tid + 256 * u) * 8, r = idx / D, c = idx % D, t = n * C + r;
                if (t < a.T) ld8<Tin>(a.k, tok_idx(a, b, t, h) * D + c, kx[u]);
                else for (int e = 0; e < 8; ++e) kx[u][e] = 0.f;
            }
            if (tid < C * NS / 8) {
                const int idx = tid * 8, r = idx / NS, c = idx % NS, t = n * C + r;
                if (t < a.T) ld8<Tin>(a.vt, tok_idx(a, b, t, h) * D + j0 + c, vx[0]);
                else for (int e = 0; e < 8; ++e) vx[0][e] = 0.f;
            }
#pragma unroll
            for (int u = 0; u < KU; ++u) {
                const int idx = (tid + 256 * u) * 8, r = idx / D, c = idx % D;
#pragma unroll
                for (int e = 0; e < 8; ++e) Ks[r * KS + c + e] = kx[u][e];
            }
            if (tid < C * NS / 8) {
                const int idx = tid * 8, r = idx / NS, c = idx % NS;
#pragma unroll
                for (int e = 0; e < 8; ++e) Vs[r * VS + c + e] = vx[0][e];
            }
        }
        if (tid < C) {
            const int r = tid, t = n * C + r;
            gl[r] = a.gamma[chunk * C * C + (C - 1) * C + r];
            const float et = t < a.T ? a.eta[tok_idx(a, b, t, h)] : 0.f;
            wv[r] = et * expf(a.lm[crow + C - 1] - a.lm[crow + r]);
            if (r == 0) {
                scal[0] = expf(a.la[crow + C - 1]);
                scal[1] = a.bco[crow + C - 1];
                scal[2] = expf(a.lm[crow + C - 1]);
            }
        }
        __syncthreads();
        float dS[EP][2], dM[EP][2];
#pragma unroll
        for (int e = 0; e < EP; ++e) dS[e][0] = dS[e][1] = dM[e][0] = dM[e][1] = 0.f;
        for (int r = 0; r < C; ++r) {
            const float2 v = *reinterpret_cast<const float2*>(Vs + r * VS + jc);
            const float g = gl[r], w = wv[r];
            const float vg0 = v.x * g, vg1 = v.y * g, vw0 = v.x * w, vw1 = v.y * w;
#pragma unroll
            for (int e = 0; e < EP; ++e) {
                const float kv = Ks[r * KS + rg + 16 * e];
                dS[e][0] = fmaf(kv, vg0, dS[e][0]);
                dS[e][1] = fmaf(kv, vg1, dS[e][1]);
                dM[e][0] = fmaf(kv, vw0, dM[e][0]);
                dM[e][1] = fmaf(kv, vw1, dM[e][1]);
            }
        }
#pragma unroll
        for (int e = 0; e < EP; ++e) {
            const int i = rg + 16 * e;
            float2* sp = reinterpret_cast<float2*>(Ss + i * NS + jc);
            float2* mp = reinterpret_cast<float2*>(Ms + i * NS + jc);
            const float2 sv = *sp, mv = *mp;
            *sp = make_float2(scal[0] * sv.x - scal[1] * mv.x + dS[e][0],
                              scal[0] * sv.y - scal[1] * mv.y + dS[e][1]);
            *mp = make_float2(scal[2] * mv.x - dM[e][0], scal[2] * mv.y - dM[e][1]);
        }
    }
}

// ------------------------------------------------------------------ B-2
// The reverse chain of the state adjoints; writes dV = dY and, per chunk, the
// adjoints of the states leaving it.
template <typename Tin, int D>
__global__ void __launch_bounds__(256)
bwd_chain_kernel(BwdArgs a)
{
    // a thread owns the column pair 2 j2, 2 j2 + 1 of the slice, rows rg + 16 e
    constexpr int NS = NSB, KS = D + 1, VS = NS + 2, AS = C + 1;
    constexpr int EP = D / 16;     // state rows per thread
    constexpr int RP = C / 16;     // chunk rows per thread
    extern __shared__ float smem[];
    float* dSs = smem;             // [D][NS]
    float* dMs = dSs + D * NS;
    float* Ks = dMs + D * NS;      // [C][D+1]
    float* Qs = Ks + C * KS;       // [C][D+1]
    float* Att = Qs + C * KS;      // [C][C+1]
    float* Tm = Att + C * AS;      // [C][C+1]
    float* dOs = Tm + C * AS;      // [C][NS+2]
    float* X = dOs + C * VS;       // [C][NS+2]  dVtilde, then dY
    float* abar = X + C * VS;      // [C]
    float* bco = abar + C;
    float* d2 = bco + C;           // b_{r-1} alpha_r
    float* gl = d2 + C;
    float* wv = gl + C;
    float* scal = wv + C;          // alphabar_C, b_C, mubar_C
    const int tid = threadIdx.x;
    const int slice = blockIdx.x % (D / NS);
    const long long bh = blockIdx.x / (D / NS);
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const int j0 = slice * NS, j2 = tid & 15, rg = tid >> 4, jc = 2 * j2;
    const size_t st = (size_t)bh * D * D;
    for (int e = 0; e < EP; ++e) {
        const int i = rg + 16 * e;
        const size_t g = st + (size_t)i * D + j0 + jc;
        *reinterpret_cast<float2*>(dSs + i * NS + jc) =
            a.dS_T ? make_float2(a.dS_T[g], a.dS_T[g + 1]) : make_float2(0.f, 0.f);
        *reinterpret_cast<float2*>(dMs + i * NS + jc) =
            a.dM_T ? make_float2(a.dM_T[g], a.dM_T[g + 1]) : make_float2(0.f, 0.f);
    }
    for (int n = a.NT - 1; n >= 0; --n) {
        const size_t chunk = (size_t)bh * a.NT + n;
        const size_t crow = chunk * C;
        float* dSSn = a.dSS + chunk * 2 * D * D;
        __syncthreads();
        for (int e = 0; e < EP; ++e) {
            const int i = rg + 16 * e;
            const float2 sv = *reinterpret_cast<const float2*>(dSs + i * NS + jc);
            const float2 mv = *reinterpret_cast<const float2*>(dMs + i * NS + jc);
            dSSn[(size_t)i * D + j0 + jc] = sv.x;
            dSSn[(size_t)i * D + j0 + jc + 1] = sv.y;
            dSSn[(size_t)D * D + (size_t)i * D + j0 + jc] = mv.x;
            dSSn[(size_t)D * D + (size_t)i * D + j0 + jc + 1] = mv.y;
        }
        for (int idx = tid; idx < C * D; idx += 256) {
            const int r = idx / D, c = idx % D, t = n * C + r;
            float kv = 0.f, qv = 0.f;
            if (t < a.T) {
                const size_t g = tok_idx(a, b, t, h) * D + c;
                kv = ldt<Tin>(a.k, g);
                qv = ldt<Tin>(a.q, g) - a.dcorr * kv;
            }
            Ks[r * KS + c] = kv;
            Qs[r * KS + c] = qv;
        }
        for (int idx = tid; idx < C * C; idx += 256) {
            const int r = idx / C, i = idx % C;
            Att[r * AS + i] = a.att[chunk * C * C + idx];
            Tm[r * AS + i] = a.tmat[chunk * C * C + idx];
        }
        for (int idx = tid; idx < C * NS; idx += 256) {
            const int r = idx / NS, c = idx % NS, t = n * C + r;
            dOs[r * VS + c] = t < a.T ? ldt<Tin>(a.dout, tok_idx(a, b, t, h) * D + j0 + c) : 0.f;
        }
        if (tid < C) {
            const int r = tid, t = n * C + r;
            abar[r] = expf(a.la[crow + r]);
            bco[r] = a.bco[crow + r];
            const float al = t < a.T ? expf(a.alpha_log[tok_idx(a, b, t, h)]) : 1.f;
            d2[r] = r > 0 ? a.bco[crow + r - 1] * al : 0.f;
            gl[r] = a.gamma[chunk * C * C + (C - 1) * C + r];
            const float et = t < a.T ? a.eta[tok_idx(a, b, t, h)] : 0.f;
            wv[r] = et * expf(a.lm[crow + C - 1] - a.lm[crow + r]);
            if (r == 0) {
                scal[0] = expf(a.la[crow + C - 1]);
                scal[1] = a.bco[crow + C - 1];
                scal[2] = expf(a.lm[crow + C - 1]);
            }
        }
        __syncthreads();
        // dVtilde = Att^T dO + Gamma_C o (K dS) - w o (K dM)
        {
            float kds[RP][2], kdm[RP][2], ad[RP][2];
#pragma unroll
            for (int e = 0; e < RP; ++e)
#pragma unroll
                for (int c = 0; c < 2; ++c) kds[e][c] = kdm[e][c] = ad[e][c] = 0.f;
            for (int i = 0; i < D; ++i) {
                const float2 ds = *reinterpret_cast<const float2*>(dSs + i * NS + jc);
                const float2 dm = *reinterpret_cast<const float2*>(dMs + i * NS + jc);
#pragma unroll
                for (int e = 0; e < RP; ++e) {
                    const float kv = Ks[(rg + 16 * e) * KS + i];
                    kds[e][0] = fmaf(kv, ds.x, kds[e][0]);
                    kds[e][1] = fmaf(kv, ds.y, kds[e][1]);
                    kdm[e][0] = fmaf(kv, dm.x, kdm[e][0]);
                    kdm[e][1] = fmaf(kv, dm.y, kdm[e][1]);
                }
            }
            // Att is lower triangular (zeros above the diagonal): full sums are exact
            for (int r2 = rg; r2 < C; ++r2) {
                const float2 od = *reinterpret_cast<const float2*>(dOs + r2 * VS + jc);
#pragma unroll
                for (int e = 0; e < RP; ++e) {
                    const float at = Att[r2 * AS + rg + 16 * e];
                    ad[e][0] = fmaf(at, od.x, ad[e][0]);
                    ad[e][1] = fmaf(at, od.y, ad[e][1]);
                }
            }
#pragma unroll
            for (int e = 0; e < RP; ++e) {
                const int r = rg + 16 * e;
                *reinterpret_cast<float2*>(X + r * VS + jc) =
                    make_float2(ad[e][0] + gl[r] * kds[e][0] - wv[r] * kdm[e][0],
                                ad[e][1] + gl[r] * kds[e][1] - wv[r] * kdm[e][1]);
            }
        }
        __syncthreads();
        float dy[RP][2];
#pragma unroll
        for (int e = 0; e < RP; ++e) dy[e][0] = dy[e][1] = 0.f;
        for (int r2 = rg; r2 < C; ++r2) {  // T lower triangular as well
            const float2 xv = *reinterpret_cast<const float2*>(X + r2 * VS + jc);
#pragma unroll
            for (int e = 0; e < RP; ++e) {
                const float tv = Tm[r2 * AS + rg + 16 * e];
                dy[e][0] = fmaf(tv, xv.x, dy[e][0]);
                dy[e][1] = fmaf(tv, xv.y, dy[e][1]);
            }
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < RP; ++e) {
            const int r = rg + 16 * e, t = n * C + r;
            *reinterpret_cast<float2*>(X + r * VS + jc) = make_float2(dy[e][0], dy[e][1]);
            if (t < a.T) {
                float* dst = a.dv + tok_idx(a, b, t, h) * D + j0 + jc;
                dst[0] = dy[e][0];
                dst[1] = dy[e][1];
            }
        }
        __syncthreads();
        const float aC = scal[0], bC = scal[1], mC = scal[2];
        float us[EP][2], um[EP][2];  // qhat^T (.) dO - K^T (.) dY terms of dS and dM
#pragma unroll
        for (int e = 0; e < EP; ++e) us[e][0] = us[e][1] = um[e][0] = um[e][1] = 0.f;
        for (int r = 0; r < C; ++r) {
            const float2 od = *reinterpret_cast<const float2*>(dOs + r * VS + jc);
            const float2 xd = *reinterpret_cast<const float2*>(X + r * VS + jc);
            const float ab = abar[r], bb = bco[r], dd = d2[r];
            const float qa0 = od.x * ab, qa1 = od.y * ab, qb0 = od.x * bb, qb1 = od.y * bb;
            const float xa0 = xd.x * ab, xa1 = xd.y * ab, x20 = xd.x * dd, x21 = xd.y * dd;
#pragma unroll
            for (int e = 0; e < EP; ++e) {
                const int i = rg + 16 * e;
                const float qv = Qs[r * KS + i], kv = Ks[r * KS + i];
                us[e][0] = fmaf(qv, qa0, fmaf(-kv, xa0, us[e][0]));
                us[e][1] = fmaf(qv, qa1, fmaf(-kv, xa1, us[e][1]));
                um[e][0] = fmaf(kv, x20, fmaf(-qv, qb0, um[e][0]));
                um[e][1] = fmaf(kv, x21, fmaf(-qv, qb1, um[e][1]));
            }
        }
#pragma unroll
        for (int e = 0; e < EP; ++e) {
            const int i = rg + 16 * e;
            float2* sp = reinterpret_cast<float2*>(dSs + i * NS + jc);
            float2* mp = reinterpret_cast<float2*>(dMs + i * NS + jc);
            const float2 ds = *sp, dm = *mp;
            *sp = make_float2(aC * ds.x + us[e][0], aC * ds.y + us[e][1]);
            *mp = make_float2(-bC * ds.x + mC * dm.x + um[e][0], -bC * ds.y + mC * dm.y + um[e][1]);
        }
    }
    __syncthreads();
    for (int e = 0; e < EP; ++e) {
        const int i = rg + 16 * e;
        const float2 sv = *reinterpret_cast<const float2*>(dSs + i * NS + jc);
        const float2 mv = *reinterpret_cast<const float2*>(dMs + i * NS + jc);
        const size_t g = st + (size_t)i * D + j0 + jc;
        a.dS0[g] = sv.x;
        a.dS0[g + 1] = sv.y;
        a.dM0[g] = mv.x;
        a.dM0[g + 1] = mv.y;
    }
}

// ------------------------------------------------------------------ B-3a
// Products with the entering states S, M and the leaving adjoints dS, dM:
// P1 = dO S^T, P2 = dO M^T, P3 = Vt dS^T, P4 = Vt dM^T, P5 = dY S^T,
// P6 = dY M^T (C x d_k each), streamed over panels of KP rows of d_k; a
// thread holds 2 rows x 4 columns of all six.  Writes dq's and dk's parts
// from them, and per chunk the coefficient adjoints they carry (row sums)
// plus <S,dS>, <M,dS>, <M,dM>.
constexpr int KP = 32;

template <typename Tin, int D>
__global__ void __launch_bounds__(256)
bwd_state_grads_kernel(BwdArgs a)
{
    constexpr int TS = D + 1;
    extern __shared__ float smem[];
    float* dOs = smem;             // [C][D+1]
    float* Vts = dOs + C * TS;
    float* dYs = Vts + C * TS;
    float* Pn = dYs + C * TS;      // 4 panels [KP][D+1]: S, M, dS, dM
    float* red = Pn + 4 * KP * TS; // [8][3]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const size_t chunk = blockIdx.x, crow = chunk * C;
    const float* Sn = a.SS + chunk * 2 * D * D;
    const float* Mn = Sn + D * D;
    const float* dSn = a.dSS + chunk * 2 * D * D;
    const float* dMn = dSn + D * D;
    for (int idx = tid; idx < C * D; idx += 256) {
        const int r = idx / D, c = idx % D, t = n * C + r;
        float o = 0.f, vv = 0.f, y = 0.f;
        if (t < a.T) {
            const size_t g = tok_idx(a, b, t, h) * D + c;
            o = ldt<Tin>(a.dout, g);
            vv = ldt<Tin>(a.vt, g);
            y = a.dv[g];
        }
        dOs[r * TS + c] = o;
        Vts[r * TS + c] = vv;
        dYs[r * TS + c] = y;
    }
    // <S, dS>, <M, dS>, <M, dM>
    float s1 = 0.f, s2 = 0.f, s3 = 0.f;
    for (int idx = tid; idx < D * D; idx += 256) {
        const float sv = Sn[idx], mv = Mn[idx], dsv = dSn[idx], dmv = dMn[idx];
        s1 = fmaf(sv, dsv, s1);
        s2 = fmaf(mv, dsv, s2);
        s3 = fmaf(mv, dmv, s3);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
        s2 += __shfl_xor_sync(0xffffffffu, s2, off);
        s3 += __shfl_xor_sync(0xffffffffu, s3, off);
    }
    if (lane == 0) {
        red[warp * 3] = s1;
        red[warp * 3 + 1] = s2;
        red[warp * 3 + 2] = s3;
    }
    const int rp = tid >> 3, kq = tid & 7;  // rows 2 rp, 2 rp + 1; k = k0 + kq + 8 m
    float abar[2], bco[2], d2[2], gl[2], w[2];
    bool in[2];
    size_t gt[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int r = 2 * rp + u, t = n * C + r;
        in[u] = t < a.T;
        gt[u] = in[u] ? tok_idx(a, b, t, h) : 0;
        abar[u] = expf(a.la[crow + r]);
        bco[u] = a.bco[crow + r];
        const float al = in[u] ? expf(a.alpha_log[gt[u]]) : 1.f;
        d2[u] = r > 0 ? a.bco[crow + r - 1] * al : 0.f;
        gl[u] = a.gamma[chunk * C * C + (C - 1) * C + r];
        const float et = in[u] ? a.eta[gt[u]] : 0.f;
        w[u] = et * expf(a.lm[crow + C - 1] - a.lm[crow + r]);
    }
    float sa[2] = {0.f, 0.f}, sb[2] = {0.f, 0.f}, sd2[2] = {0.f, 0.f}, sgl[2] = {0.f, 0.f},
          sw[2] = {0.f, 0.f};
    for (int k0 = 0; k0 < D; k0 += KP) {
        __syncthreads();
        for (int idx = tid; idx < KP * D; idx += 256) {
            const int kk = idx / D, c = idx % D;
            const size_t g = (size_t)(k0 + kk) * D + c;
            Pn[kk * TS + c] = Sn[g];
            Pn[KP * TS + kk * TS + c] = Mn[g];
            Pn[2 * KP * TS + kk * TS + c] = dSn[g];
            Pn[3 * KP * TS + kk * TS + c] = dMn[g];
        }
        __syncthreads();
        float p[6][2][4];
#pragma unroll
        for (int x = 0; x < 6; ++x)
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int m = 0; m < 4; ++m) p[x][u][m] = 0.f;
        for (int c = 0; c < D; ++c) {
            float o[2], vv[2], y[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                o[u] = dOs[(2 * rp + u) * TS + c];
                vv[u] = Vts[(2 * rp + u) * TS + c];
                y[u] = dYs[(2 * rp + u) * TS + c];
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int kk = kq + 8 * m;
                const float sv = Pn[kk * TS + c], mv = Pn[KP * TS + kk * TS + c];
                const float dsv = Pn[2 * KP * TS + kk * TS + c];
                const float dmv = Pn[3 * KP * TS + kk * TS + c];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    p[0][u][m] = fmaf(o[u], sv, p[0][u][m]);
                    p[1][u][m] = fmaf(o[u], mv, p[1][u][m]);
                    p[2][u][m] = fmaf(vv[u], dsv, p[2][u][m]);
                    p[3][u][m] = fmaf(vv[u], dmv, p[3][u][m]);
                    p[4][u][m] = fmaf(y[u], sv, p[4][u][m]);
                    p[5][u][m] = fmaf(y[u], mv, p[5][u][m]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (!in[u]) continue;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int k = k0 + kq + 8 * m;
                const size_t g = gt[u] * D + k;
                const float kv = ldt<Tin>(a.k, g);
                const float qh = ldt<Tin>(a.q, g) - a.dcorr * kv;
                a.dq[g] = abar[u] * p[0][u][m] - bco[u] * p[1][u][m];
                a.dk[g] = gl[u] * p[2][u][m] - w[u] * p[3][u][m] - abar[u] * p[4][u][m] +
                          d2[u] * p[5][u][m];
                sa[u] = fmaf(qh, p[0][u][m], fmaf(-kv, p[4][u][m], sa[u]));
                sb[u] = fmaf(-qh, p[1][u][m], sb[u]);
                sd2[u] = fmaf(kv, p[5][u][m], sd2[u]);
                sgl[u] = fmaf(kv, p[2][u][m], sgl[u]);
                sw[u] = fmaf(-kv, p[3][u][m], sw[u]);
            }
        }
    }
    // the eight threads of a row pair hold its partial sums
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            sa[u] += __shfl_xor_sync(0xffffffffu, sa[u], off);
            sb[u] += __shfl_xor_sync(0xffffffffu, sb[u], off);
            sd2[u] += __shfl_xor_sync(0xffffffffu, sd2[u], off);
            sgl[u] += __shfl_xor_sync(0xffffffffu, sgl[u], off);
            sw[u] += __shfl_xor_sync(0xffffffffu, sw[u], off);
        }
    }
    float* rec = a.crec_bw + chunk * kBwdRec;
    if (kq == 0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int r = 2 * rp + u;
            rec[r] = sa[u];
            rec[C + r] = sb[u];
            rec[2 * C + r] = sd2[u];
            rec[3 * C + r] = sgl[u];
            rec[4 * C + r] = sw[u];
        }
    }
    __syncthreads();
    if (tid < 3) {
        float acc = 0.f;
        for (int w8 = 0; w8 < 8; ++w8) acc += red[w8 * 3 + tid];
        rec[5 * C + tid] = acc;
    }
}

// ------------------------------------------------------------------ B-3b
// Chunk-local products and the gate gradients.
template <typename Tin, int D>
__global__ void __launch_bounds__(256)
bwd_local_grads_kernel(BwdArgs a)
{
    constexpr int TS = D + 1, AS = C + 1;
    extern __shared__ float smem[];
    float* Ks = smem;              // [C][D+1]
    float* Qs = Ks + C * TS;       // qhat
    float* Vts = Qs + C * TS;
    float* dOs = Vts + C * TS;     // dO, then (dO Vt^T) o Gamma  [C][C+1]
    float* dYs = dOs + C * TS;     // dY, then dPK                [C][C+1]
    float* Gp = dYs + C * TS;      // [C][C+1] Gamma without eta
    float* dG = Gp + C * AS;       // [C][C+1] adjoint of Gamma, then R
    const BwdVec v = bwd_vec(dG + C * AS);
    float* v_al = v.al;
    float* v_be = v.be;
    float* v_et = v.et;
    float* v_la = v.la;
    float* v_lm = v.lm;
    float* v_b = v.b;
    float* v_da = v.da;
    const int tid = threadIdx.x;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const size_t chunk = blockIdx.x, crow = chunk * C;
    for (int idx = tid; idx < C * D; idx += 256) {
        const int r = idx / D, c = idx % D, t = n * C + r;
        float kv = 0.f, qv = 0.f, vv = 0.f, o = 0.f, y = 0.f;
        if (t < a.T) {
            const size_t g = tok_idx(a, b, t, h) * D + c;
            kv = ldt<Tin>(a.k, g);
            qv = ldt<Tin>(a.q, g) - a.dcorr * kv;
            vv = ldt<Tin>(a.vt, g);
            o = ldt<Tin>(a.dout, g);
            y = a.dv[g];
        }
        Ks[r * TS + c] = kv;
        Qs[r * TS + c] = qv;
        Vts[r * TS + c] = vv;
        dOs[r * TS + c] = o;
        dYs[r * TS + c] = y;
    }
    if (tid < C) {
        const int r = tid, t = n * C + r;
        const bool in = t < a.T;
        const size_t gi = in ? tok_idx(a, b, t, h) : 0;
        v_al[r] = in ? expf(a.alpha_log[gi]) : 1.f;
        v_be[r] = in ? a.beta[gi] : 0.f;
        v_et[r] = in ? a.eta[gi] : 0.f;
        v_la[r] = a.la[crow + r];
        v_lm[r] = a.lm[crow + r];
        v_b[r] = a.bco[crow + r];
    }
    __syncthreads();
    // Gamma without eta by its column recurrence: Gp_{i,i} = beta_i,
    // Gp_{r,i} = alpha_r Gp_{r-1,i} + beta_r mubar_r / mubar_i
    if (tid < C) {
        const int i = tid;
        float g = 0.f;
        for (int r = 0; r < C; ++r) {
            if (r < i) {
                Gp[r * AS + i] = 0.f;
            } else {
                g = (r == i) ? v_be[i] : fmaf(v_al[r], g, v_be[r] * expf(v_lm[r] - v_lm[i]));
                Gp[r * AS + i] = g;
            }
        }
    }
    // the four C x C products over 4 x 4 register tiles: rows rg + 16 u, columns ig + 16 v
    const int rg = tid >> 4, ig = tid & 15;
    float dov[4][4], qk[4][4], dyv[4][4], kk[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) dov[u][v] = qk[u][v] = dyv[u][v] = kk[u][v] = 0.f;
    for (int c = 0; c < D; ++c) {
        float ro[4], rq[4], ry[4], rk[4], iv[4], ik[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = rg + 16 * u;
            ro[u] = dOs[r * TS + c];
            rq[u] = Qs[r * TS + c];
            ry[u] = dYs[r * TS + c];
            rk[u] = Ks[r * TS + c];
        }
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int i = ig + 16 * v;
            iv[v] = Vts[i * TS + c];
            ik[v] = Ks[i * TS + c];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                dov[u][v] = fmaf(ro[u], iv[v], dov[u][v]);
                qk[u][v] = fmaf(rq[u], ik[v], qk[u][v]);
                dyv[u][v] = fmaf(ry[u], iv[v], dyv[u][v]);
                kk[u][v] = fmaf(rk[u], ik[v], kk[u][v]);
            }
    }
    __syncthreads();  // dO and dY tiles are no longer read; Gp is complete
    float* dOVG = dOs;  // [C][C+1]
    float* dPK = dYs;   // [C][C+1]
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int r = rg + 16 * u, i = ig + 16 * v;
            const float g = v_et[i] * Gp[r * AS + i];
            float ovg = 0.f, pk = 0.f, dg = 0.f;
            if (i <= r) {
                ovg = dov[u][v] * g;
                dg = dov[u][v] * qk[u][v];
            }
            if (i < r) pk = -dyv[u][v] * v_et[i] * Gp[(r - 1) * AS + i];  // dA o Gamma-
            dOVG[r * AS + i] = ovg;
            dPK[r * AS + i] = pk;
            dG[r * AS + i] = dg;
        }
    __syncthreads();
    // Gamma-_{r,i} = Gamma_{r-1,i}: dA o (P K^T) lands on row r - 1 (one writer per entry)
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int r = rg + 16 * u, i = ig + 16 * v;
            if (i < r) dG[(r - 1) * AS + i] += -dyv[u][v] * v_al[r] * kk[u][v];
        }
    const float* rec = a.crec_bw + chunk * kBwdRec;
    __syncthreads();
    if (tid < C) dG[(C - 1) * AS + tid] += rec[3 * C + tid];  // Gamma_{C,i} in the state update
    // dQhat += dOVG K ; dK += dOVG^T Qhat + dPK^T P + Diag(alpha) dPK K ; d alpha from P.
    // A thread holds rows 2 rp, 2 rp + 1 and columns cg + 8 m.  dOVG and dPK are
    // stored with zeros outside their triangles, so full-range sums are exact.
    {
        constexpr int NM = D / 8;
        const int rp = tid >> 3, cg = tid & 7;
        float dq[2][NM], dp[2][NM];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int m = 0; m < NM; ++m) dq[u][m] = dp[u][m] = 0.f;
        for (int i = 0; i <= 2 * rp + 1; ++i) {
            const float g0 = dOVG[(2 * rp) * AS + i], g1 = dOVG[(2 * rp + 1) * AS + i];
            const float p0 = dPK[(2 * rp) * AS + i], p1 = dPK[(2 * rp + 1) * AS + i];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const float kv = Ks[i * TS + cg + 8 * m];
                dq[0][m] = fmaf(g0, kv, dq[0][m]);
                dq[1][m] = fmaf(g1, kv, dq[1][m]);
                dp[0][m] = fmaf(p0, kv, dp[0][m]);
                dp[1][m] = fmaf(p1, kv, dp[1][m]);
            }
        }
        float dk[2][NM];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int m = 0; m < NM; ++m) dk[u][m] = 0.f;
        for (int r2 = 2 * rp; r2 < C; ++r2) {
            const float al2 = v_al[r2];
            const float g0 = dOVG[r2 * AS + 2 * rp], g1 = dOVG[r2 * AS + 2 * rp + 1];
            const float p0 = dPK[r2 * AS + 2 * rp] * al2, p1 = dPK[r2 * AS + 2 * rp + 1] * al2;
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const float qv = Qs[r2 * TS + cg + 8 * m], kv = Ks[r2 * TS + cg + 8 * m];
                dk[0][m] = fmaf(g0, qv, fmaf(p0, kv, dk[0][m]));
                dk[1][m] = fmaf(g1, qv, fmaf(p1, kv, dk[1][m]));
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int r = 2 * rp + u, t = n * C + r;
            const float alr = v_al[r];
            float dar = 0.f;
#pragma unroll
            for (int m = 0; m < NM; ++m) dar = fmaf(dp[u][m], Ks[r * TS + cg + 8 * m], dar);
            if (t < a.T) {
                // every load before any store: the stores would otherwise pin the
                // loads that follow them in program order
                const size_t g0 = tok_idx(a, b, t, h) * D + cg;
                float qo[NM], ko[NM];
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    qo[m] = a.dq[g0 + 8 * m];
                    ko[m] = a.dk[g0 + 8 * m];
                }
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    const float dqt = qo[m] + dq[u][m];
                    a.dq[g0 + 8 * m] = dqt;
                    a.dk[g0 + 8 * m] = ko[m] + fmaf(alr, dp[u][m], dk[u][m]) - a.dcorr * dqt;
                }
            }
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) dar += __shfl_xor_sync(0xffffffffu, dar, off);
            if (cg == 0) v_da[r] = dar;
        }
    }
    __syncthreads();
    bwd_coeff_phase(a, rec, v, dG, Gp, v.dbe + C, tid, n, b, h);
}

// A non-blocking stream of the current device for work forked off a call's
// stream, created on first use by each host thread and kept.
cudaError_t side_stream(cudaStream_t* out)
{
    thread_local cudaStream_t streams[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!streams[dev] &&
        (e = cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking)) != cudaSuccess)
        return e;
    *out = streams[dev];
    return cudaSuccess;
}

template <typename Tin, int D>
cudaError_t launch_bwd_typed(const BwdArgs& a, cudaStream_t s)
{
    const long long chunks = (long long)a.B * a.H * a.NT;
    const long long chains = (long long)a.B * a.H * (D / NSB);
    const size_t sm0 = sizeof(float) * (2 * C * (D + 1) + 2 * C * (C + 1) + C);
    const size_t sm1 = sizeof(float) * (2 * D * NSB + C * (D + 1) + C * (NSB + 2) + 2 * C + 4);
    const size_t sm2 = sizeof(float) * (2 * D * NSB + 2 * C * (D + 1) + 2 * C * (C + 1) +
                                        2 * C * (NSB + 2) + 5 * C + 4);
    const size_t sm3a = sizeof(float) * (3 * C * (D + 1) + 4 * KP * (D + 1) + 24);
    const size_t sm3b = sizeof(float) * (5 * C * (D + 1) + 2 * C * (C + 1) + kBwdVecFloats + kBwdRec);
    cudaError_t e;
#define MDN_SET_SMEM(K, BYTES)                                                          \
    if ((e = cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize,       \
                                  (int)(BYTES))) != cudaSuccess)                        \
        return e;
    MDN_SET_SMEM((bwd_prep_kernel<Tin, D>), sm0)
    MDN_SET_SMEM((bwd_states_kernel<Tin, D>), sm1)
    MDN_SET_SMEM((bwd_chain_kernel<Tin, D>), sm2)
    MDN_SET_SMEM((bwd_state_grads_kernel<Tin, D>), sm3a)
    MDN_SET_SMEM((bwd_local_grads_kernel<Tin, D>), sm3b)
#undef MDN_SET_SMEM
    if (std::is_same<Tin, __nv_bfloat16>::value && D == 128 && a.bc_u) {
        // bf16, d = 128: T and Att, the chain's operands and the rebuild
        // increments on tensor cores, the entering states by an elementwise
        // scan, the reverse chain and both per-chunk product kernels on
        // tensor cores
        if ((e = launch_bwd_prep_tc(a, s))) return e;
        if ((e = launch_bwd_chain_prep_tc(a, s))) return e;
        if ((e = launch_bwd_chain_tc(a, s))) return e;
        if ((e = launch_bwd_state_grads_tc(a, s))) return e;
        return launch_bwd_local_grads_tc(a, s);
    }
    // The state rebuild depends only on the chunk coefficients and is needed
    // only by B-3a: it runs on a side stream, beside B-0 and the reverse chain
    // (both chains leave most of each SM idle), and joins before B-3a.
    cudaStream_t side;
    if ((e = side_stream(&side))) return e;
    cudaEvent_t fork, join;
    if ((e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming))) return e;
    if ((e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming))) {
        cudaEventDestroy(fork);
        return e;
    }
    // released once the device is done with them
    struct Events {
        cudaEvent_t a, b;
        ~Events() { cudaEventDestroy(a); cudaEventDestroy(b); }
    } ev{fork, join};
    if ((e = cudaEventRecord(fork, s)) || (e = cudaStreamWaitEvent(side, fork, 0))) return e;
    {
        ProfScope ps(kBwdStates, side);
        bwd_states_kernel<Tin, D><<<(unsigned)chains, 256, sm1, side>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    if ((e = cudaEventRecord(join, side))) return e;
    {
        ProfScope ps(kBwdPrep, s);
        bwd_prep_kernel<Tin, D><<<(unsigned)chunks, 256, sm0, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    {
        ProfScope ps(kBwdChain, s);
        bwd_chain_kernel<Tin, D><<<(unsigned)chains, 256, sm2, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    if ((e = cudaStreamWaitEvent(s, join, 0))) return e;
    {
        ProfScope ps(kBwdStateGrads, s);
        bwd_state_grads_kernel<Tin, D><<<(unsigned)chunks, 256, sm3a, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    {
        ProfScope ps(kBwdLocal, s);
        bwd_local_grads_kernel<Tin, D><<<(unsigned)chunks, 256, sm3b, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_bwd_simt(const BwdArgs& a, mdn_dtype dt, cudaStream_t s)
{
    if (dt == MDN_F32)
        return a.D == 64 ? launch_bwd_typed<float, 64>(a, s) : launch_bwd_typed<float, 128>(a, s);
    return a.D == 64 ? launch_bwd_typed<__nv_bfloat16, 64>(a, s)
                     : launch_bwd_typed<__nv_bfloat16, 128>(a, s);
}

}  // namespace mdn
