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
    if (tid < C) {
        const int t = n * C + tid;
        alpha_s[tid] = t < a.T ? expf(a.alpha_log[tok_idx(a, b, t, h)]) : 1.f;
    }
    __syncthreads();
    const float* G = a.gamma + chunk * C * C;
    float* att = a.att + chunk * C * C;
    for (int idx = tid; idx < C * C; idx += 256) {
        const int r = idx / C, i = idx % C;
        float av = 0.f, tv = 0.f;
        if (i <= r) {
            float kk = 0.f, qk = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; ++c) {
                const float ki = Ks[i * KS + c];
                kk = fmaf(Ks[r * KS + c], ki, kk);
                qk = fmaf(Qs[r * KS + c], ki, qk);
            }
            tv = qk * G[r * C + i];
            if (i < r) av = alpha_s[r] * kk * G[(r - 1) * C + i];
        }
        As[r * AS + i] = av;
        att[idx] = tv;
    }
    __syncthreads();
    // unit lower-triangular inverse by forward substitution, one column per thread
    if (tid < C) {
        const int c = tid;
        for (int r = 0; r < C; ++r) {
            float s = 0.f;
            if (r == c) {
                s = 1.f;
            } else if (r > c) {
                for (int i = c; i < r; ++i) s = fmaf(-As[r * AS + i], Ts[i * AS + c], s);
            }
            Ts[r * AS + c] = s;
        }
    }
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
    constexpr int NS = NSB, KS = D + 1, VS = NS + 1;
    constexpr int EPT = D * NS / 256;
    extern __shared__ float smem[];
    float* Ss = smem;              // [D][NS]
    float* Ms = Ss + D * NS;
    float* Ks = Ms + D * NS;       // [C][D+1]
    float* Vs = Ks + C * KS;       // [C][NS+1]
    float* gl = Vs + C * VS;       // [C] Gamma_{C,r}
    float* wv = gl + C;            // [C] w_r
    float* scal = wv + C;          // alphabar_C, b_C, mubar_C
    const int tid = threadIdx.x;
    const int slice = blockIdx.x % (D / NS);
    const long long bh = blockIdx.x / (D / NS);
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const int j0 = slice * NS, j = tid % NS, rg = tid / NS;
    const size_t st = (size_t)bh * D * D;
    for (int e = 0; e < EPT; ++e) {
        const int i = rg + 8 * e;
        Ss[i * NS + j] = a.S0 ? a.S0[st + (size_t)i * D + j0 + j] : 0.f;
        Ms[i * NS + j] = a.M0 ? a.M0[st + (size_t)i * D + j0 + j] : 0.f;
    }
    for (int n = 0; n < a.NT; ++n) {
        const size_t chunk = (size_t)bh * a.NT + n;
        const size_t crow = chunk * C;
        float* SSn = a.SS + chunk * 2 * D * D;
        __syncthreads();
        for (int e = 0; e < EPT; ++e) {
            const int i = rg + 8 * e;
            SSn[(size_t)i * D + j0 + j] = Ss[i * NS + j];
            SSn[(size_t)D * D + (size_t)i * D + j0 + j] = Ms[i * NS + j];
        }
        for (int idx = tid; idx < C * D; idx += 256) {
            const int r = idx / D, c = idx % D, t = n * C + r;
            Ks[r * KS + c] = t < a.T ? ldt<Tin>(a.k, tok_idx(a, b, t, h) * D + c) : 0.f;
        }
        for (int idx = tid; idx < C * NS; idx += 256) {
            const int r = idx / NS, c = idx % NS, t = n * C + r;
            Vs[r * VS + c] = t < a.T ? ldt<Tin>(a.vt, tok_idx(a, b, t, h) * D + j0 + c) : 0.f;
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
#pragma unroll 4
        for (int e = 0; e < EPT; ++e) {
            const int i = rg + 8 * e;
            float dS = 0.f, dM = 0.f;
            for (int r = 0; r < C; ++r) {
                const float kv = Ks[r * KS + i] * Vs[r * VS + j];
                dS = fmaf(kv, gl[r], dS);
                dM = fmaf(kv, wv[r], dM);
            }
            const float s = Ss[i * NS + j], m = Ms[i * NS + j];
            Ss[i * NS + j] = scal[0] * s - scal[1] * m + dS;
            Ms[i * NS + j] = scal[2] * m - dM;
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
    constexpr int NS = NSB, KS = D + 1, VS = NS + 1, AS = C + 1;
    constexpr int EPT = D * NS / 256;   // state entries per thread
    constexpr int RPT = C * NS / 256;   // chunk rows per thread
    extern __shared__ float smem[];
    float* dSs = smem;             // [D][NS]
    float* dMs = dSs + D * NS;
    float* Ks = dMs + D * NS;      // [C][D+1]
    float* Qs = Ks + C * KS;       // [C][D+1]
    float* Att = Qs + C * KS;      // [C][C+1]
    float* Tm = Att + C * AS;      // [C][C+1]
    float* dOs = Tm + C * AS;      // [C][NS+1]
    float* X = dOs + C * VS;       // [C][NS+1]  dVtilde, then dY
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
    const int j0 = slice * NS, j = tid % NS, rg = tid / NS;
    const size_t st = (size_t)bh * D * D;
    for (int e = 0; e < EPT; ++e) {
        const int i = rg + 8 * e;
        dSs[i * NS + j] = a.dS_T ? a.dS_T[st + (size_t)i * D + j0 + j] : 0.f;
        dMs[i * NS + j] = a.dM_T ? a.dM_T[st + (size_t)i * D + j0 + j] : 0.f;
    }
    for (int n = a.NT - 1; n >= 0; --n) {
        const size_t chunk = (size_t)bh * a.NT + n;
        const size_t crow = chunk * C;
        float* dSSn = a.dSS + chunk * 2 * D * D;
        __syncthreads();
        for (int e = 0; e < EPT; ++e) {
            const int i = rg + 8 * e;
            dSSn[(size_t)i * D + j0 + j] = dSs[i * NS + j];
            dSSn[(size_t)D * D + (size_t)i * D + j0 + j] = dMs[i * NS + j];
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
#pragma unroll
        for (int e = 0; e < RPT; ++e) {
            const int r = rg + 8 * e;
            float kds = 0.f, kdm = 0.f, ad = 0.f;
            for (int i = 0; i < D; ++i) {
                const float kv = Ks[r * KS + i];
                kds = fmaf(kv, dSs[i * NS + j], kds);
                kdm = fmaf(kv, dMs[i * NS + j], kdm);
            }
            for (int r2 = r; r2 < C; ++r2) ad = fmaf(Att[r2 * AS + r], dOs[r2 * VS + j], ad);
            X[r * VS + j] = ad + gl[r] * kds - wv[r] * kdm;
        }
        __syncthreads();
        float dy[RPT];
#pragma unroll
        for (int e = 0; e < RPT; ++e) {
            const int r = rg + 8 * e;
            float s = 0.f;
            for (int r2 = r; r2 < C; ++r2) s = fmaf(Tm[r2 * AS + r], X[r2 * VS + j], s);
            dy[e] = s;
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < RPT; ++e) {
            const int r = rg + 8 * e, t = n * C + r;
            X[r * VS + j] = dy[e];
            if (t < a.T) a.dv[tok_idx(a, b, t, h) * D + j0 + j] = dy[e];
        }
        __syncthreads();
        const float aC = scal[0], bC = scal[1], mC = scal[2];
#pragma unroll 4
        for (int e = 0; e < EPT; ++e) {
            const int i = rg + 8 * e;
            float qs = 0.f, qm = 0.f, ks = 0.f, km = 0.f;
            for (int r = 0; r < C; ++r) {
                const float qd = Qs[r * KS + i] * dOs[r * VS + j];
                const float kd = Ks[r * KS + i] * X[r * VS + j];
                qs = fmaf(qd, abar[r], qs);
                qm = fmaf(qd, bco[r], qm);
                ks = fmaf(kd, abar[r], ks);
                km = fmaf(kd, d2[r], km);
            }
            const float ds = dSs[i * NS + j], dm = dMs[i * NS + j];
            dSs[i * NS + j] = aC * ds + qs - ks;
            dMs[i * NS + j] = -bC * ds + mC * dm - qm + km;
        }
    }
    __syncthreads();
    for (int e = 0; e < EPT; ++e) {
        const int i = rg + 8 * e;
        a.dS0[st + (size_t)i * D + j0 + j] = dSs[i * NS + j];
        a.dM0[st + (size_t)i * D + j0 + j] = dMs[i * NS + j];
    }
}

// ------------------------------------------------------------------ B-3a
// Products with the entering states S, M and the leaving adjoints dS, dM:
// P1 = dO S^T, P2 = dO M^T, P3 = Vt dS^T, P4 = Vt dM^T, P5 = dY S^T,
// P6 = dY M^T (C x d_k each), streamed over panels of KP rows of d_k.
// Writes dq's and dk's parts from them, and per chunk the coefficient
// adjoints they carry (row sums) plus <S,dS>, <M,dS>, <M,dM>.
constexpr int KP = 16;

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
    const int r = tid >> 2, q4 = tid & 3;  // row of the chunk; k = k0 + q4 + 4m
    const int t = n * C + r;
    const float abar = expf(a.la[crow + r]), bco = a.bco[crow + r];
    const float al = t < a.T ? expf(a.alpha_log[tok_idx(a, b, t, h)]) : 1.f;
    const float d2 = r > 0 ? a.bco[crow + r - 1] * al : 0.f;
    const float gl = a.gamma[chunk * C * C + (C - 1) * C + r];
    const float et = t < a.T ? a.eta[tok_idx(a, b, t, h)] : 0.f;
    const float w = et * expf(a.lm[crow + C - 1] - a.lm[crow + r]);
    float sa = 0.f, sb = 0.f, sd2 = 0.f, sgl = 0.f, sw = 0.f;
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
        float p[6][KP / 4];
#pragma unroll
        for (int m = 0; m < KP / 4; ++m)
#pragma unroll
            for (int u = 0; u < 6; ++u) p[u][m] = 0.f;
        for (int c = 0; c < D; ++c) {
            const float o = dOs[r * TS + c], vv = Vts[r * TS + c], y = dYs[r * TS + c];
#pragma unroll
            for (int m = 0; m < KP / 4; ++m) {
                const int kk = q4 + 4 * m;
                const float sv = Pn[kk * TS + c], mv = Pn[KP * TS + kk * TS + c];
                const float dsv = Pn[2 * KP * TS + kk * TS + c];
                const float dmv = Pn[3 * KP * TS + kk * TS + c];
                p[0][m] = fmaf(o, sv, p[0][m]);
                p[1][m] = fmaf(o, mv, p[1][m]);
                p[2][m] = fmaf(vv, dsv, p[2][m]);
                p[3][m] = fmaf(vv, dmv, p[3][m]);
                p[4][m] = fmaf(y, sv, p[4][m]);
                p[5][m] = fmaf(y, mv, p[5][m]);
            }
        }
        if (t < a.T) {
#pragma unroll
            for (int m = 0; m < KP / 4; ++m) {
                const int k = k0 + q4 + 4 * m;
                const size_t g = tok_idx(a, b, t, h) * D + k;
                const float kv = ldt<Tin>(a.k, g);
                const float qh = ldt<Tin>(a.q, g) - a.dcorr * kv;
                a.dq[g] = abar * p[0][m] - bco * p[1][m];
                a.dk[g] = gl * p[2][m] - w * p[3][m] - abar * p[4][m] + d2 * p[5][m];
                sa = fmaf(qh, p[0][m], sa);
                sa = fmaf(-kv, p[4][m], sa);
                sb = fmaf(-qh, p[1][m], sb);
                sd2 = fmaf(kv, p[5][m], sd2);
                sgl = fmaf(kv, p[2][m], sgl);
                sw = fmaf(-kv, p[3][m], sw);
            }
        }
    }
    // the four threads of a row hold its partial sums
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        sa += __shfl_xor_sync(0xffffffffu, sa, off);
        sb += __shfl_xor_sync(0xffffffffu, sb, off);
        sd2 += __shfl_xor_sync(0xffffffffu, sd2, off);
        sgl += __shfl_xor_sync(0xffffffffu, sgl, off);
        sw += __shfl_xor_sync(0xffffffffu, sw, off);
    }
    float* rec = a.crec_bw + chunk * kBwdRec;
    if (q4 == 0) {
        rec[r] = sa;
        rec[C + r] = sb;
        rec[2 * C + r] = sd2;
        rec[3 * C + r] = sgl;
        rec[4 * C + r] = sw;
    }
    __syncthreads();
    if (tid < 3) {
        float s = 0.f;
        for (int w8 = 0; w8 < 8; ++w8) s += red[w8 * 3 + tid];
        rec[5 * C + tid] = s;
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
    float* v_al = dG + C * AS;     // alpha
    float* v_be = v_al + C;        // beta
    float* v_et = v_be + C;        // eta
    float* v_la = v_et + C;        // la (chunk-local cumulative log alpha)
    float* v_lm = v_la + C;        // lm
    float* v_b = v_lm + C;         // b
    float* v_da = v_b + C;         // d alpha (direct)
    float* v_db = v_da + C;        // adjoint of b
    float* v_dla = v_db + C;       // adjoint of la
    float* v_dlm = v_dla + C;      // adjoint of lm
    float* v_de = v_dlm + C;       // adjoint of eta
    float* v_dbe = v_de + C;       // adjoint of beta
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
    // the four C x C products, 16 entries per thread
    constexpr int EC = C * C / 256;
    float dov[EC], qk[EC], dyv[EC], kk[EC];
#pragma unroll
    for (int e = 0; e < EC; ++e) {
        const int idx = tid + 256 * e, r = idx / C, i = idx % C;
        float x1 = 0.f, x2 = 0.f, x3 = 0.f, x4 = 0.f;
        if (i <= r) {
#pragma unroll 4
            for (int c = 0; c < D; ++c) {
                const float vi = Vts[i * TS + c], ki = Ks[i * TS + c];
                x1 = fmaf(dOs[r * TS + c], vi, x1);
                x2 = fmaf(Qs[r * TS + c], ki, x2);
                x3 = fmaf(dYs[r * TS + c], vi, x3);
                x4 = fmaf(Ks[r * TS + c], ki, x4);
            }
        }
        dov[e] = x1;
        qk[e] = x2;
        dyv[e] = x3;
        kk[e] = x4;
    }
    __syncthreads();  // dO and dY tiles are no longer read; Gp is complete
    float* dOVG = dOs;  // [C][C+1]
    float* dPK = dYs;   // [C][C+1]
#pragma unroll
    for (int e = 0; e < EC; ++e) {
        const int idx = tid + 256 * e, r = idx / C, i = idx % C;
        const float g = v_et[i] * Gp[r * AS + i];
        float ovg = 0.f, pk = 0.f, dg = 0.f;
        if (i <= r) {
            ovg = dov[e] * g;
            dg = dov[e] * qk[e];
        }
        if (i < r) pk = -dyv[e] * v_et[i] * Gp[(r - 1) * AS + i];  // dA o Gamma-
        dOVG[r * AS + i] = ovg;
        dPK[r * AS + i] = pk;
        dG[r * AS + i] = dg;
    }
    __syncthreads();
    // Gamma-_{r,i} = Gamma_{r-1,i}: dA o (P K^T) lands on row r - 1 (one writer per entry)
#pragma unroll
    for (int e = 0; e < EC; ++e) {
        const int idx = tid + 256 * e, r = idx / C, i = idx % C;
        if (i < r) dG[(r - 1) * AS + i] += -dyv[e] * v_al[r] * kk[e];
    }
    const float* rec = a.crec_bw + chunk * kBwdRec;
    __syncthreads();
    if (tid < C) dG[(C - 1) * AS + tid] += rec[3 * C + tid];  // Gamma_{C,i} in the state update
    // dQhat += dOVG K ; dK += dOVG^T Qhat + dPK^T P + Diag(alpha) dPK K ; d alpha from P
    {
        const int r = tid >> 2, q4 = tid & 3, t = n * C + r;
        const float alr = v_al[r];
        float dar = 0.f;
        for (int c = q4; c < D; c += 4) {
            float dq = 0.f, dk = 0.f, dp = 0.f;
            for (int i = 0; i <= r; ++i) dq = fmaf(dOVG[r * AS + i], Ks[i * TS + c], dq);
            for (int r2 = r; r2 < C; ++r2) dk = fmaf(dOVG[r2 * AS + r], Qs[r2 * TS + c], dk);
            for (int r2 = r + 1; r2 < C; ++r2)
                dk = fmaf(dPK[r2 * AS + r] * v_al[r2], Ks[r2 * TS + c], dk);
            for (int i = 0; i < r; ++i) dp = fmaf(dPK[r * AS + i], Ks[i * TS + c], dp);
            dk = fmaf(alr, dp, dk);
            dar = fmaf(dp, Ks[r * TS + c], dar);
            if (t < a.T) {
                const size_t g = tok_idx(a, b, t, h) * D + c;
                const float dqt = a.dq[g] + dq;
                a.dq[g] = dqt;
                a.dk[g] = a.dk[g] + dk - a.dcorr * dqt;
            }
        }
        dar += __shfl_xor_sync(0xffffffffu, dar, 1);
        dar += __shfl_xor_sync(0xffffffffu, dar, 2);
        if (q4 == 0) v_da[r] = dar;
    }
    __syncthreads();
    // coefficient adjoints -> la, lm, beta, eta, alpha
    if (tid < C) {
        const int r = tid;
        const float dD2 = rec[2 * C + r];
        const float b_prev = r > 0 ? v_b[r - 1] : 0.f;
        v_da[r] += dD2 * b_prev;                           // D2_r = b_{r-1} alpha_r
        float db = rec[C + r];
        if (r + 1 < C) db += rec[2 * C + r + 1] * v_al[r + 1];
        float dabar = rec[r];
        if (r == C - 1) {
            dabar += rec[5 * C];                           // alphabar_C S
            db -= rec[5 * C + 1];                          // - b_C M
        }
        v_db[r] = db;
        const float abar = expf(v_la[r]);
        v_dla[r] = dabar * abar + db * v_b[r];
        const float wr = v_et[r] * expf(v_lm[C - 1] - v_lm[r]);
        const float dw = rec[4 * C + r];
        v_dlm[r] = -dw * wr;
        v_de[r] = dw * expf(v_lm[C - 1] - v_lm[r]);
        v_dbe[r] = 0.f;
    }
    __syncthreads();
    if (tid == 0) {
        float s = rec[5 * C + 2] * expf(v_lm[C - 1]);      // mubar_C M
        for (int r = 0; r < C; ++r) s += rec[4 * C + r] * v_et[r] * expf(v_lm[C - 1] - v_lm[r]);
        v_dlm[C - 1] += s;
        // b_r = sum_{j<=r} exp(la_r - la_j) beta_j mubar_j: reverse recurrence
        float Rb = 0.f;
        for (int j = C - 1; j >= 0; --j) {
            Rb = v_db[j] + (j + 1 < C ? v_al[j + 1] * Rb : 0.f);
            const float mb = expf(v_lm[j]);
            const float tj = v_be[j] * mb * Rb;
            v_dbe[j] += mb * Rb;
            v_dla[j] -= tj;
            v_dlm[j] += tj;
        }
    }
    __syncthreads();
    // Gamma = eta o Gp: row and column sums of dG o Gamma, and eta's share
    if (tid < C) {
        const int x = tid;
        float rs = 0.f, cs = 0.f, ce = 0.f;
        for (int y = 0; y <= x; ++y) rs = fmaf(dG[x * AS + y], v_et[y] * Gp[x * AS + y], rs);
        for (int y = x; y < C; ++y) {
            const float gp = Gp[y * AS + x];
            cs = fmaf(dG[y * AS + x], v_et[x] * gp, cs);
            ce = fmaf(dG[y * AS + x], gp, ce);
        }
        v_dla[x] += rs;
        v_dlm[x] -= cs;
        v_de[x] += ce;
    }
    __syncthreads();
    // R_{j,i} = sum_{r>=j} dG_{r,i} exp(la_r - la_j), in place, one column per thread
    if (tid < C) {
        const int i = tid;
        float R = 0.f;
        for (int j = C - 1; j >= i; --j) {
            R = dG[j * AS + i] + (j + 1 < C ? v_al[j + 1] * R : 0.f);
            dG[j * AS + i] = R;
        }
    }
    __syncthreads();
    // U_j = sum_{i<=j} eta_i exp(lm_j - lm_i) R_{j,i}
    if (tid < C) {
        const int j = tid;
        float U = 0.f;
        for (int i = 0; i <= j; ++i) U = fmaf(v_et[i] * expf(v_lm[j] - v_lm[i]), dG[j * AS + i], U);
        v_dbe[j] += U;
        v_dla[j] -= v_be[j] * U;
        v_dlm[j] += v_be[j] * U;
    }
    __syncthreads();
    if (tid == 0) {
        // reverse cumulative sums: la, lm are inclusive prefix sums of the log gates
        float sla = 0.f, slm = 0.f;
        for (int j = C - 1; j >= 0; --j) {
            sla += v_dla[j];
            slm += v_dlm[j];
            v_dla[j] = sla;
            v_dlm[j] = slm;
        }
    }
    __syncthreads();
    if (tid < C) {
        const int j = tid, t = n * C + j;
        if (t < a.T) {
            const size_t gi = tok_idx(a, b, t, h);
            a.dalpha_log[gi] = v_da[j] * v_al[j] + v_dla[j];
            a.dmu_log[gi] = v_dlm[j];
            a.dbeta[gi] = v_dbe[j];
            a.deta[gi] = v_de[j];
        }
    }
}

template <typename Tin, int D>
cudaError_t launch_bwd_typed(const BwdArgs& a, cudaStream_t s)
{
    const long long chunks = (long long)a.B * a.H * a.NT;
    const long long chains = (long long)a.B * a.H * (D / NSB);
    const size_t sm0 = sizeof(float) * (2 * C * (D + 1) + 2 * C * (C + 1) + C);
    const size_t sm1 = sizeof(float) * (2 * D * NSB + C * (D + 1) + C * (NSB + 1) + 2 * C + 4);
    const size_t sm2 = sizeof(float) * (2 * D * NSB + 2 * C * (D + 1) + 2 * C * (C + 1) +
                                        2 * C * (NSB + 1) + 5 * C + 4);
    const size_t sm3a = sizeof(float) * (3 * C * (D + 1) + 4 * KP * (D + 1) + 24);
    const size_t sm3b = sizeof(float) * (5 * C * (D + 1) + 2 * C * (C + 1) + 12 * C);
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
    {
        ProfScope ps(kBwdPrep, s);
        bwd_prep_kernel<Tin, D><<<(unsigned)chunks, 256, sm0, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    {
        ProfScope ps(kBwdStates, s);
        bwd_states_kernel<Tin, D><<<(unsigned)chains, 256, sm1, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    {
        ProfScope ps(kBwdChain, s);
        bwd_chain_kernel<Tin, D><<<(unsigned)chains, 256, sm2, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
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
