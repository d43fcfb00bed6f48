// K-2, K-3, K-4 on CUDA cores in fp32: the chunkwise MDN forward pass.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, steps 3-4.  Per chunk of C = 64 tokens (states
// S, M entering the chunk; r, i index positions inside the chunk):
//
//   K-2 (intra, parallel over chunks)
//     A     = (P K^T) o Gamma-,   P = Diag(alpha) K,  Gamma-_{r,i} = Gamma_{r-1,i}, i < r
//     [U | Y | Z] = (I + A)^{-1} [V | Diag(alphabar_{r-1} alpha_r) K | Diag(b_{r-1} alpha_r) K]
//       (forward substitution, one right-hand-side column per thread)
//   K-3 (inter, sequential over chunks, parallel over heads and d_v slices)
//     Vtilde = U - Y S + Z M
//     Oi     = Diag(alphabar) Qhat S - Diag(b) Qhat M      (carried-state part of o)
//     S'     = alphabar_C S - b_C M + K^T Diag(Gamma_{C,.}) Vtilde
//     M'     = mubar_C M - K^T Diag(eta_i mubar_C / mubar_i) Vtilde
//   K-4 (output, parallel over chunks)
//     O      = Oi + ((Qhat K^T) o Gamma) Vtilde
//
// "alphabar_{0->C-1}" and "b_{0->C-1}" in the pages' Y and Z are read as the
// values at the previous position (alphabar_0 = 1, b_0 = 0), which makes
// Diag(alphabar_{r-1}) P = Diag(alphabar_{r-1} alpha_r) K.  Columns of d_v are
// independent in K-3 (Vtilde[:, j] and S[:, j], M[:, j] only touch column j),
// so K-3 splits d_v into slices of 32 columns, one block each.
//
// This path computes in fp32 throughout and serves fp32 inputs (and bf16
// inputs when asked); bf16 inputs normally take the tensor-core path.
#include "mdn_internal.cuh"

namespace mdn {
namespace {

template <typename Tin>
__device__ __forceinline__ float ld_tok(const void* base, size_t idx) {
    return ld_elem(static_cast<const Tin*>(base) + idx);
}

// ------------------------------------------------------------------ K-2
template <typename Tin, int D>
__global__ void __launch_bounds__(128)
intra_simt_kernel(ChunkArgs a)
{
    constexpr int C = kChunk, KS = D + 1, XS = 3 * D, AS = C + 1;
    extern __shared__ float smem[];
    float* Ks = smem;              // [C][D+1]
    float* As = Ks + C * KS;       // [C][C+1]
    float* X = As + C * AS;        // [C][3D]
    float* alpha_s = X + C * XS;   // [C]
    float* sy = alpha_s + C;       // [C] alphabar_{r-1} alpha_r
    float* sz = sy + C;            // [C] b_{r-1} alpha_r

    const int tid = threadIdx.x;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const long long chunk = blockIdx.x;
    const size_t crow = (size_t)bh * a.NT * C + (size_t)n * C;  // row of la/bco

    for (int idx = tid; idx < C * D; idx += blockDim.x) {
        const int r = idx / D, c = idx % D;
        const int t = n * C + r;
        float kv = 0.f, vv = 0.f;
        if (t < a.T) {
            const size_t g = (((size_t)b * a.T + t) * a.H + h) * D + c;
            kv = ld_tok<Tin>(a.k, g);
            vv = ld_tok<Tin>(a.v, g);
        }
        Ks[r * KS + c] = kv;
        X[r * XS + c] = vv;
    }
    if (tid < C) {
        const int r = tid, t = n * C + r;
        float ar = 1.f;
        if (t < a.T) {
            float al, ml, be, et;
            gates_at(a.gates(), ((size_t)b * a.T + t) * a.H + h, al, ml, be, et);
            ar = expf(al);
        }
        const float abar_prev = (r > 0) ? expf(a.la[crow + r - 1]) : 1.f;
        const float b_prev = (r > 0) ? a.bco[crow + r - 1] : 0.f;
        alpha_s[r] = ar;
        sy[r] = abar_prev * ar;
        sz[r] = b_prev * ar;
    }
    __syncthreads();

    const float* G = a.gamma + (size_t)chunk * C * C;
    for (int idx = tid; idx < C * C; idx += blockDim.x) {
        const int r = idx / C, i = idx % C;
        float val = 0.f;
        if (i < r) {
            float dot = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; ++c) dot = fmaf(Ks[r * KS + c], Ks[i * KS + c], dot);
            val = alpha_s[r] * dot * G[(r - 1) * C + i];
        }
        As[r * AS + i] = val;
    }
    for (int idx = tid; idx < C * 2 * D; idx += blockDim.x) {
        const int r = idx / (2 * D), c = idx % (2 * D);
        const float kv = Ks[r * KS + (c % D)];
        X[r * XS + D + c] = (c < D ? sy[r] : sz[r]) * kv;
    }
    __syncthreads();

    // Forward substitution: X_r -= sum_{i<r} A_{r,i} X_i, column by column.
    for (int c = tid; c < XS; c += blockDim.x) {
        for (int r = 1; r < C; ++r) {
            float acc = X[r * XS + c];
            for (int i = 0; i < r; ++i) acc = fmaf(-As[r * AS + i], X[i * XS + c], acc);
            X[r * XS + c] = acc;
        }
    }
    __syncthreads();

    const size_t out = (size_t)chunk * C * D;
    for (int idx = tid; idx < C * D; idx += blockDim.x) {
        const int r = idx / D, c = idx % D;
        a.U[out + idx] = X[r * XS + c];
        a.Y[out + idx] = X[r * XS + D + c];
        a.Z[out + idx] = X[r * XS + 2 * D + c];
    }
}

// ------------------------------------------------------------------ K-3
constexpr int kSlice = 32;  // d_v columns per block

template <typename Tin, int D>
__global__ void __launch_bounds__(256)
inter_simt_kernel(ChunkArgs a)
{
    constexpr int C = kChunk, NS = kSlice, KS = D + 1, VS = NS + 1;
    constexpr int RPT = C * NS / 256;   // Vtilde / Oi outputs per thread
    constexpr int EPT = D * NS / 256;   // state entries per thread
    extern __shared__ float smem[];
    float* Ss = smem;              // [D][NS]
    float* Ms = Ss + D * NS;       // [D][NS]
    float* tile = Ms + D * NS;     // [C][D+1]
    float* Vs = tile + C * KS;     // [C][NS+1]
    float* abar_s = Vs + C * VS;   // [C]
    float* b_s = abar_s + C;       // [C]
    float* wS = b_s + C;           // [C] Gamma_{C,r}
    float* wM = wS + C;            // [C] eta_r mubar_C / mubar_r
    float* scal = wM + C;          // [3] alphabar_C, b_C, mubar_C

    const int tid = threadIdx.x;
    const int nslices = D / NS;
    const int slice = blockIdx.x % nslices;
    const Chain ch = chain_of(a, blockIdx.x / nslices);
    const int b = ch.b, h = ch.h;
    const int j0 = slice * NS;
    const int j = tid % NS;        // column inside the slice
    const int rg = tid / NS;       // 0..7

    const size_t st_base = (size_t)ch.sh * D * D;
    for (int e = 0; e < EPT; ++e) {
        const int i = rg + 8 * e;
        Ss[i * NS + j] = a.S0 ? a.S0[st_base + (size_t)i * D + j0 + j] : 0.f;
        Ms[i * NS + j] = a.M0 ? a.M0[st_base + (size_t)i * D + j0 + j] : 0.f;
    }

    for (int nc = 0; nc < ch.nt; ++nc) {
        const int n = ch.n0 + nc;  // chunk of the input rows
        const size_t chunk = (size_t)ch.chunk0 + nc;
        const size_t crow = chunk * C;
        const size_t cmat = chunk * C * D;
        __syncthreads();  // previous chunk's state update is complete
        // Y tile and the per-position coefficients.
        for (int idx = tid; idx < C * D; idx += 256) tile[(idx / D) * KS + idx % D] = a.Y[cmat + idx];
        if (tid < C) {
            const int r = tid, t = n * C + r;
            abar_s[r] = expf(a.la[crow + r]);
            b_s[r] = a.bco[crow + r];
            wS[r] = a.gamma[chunk * C * C + (C - 1) * C + r];
            float et = 0.f;
            if (t < a.T) {
                float al, ml, be;
                gates_at(a.gates(), ((size_t)b * a.T + t) * a.H + h, al, ml, be, et);
            }
            wM[r] = et * expf(a.lm[crow + C - 1] - a.lm[crow + r]);
            if (r == 0) {
                scal[0] = expf(a.la[crow + C - 1]);
                scal[1] = a.bco[crow + C - 1];
                scal[2] = expf(a.lm[crow + C - 1]);
            }
        }
        __syncthreads();
        float acc[RPT];
#pragma unroll
        for (int e = 0; e < RPT; ++e) {
            const int r = rg + 8 * e;
            float s = a.U[cmat + (size_t)r * D + j0 + j];
            for (int i = 0; i < D; ++i) s = fmaf(-tile[r * KS + i], Ss[i * NS + j], s);
            acc[e] = s;
        }
        __syncthreads();
        for (int idx = tid; idx < C * D; idx += 256) tile[(idx / D) * KS + idx % D] = a.Z[cmat + idx];
        __syncthreads();
#pragma unroll
        for (int e = 0; e < RPT; ++e) {
            const int r = rg + 8 * e;
            float s = acc[e];
            for (int i = 0; i < D; ++i) s = fmaf(tile[r * KS + i], Ms[i * NS + j], s);
            Vs[r * VS + j] = s;
            const int t = nc * C + r;  // token of the chain
            if (t < ch.len)
                st_elem(static_cast<Tin*>(a.vt) + ((size_t)(ch.out0 + t) * a.H + h) * D + j0 + j, s);
        }
        __syncthreads();
        // Qhat tile, then the carried-state part of o.
        for (int idx = tid; idx < C * D; idx += 256) {
            const int r = idx / D, c = idx % D, t = n * C + r;
            float qh = 0.f;
            if (t < a.T) {
                const size_t g = (((size_t)b * a.T + t) * a.H + h) * D + c;
                qh = ld_tok<Tin>(a.q, g) - a.dcorr * ld_tok<Tin>(a.k, g);
            }
            tile[r * KS + c] = qh;
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < RPT; ++e) {
            const int r = rg + 8 * e;
            float s1 = 0.f, s2 = 0.f;
            for (int i = 0; i < D; ++i) {
                const float qv = tile[r * KS + i];
                s1 = fmaf(qv, Ss[i * NS + j], s1);
                s2 = fmaf(qv, Ms[i * NS + j], s2);
            }
            a.Oi[crow * D + (size_t)r * D + j0 + j] = abar_s[r] * s1 - b_s[r] * s2;
        }
        __syncthreads();
        // K tile, then the state update.
        for (int idx = tid; idx < C * D; idx += 256) {
            const int r = idx / D, c = idx % D, t = n * C + r;
            tile[r * KS + c] = (t < a.T)
                ? ld_tok<Tin>(a.k, (((size_t)b * a.T + t) * a.H + h) * D + c) : 0.f;
        }
        __syncthreads();
        const float abarC = scal[0], bC = scal[1], mubarC = scal[2];
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
            const int i = rg + 8 * e;
            float dS = 0.f, dM = 0.f;
            for (int r = 0; r < C; ++r) {
                const float kv = tile[r * KS + i] * Vs[r * VS + j];
                dS = fmaf(kv, wS[r], dS);
                dM = fmaf(kv, wM[r], dM);
            }
            const float s = Ss[i * NS + j], m = Ms[i * NS + j];
            Ss[i * NS + j] = abarC * s - bC * m + dS;
            Ms[i * NS + j] = mubarC * m - dM;
        }
    }
    __syncthreads();
    for (int e = 0; e < EPT; ++e) {
        const int i = rg + 8 * e;
        a.S_T[st_base + (size_t)i * D + j0 + j] = Ss[i * NS + j];
        a.M_T[st_base + (size_t)i * D + j0 + j] = Ms[i * NS + j];
    }
}

// ------------------------------------------------------------------ K-4
template <typename Tin, int D>
__global__ void __launch_bounds__(256)
output_simt_kernel(ChunkArgs a)
{
    constexpr int C = kChunk, KS = D + 1, AS = C + 1;
    extern __shared__ float smem[];
    float* Qs = smem;              // [C][D+1]  qhat
    float* Ks = Qs + C * KS;       // [C][D+1]
    float* As = Ks + C * KS;       // [C][C+1]  (Qhat K^T) o Gamma
    float* Vs = As + C * AS;       // [C][D]    Vtilde

    const int tid = threadIdx.x;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const size_t chunk = blockIdx.x;
    const ChunkOut co = chunk_out(a, b, n);  // where this chunk's rows of vt and o live
    for (int idx = tid; idx < C * D; idx += 256) {
        const int r = idx / D, c = idx % D, t = n * C + r;
        float qv = 0.f, kv = 0.f, vv = 0.f;
        if (r < co.valid) {
            const size_t g = (((size_t)b * a.T + t) * a.H + h) * D + c;
            kv = ld_tok<Tin>(a.k, g);
            qv = ld_tok<Tin>(a.q, g) - a.dcorr * kv;
            vv = ld_tok<Tin>(a.vt, ((size_t)(co.row0 + r) * a.H + h) * D + c);
        }
        Qs[r * KS + c] = qv;
        Ks[r * KS + c] = kv;
        Vs[r * D + c] = vv;
    }
    __syncthreads();
    const float* G = a.gamma + chunk * C * C;
    for (int idx = tid; idx < C * C; idx += 256) {
        const int r = idx / C, i = idx % C;
        float val = 0.f;
        if (i <= r) {
            float dot = 0.f;
#pragma unroll 8
            for (int c = 0; c < D; ++c) dot = fmaf(Qs[r * KS + c], Ks[i * KS + c], dot);
            val = dot * G[r * C + i];
        }
        As[r * AS + i] = val;
    }
    __syncthreads();
    const size_t orow = chunk * C * D;  // Oi is [B*H, NT*C, D]
    for (int idx = tid; idx < C * D; idx += 256) {
        const int r = idx / D, c = idx % D;
        float s = a.Oi[orow + idx];
        for (int i = 0; i <= r; ++i) s = fmaf(As[r * AS + i], Vs[i * D + c], s);
        if (r < co.valid)
            st_elem(static_cast<Tin*>(a.o) + ((size_t)(co.row0 + r) * a.H + h) * D + c, s);
    }
}

template <typename Tin, int D>
cudaError_t launch_simt_typed(const ChunkArgs& a, cudaStream_t s)
{
    constexpr int C = kChunk;
    const long long chunks = (long long)a.B * a.H * a.NT;
    const size_t smem2 = sizeof(float) * (C * (D + 1) + C * (C + 1) + C * 3 * D + 3 * C);
    const size_t smem3 = sizeof(float) * (2 * D * kSlice + C * (D + 1) + C * (kSlice + 1) + 4 * C + 4);
    const size_t smem4 = sizeof(float) * (2 * C * (D + 1) + C * (C + 1) + C * D);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(intra_simt_kernel<Tin, D>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2)))
        return e;
    if ((e = cudaFuncSetAttribute(inter_simt_kernel<Tin, D>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3)))
        return e;
    if ((e = cudaFuncSetAttribute(output_simt_kernel<Tin, D>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem4)))
        return e;
    {
        ProfScope ps(kIntraSimt, s);
        intra_simt_kernel<Tin, D><<<(unsigned)chunks, 128, smem2, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    {
        ProfScope ps(kInterSimt, s);
        const long long chains = a.cu_chunks ? (long long)a.nseq * a.H : (long long)a.B * a.H;
        inter_simt_kernel<Tin, D><<<(unsigned)(chains * (D / kSlice)), 256, smem3, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    {
        ProfScope ps(kOutputSimt, s);
        output_simt_kernel<Tin, D><<<(unsigned)chunks, 256, smem4, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs& a, mdn_dtype dt, cudaStream_t s)
{
    if (dt == MDN_F32) {
        return a.D == 64 ? launch_simt_typed<float, 64>(a, s) : launch_simt_typed<float, 128>(a, s);
    }
    return a.D == 64 ? launch_simt_typed<__nv_bfloat16, 64>(a, s)
                     : launch_simt_typed<__nv_bfloat16, 128>(a, s);
}

}  // namespace mdn
