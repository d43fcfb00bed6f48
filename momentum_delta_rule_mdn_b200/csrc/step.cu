// K-5: one decode token, the stepwise recurrence applied in place.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 1; ijyty.com article, section 6 (decoding
// switches to the token-by-token recurrence):
//   vtilde_j = v_j - alpha sum_i S_ij k_i
//   M_ij <- mu M_ij - eta k_i vtilde_j
//   S_ij <- alpha S_ij - beta M_ij
//   o_j   = sum_i S_ij (q_i - d k_i)
//
// Bound by HBM: each state element is read once and written once.  Columns
// are independent, so one block owns one (b, h) and NC columns (64 for large
// batches; 32 or 16 when fewer blocks would leave SMs idle); a thread owns RP
// rows x 4 adjacent columns (float4).  The two column sums over rows reduce
// within a warp by shuffles, then across the 8 warps in shared memory.  All
// state loads are issued before the first reduction.  On request the step also
// measures ||S_t - S_{t-1}||_F per head (article, section 8: the decoding
// diagnostic): each block adds its share of the squared norm atomically into a
// zeroed [B*H] array, and a final pass takes the square roots.  (Running the
// blocks of a head as a thread-block cluster that reduces through distributed
// shared memory saves those two small launches but measured slower on B200:
// the cluster barrier holds both blocks of a head until the slower finishes.)
#include "mdn_internal.cuh"

namespace mdn {
namespace {

// Sum of x over the lanes of this warp that share lane % CG (the row groups of
// one column group); the result is valid in every lane.
template <int CG>
__device__ __forceinline__ float rows_sum(float x) {
#pragma unroll
    for (int off = CG; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <typename Tin, int D, int NC, bool DS>
__global__ void __launch_bounds__(256)
step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
            const float* __restrict__ alpha_log, const float* __restrict__ mu_log,
            const float* __restrict__ beta, const float* __restrict__ eta, float dcorr,
            float* __restrict__ S, float* __restrict__ M, Tin* __restrict__ o,
            Tin* __restrict__ vt_out, float* __restrict__ ds_norm)
{
    constexpr int CG = NC / 4;      // float4 column groups
    constexpr int RG = 256 / CG;    // row groups
    constexpr int RP = D / RG;      // rows per thread
    constexpr int PARTS = D / NC;   // blocks per head
    static_assert(RP >= 1 && CG <= 32, "shape");
    __shared__ float ks[D], qs[D];
    __shared__ float red[8][NC];
    __shared__ float vts[NC];
    __shared__ float dsw[8];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long bh = blockIdx.x / PARTS;
    const int col_base = (blockIdx.x % PARTS) * NC;
    const int cg = tid % CG, rg = tid / CG;
    const int col = col_base + cg * 4;

    float* Sh = S + (size_t)bh * D * D;
    float* Mh = M + (size_t)bh * D * D;
    float4 s4[RP], m4[RP];
#pragma unroll
    for (int e = 0; e < RP; ++e) {
        const int i = rg * RP + e;
        s4[e] = __ldcs(reinterpret_cast<const float4*>(Sh + (size_t)i * D + col));
        m4[e] = __ldcs(reinterpret_cast<const float4*>(Mh + (size_t)i * D + col));
    }
    const float alpha = expf(alpha_log[bh]);
    const float mu = expf(mu_log[bh]);
    const float be = beta[bh];
    const float et = eta[bh];
    for (int i = tid; i < D; i += 256) {
        const float kv = ld_elem(k + (size_t)bh * D + i);
        ks[i] = kv;
        qs[i] = ld_elem(q + (size_t)bh * D + i) - dcorr * kv;
    }
    __syncthreads();

    // vtilde = v - S^T (alpha k)
    float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < RP; ++e) {
        const float kv = ks[rg * RP + e];
        p[0] = fmaf(s4[e].x, kv, p[0]);
        p[1] = fmaf(s4[e].y, kv, p[1]);
        p[2] = fmaf(s4[e].z, kv, p[2]);
        p[3] = fmaf(s4[e].w, kv, p[3]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) p[c] = rows_sum<CG>(p[c]);
    if (lane < CG) {
#pragma unroll
        for (int c = 0; c < 4; ++c) red[warp][cg * 4 + c] = p[c];
    }
    __syncthreads();
    if (tid < NC) {
        float sum = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) sum += red[g][tid];
        const float vtj = ld_elem(v + (size_t)bh * D + col_base + tid) - alpha * sum;
        vts[tid] = vtj;
        if (vt_out) st_elem(vt_out + (size_t)bh * D + col_base + tid, vtj);
    }
    __syncthreads();

    float vv[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) vv[c] = vts[cg * 4 + c];
    float po[4] = {0.f, 0.f, 0.f, 0.f};
    float ds = 0.f;  // sum of (S_t - S_{t-1})^2 over this thread's elements
#pragma unroll
    for (int e = 0; e < RP; ++e) {
        const int i = rg * RP + e;
        const float ek = et * ks[i];
        const float qv = qs[i];
        float* sp = &s4[e].x;
        float* mp = &m4[e].x;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float mnew = fmaf(mu, mp[c], -ek * vv[c]);
            const float snew = fmaf(alpha, sp[c], -be * mnew);
            ds = fmaf(snew - sp[c], snew - sp[c], ds);
            mp[c] = mnew;
            sp[c] = snew;
            po[c] = fmaf(snew, qv, po[c]);
        }
        __stcs(reinterpret_cast<float4*>(Sh + (size_t)i * D + col), s4[e]);
        __stcs(reinterpret_cast<float4*>(Mh + (size_t)i * D + col), m4[e]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) po[c] = rows_sum<CG>(po[c]);
    if (lane < CG) {
#pragma unroll
        for (int c = 0; c < 4; ++c) red[warp][cg * 4 + c] = po[c];
    }
    __syncthreads();
    if (DS) {  // this block's share of ||S_t - S_{t-1}||_F^2
        ds = rows_sum<1>(ds);
        if (lane == 0) dsw[warp] = ds;
    }
    if (tid < NC) {
        float sum = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) sum += red[g][tid];
        st_elem(o + (size_t)bh * D + col_base + tid, sum);
    }
    if (DS) {
        __syncthreads();
        if (tid == 0) {
            float t = 0.f;
#pragma unroll
            for (int g = 0; g < 8; ++g) t += dsw[g];
            atomicAdd(ds_norm + bh, t);
        }
    }
}

// In place: x <- sqrt(x) (squared norms to norms).
__global__ void sqrt_kernel(float* x, long long n)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) x[i] = sqrtf(x[i]);
}

template <typename Tin, int D>
cudaError_t launch_step_typed(const void* q, const void* k, const void* v,
                              const float* alpha_log, const float* mu_log, const float* beta,
                              const float* eta, float dcorr, float* S, float* M, int B, int H,
                              void* o, void* vt, float* ds_norm, cudaStream_t s)
{
    const long long heads = (long long)B * H;
    if (heads == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // narrowest column split that still reaches two blocks per SM
    const int nc = heads * (D / 64) >= 2LL * sms ? 64 : (heads * (D / 32) >= 2LL * sms ? 32 : 16);
    if (ds_norm && (e = cudaMemsetAsync(ds_norm, 0, heads * sizeof(float), s)) != cudaSuccess)
        return e;
    ProfScope ps(kStep, s);
    const Tin* qq = static_cast<const Tin*>(q);
    const Tin* kk = static_cast<const Tin*>(k);
    const Tin* vv = static_cast<const Tin*>(v);
    Tin* oo = static_cast<Tin*>(o);
    Tin* tt = static_cast<Tin*>(vt);
#define MDN_STEP_LAUNCH(NC_)                                                                     \
    do {                                                                                         \
        const unsigned grid = (unsigned)(heads * (D / NC_));                                     \
        if (ds_norm)                                                                             \
            step_kernel<Tin, D, NC_, true><<<grid, 256, 0, s>>>(                                 \
                qq, kk, vv, alpha_log, mu_log, beta, eta, dcorr, S, M, oo, tt, ds_norm);         \
        else                                                                                     \
            step_kernel<Tin, D, NC_, false><<<grid, 256, 0, s>>>(                                \
                qq, kk, vv, alpha_log, mu_log, beta, eta, dcorr, S, M, oo, tt, nullptr);         \
    } while (0)
    if (nc == 64) MDN_STEP_LAUNCH(64);
    else if (nc == 32) MDN_STEP_LAUNCH(32);
    else MDN_STEP_LAUNCH(16);
#undef MDN_STEP_LAUNCH
    if ((e = cudaGetLastError()) != cudaSuccess || !ds_norm) return e;
    sqrt_kernel<<<(unsigned)((heads + 255) / 256), 256, 0, s>>>(ds_norm, heads);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const void* q, const void* k, const void* v, mdn_dtype dt,
                        const float* alpha_log, const float* mu_log, const float* beta,
                        const float* eta, float dcorr, float* S, float* M, int B, int H,
                        int D, void* o, void* vt, float* ds_norm, cudaStream_t s)
{
    if (dt == MDN_F32)
        return D == 64 ? launch_step_typed<float, 64>(q, k, v, alpha_log, mu_log, beta, eta,
                                                      dcorr, S, M, B, H, o, vt, ds_norm, s)
                       : launch_step_typed<float, 128>(q, k, v, alpha_log, mu_log, beta, eta,
                                                       dcorr, S, M, B, H, o, vt, ds_norm, s);
    return D == 64 ? launch_step_typed<__nv_bfloat16, 64>(q, k, v, alpha_log, mu_log, beta, eta,
                                                          dcorr, S, M, B, H, o, vt, ds_norm, s)
                   : launch_step_typed<__nv_bfloat16, 128>(q, k, v, alpha_log, mu_log, beta,
                                                           eta, dcorr, S, M, B, H, o, vt, ds_norm, s);
}

}  // namespace mdn
