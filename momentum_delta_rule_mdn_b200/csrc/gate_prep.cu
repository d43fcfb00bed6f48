// K-1: chunk coefficients in the log domain (la, lm, lc, b) and Gamma.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 5: every cumulative product of the chunk
// (alphabar, mubar, c) is kept in the log domain, built with cumsum and
// logcumsumexp.  One warp owns one chunk of 64 positions (two per lane); the
// prefix sums and the log-sum-exp prefix are warp-shuffle scans.
//
// The gates are read as given, or computed from their pre-activations as
// they are read (the fused parameterisation, see GateSrc).
//
// Positions past the end of the sequence act as steps that leave S and M
// unchanged (alpha = mu = 1, beta = eta = 0), so a short last chunk needs no
// special case downstream.
//
// Gamma_{r,i} = eta_i (alphabar_r / mubar_i)(c_r - c_{i-1}) is accumulated
// down each column i by its first-order recurrence
//     Gamma_{r,i} = alpha_r Gamma_{r-1,i} + eta_i beta_r mubar_r / mubar_i,
// a sum of non-negative terms (mubar_r / mubar_i as a running product of mu).  Evaluating the difference c_r - c_{i-1} from
// lc (the pages' log-broadcast) cancels catastrophically in fp32 when
// mu/alpha < 1 over a run of tokens; the recurrence has no subtraction.
#include "mdn_internal.cuh"

namespace mdn {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__global__ void __launch_bounds__(128)
gate_prep_kernel(const GateSrc src, int B, int T, int H, int NT, float* __restrict__ la, float* __restrict__ lm,
                 float* __restrict__ lc, float* __restrict__ bco, float* __restrict__ gamma)
{
    const int lane = threadIdx.x & 31;
    const long long chunk = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (chunk >= (long long)B * H * NT) return;
    const int n = (int)(chunk % NT);
    const long long bh = chunk / NT;
    const int b = (int)(bh / H), h = (int)(bh % H);

    // Positions 2*lane and 2*lane+1 of chunk n.
    const int t0 = n * kChunk + 2 * lane;
    float a[2] = {0.f, 0.f}, m[2] = {0.f, 0.f}, be[2] = {0.f, 0.f}, et[2] = {0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int t = t0 + e;
        if (t < T) {
            gates_at(src, ((size_t)b * T + t) * H + h, a[e], m[e], be[e], et[e]);
        }
    }
    float la_v[2], lm_v[2], lc_v[2];
    chunk_log_coeffs(a, m, be, lane, la_v, lm_v, lc_v);

    const size_t row = (size_t)bh * NT * kChunk + (size_t)n * kChunk + 2 * lane;
    reinterpret_cast<float2*>(la + row)[0] = make_float2(la_v[0], la_v[1]);
    reinterpret_cast<float2*>(lm + row)[0] = make_float2(lm_v[0], lm_v[1]);
    reinterpret_cast<float2*>(lc + row)[0] = make_float2(lc_v[0], lc_v[1]);
    reinterpret_cast<float2*>(bco + row)[0] =
        make_float2(expf(la_v[0] + lc_v[0]), expf(la_v[1] + lc_v[1]));

    if (gamma == nullptr) return;
    // Column recurrence; this lane owns columns i0 = lane and i1 = lane + 32.
    // With f started at 0, f_r = mu_r f_{r-1} + [r == i] is mubar_r / mubar_i
    // from the diagonal down (a running product of mu: non-negative factors,
    // no exponential per element) and 0 above it, so
    //     h_r = alpha_r h_{r-1} + beta_r f_r,   Gamma_{r,i} = eta_i h_r
    // needs no case for the rows above the diagonal.  Each row's alpha, beta,
    // mu come from shared memory as one broadcast 16-byte load.
    __shared__ float4 rowc[4][kChunk];
    float4* rc = rowc[threadIdx.x >> 5];
#pragma unroll
    for (int e = 0; e < 2; ++e) rc[2 * lane + e] = make_float4(expf(a[e]), be[e], expf(m[e]), 0.f);
    const int i0 = lane, i1 = lane + 32;
    // Position p sits in lane p/2, element p%2: fetch both elements, pick locally.
    auto fetch = [&](const float (&x)[2], int p) {
        const float e0 = __shfl_sync(kFull, x[0], p >> 1);
        const float e1 = __shfl_sync(kFull, x[1], p >> 1);
        return (p & 1) ? e1 : e0;
    };
    const float eta_i0 = fetch(et, i0), eta_i1 = fetch(et, i1);
    __syncwarp();
    float h0 = 0.f, h1 = 0.f, f0 = 0.f, f1 = 0.f;
    float* G = gamma + (size_t)chunk * kChunk * kChunk;
#pragma unroll 4
    for (int r = 0; r < kChunk; ++r) {
        const float4 c = rc[r];
        f0 = fmaf(c.z, f0, r == i0 ? 1.f : 0.f);
        f1 = fmaf(c.z, f1, r == i1 ? 1.f : 0.f);
        h0 = fmaf(c.x, h0, c.y * f0);
        h1 = fmaf(c.x, h1, c.y * f1);
        G[r * kChunk + i0] = eta_i0 * h0;
        G[r * kChunk + i1] = eta_i1 * h1;
    }
}

}  // namespace

cudaError_t launch_gate_prep(const GateSrc& g, int B, int T, int H, float* la, float* lm,
                             float* lc, float* bco, float* gamma, cudaStream_t s)
{
    const int NT = (T + kChunk - 1) / kChunk;
    const long long chunks = (long long)B * H * NT;
    if (chunks == 0) return cudaSuccess;
    const int warps_per_block = 4;
    const long long blocks = (chunks + warps_per_block - 1) / warps_per_block;
    ProfScope ps(kGatePrep, s);
    gate_prep_kernel<<<(unsigned)blocks, 32 * warps_per_block, 0, s>>>(
        g, B, T, H, NT, la, lm, lc, bco, gamma);
    return cudaGetLastError();
}

}  // namespace mdn
