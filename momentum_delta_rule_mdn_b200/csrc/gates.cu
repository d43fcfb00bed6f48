// K-0: the four gates of every token from their pre-activations, by the
// stable parameterisation of gate_math.cuh ("MDN: Parallelizing Stepwise
// Momentum for Delta Linear Attention", paper.rainbus.top summary, step 6;
// ijyty.com article, sections 5 and 8).  Elementwise and HBM-bound: 16 bytes
// in, 16 bytes out per element, 16-byte accesses when the arrays allow.
#include "gate_math.cuh"
#include "mdn_internal.cuh"

namespace mdn {
namespace {

using gate::gate_one;

template <int ACT, bool VEC>
__global__ void __launch_bounds__(256)
gate_params_kernel(const float* __restrict__ x, const float* __restrict__ a,
                   const float* __restrict__ b, const float* __restrict__ c, long long n,
                   float s, float mu_min, float* __restrict__ al, float* __restrict__ ml,
                   float* __restrict__ be, float* __restrict__ et)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    if (VEC) {  // n % 4 == 0 and every array 16-byte aligned
        const long long n4 = n >> 2;
        for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
            const float4 x4 = __ldcs(reinterpret_cast<const float4*>(x) + i);
            const float4 a4 = __ldcs(reinterpret_cast<const float4*>(a) + i);
            const float4 b4 = __ldcs(reinterpret_cast<const float4*>(b) + i);
            const float4 c4 = __ldcs(reinterpret_cast<const float4*>(c) + i);
            float4 o1, o2, o3, o4;
            gate_one<ACT>(x4.x, a4.x, b4.x, c4.x, s, mu_min, o1.x, o2.x, o3.x, o4.x);
            gate_one<ACT>(x4.y, a4.y, b4.y, c4.y, s, mu_min, o1.y, o2.y, o3.y, o4.y);
            gate_one<ACT>(x4.z, a4.z, b4.z, c4.z, s, mu_min, o1.z, o2.z, o3.z, o4.z);
            gate_one<ACT>(x4.w, a4.w, b4.w, c4.w, s, mu_min, o1.w, o2.w, o3.w, o4.w);
            reinterpret_cast<float4*>(al)[i] = o1;
            reinterpret_cast<float4*>(ml)[i] = o2;
            reinterpret_cast<float4*>(be)[i] = o3;
            reinterpret_cast<float4*>(et)[i] = o4;
        }
    } else {
        for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
            gate_one<ACT>(x[i], a[i], b[i], c[i], s, mu_min, al[i], ml[i], be[i], et[i]);
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

cudaError_t launch_gate_params(const float* x_eta, const float* a, const float* b, const float* c,
                               long long n, float s_scale, float mu_log_min, int eta_act,
                               float* alpha_log, float* mu_log, float* beta, float* eta,
                               cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    const void* ptrs[] = {x_eta, a, b, c, alpha_log, mu_log, beta, eta};
    bool vec = (n & 3) == 0;
    for (const void* p : ptrs) vec = vec && aligned16(p);
    const long long items = vec ? n / 4 : n;
    // One item per thread: on B200 this streams at the rate of a plain copy
    // of the same eight arrays, where a grid-stride loop over a few CTAs per
    // SM lost up to a fifth of it.  The loop remains only past 2^30 CTAs.
    const long long want = (items + 255) / 256;
    const unsigned grid = (unsigned)(want < (1LL << 30) ? want : (1LL << 30));
    ProfScope ps(kGateParams, s);
#define MDN_GATES_LAUNCH(ACT, VEC)                                                          \
    gate_params_kernel<ACT, VEC><<<grid, 256, 0, s>>>(x_eta, a, b, c, n, s_scale, mu_log_min, \
                                                      alpha_log, mu_log, beta, eta)
    if (eta_act == 0) {
        if (vec) MDN_GATES_LAUNCH(0, true); else MDN_GATES_LAUNCH(0, false);
    } else {
        if (vec) MDN_GATES_LAUNCH(1, true); else MDN_GATES_LAUNCH(1, false);
    }
#undef MDN_GATES_LAUNCH
    return cudaGetLastError();
}

}  // namespace mdn
