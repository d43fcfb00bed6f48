// The stable gate parameterisation, per token (shared by the gate kernel and
// the chunk kernels that read pre-activations directly).
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 6; ijyty.com article, sections 5 and 8:
//   eta    = tanh(x) + 1            (or 2 sigmoid(x), the ablated variant)
//   theta  = arctan(eta s)
//   alpha  = cos^2(theta) sigmoid(a),   beta = sin^2(theta) sigmoid(b)
//   log mu = max(log sigmoid(c), mu_log_min)
// With u = eta s, cos^2(arctan u) = 1 / (1 + u^2) and sin^2 = u^2 / (1 + u^2),
// so alpha is written in the log domain as log sigmoid(a) - log1p(u^2) and
// sin^2 as 1 / (1 + 1/u^2) (exact at u = 0 and when u^2 overflows), with no
// trigonometric call.  tanh(x) + 1 equals 2 sigmoid(2x), which keeps full
// relative precision where tanh(x) is close to -1, so both activations are
// 2 sigmoid(k x) with k = 2 or 1.
#pragma once

namespace mdn {
namespace gate {

// log sigmoid(z) = min(z, 0) - log(1 + e^{-|z|}).  The log-domain outputs
// need absolute accuracy only: with t = e^{-|z|} in (0, 1], the fast exp's
// relative error (a few ulp plus |z| 2^-24) costs t |z| 2^-24 <= 2^-24 / e
// absolutely, and log(1 + t) by the fast log about 2^-22.
__device__ __forceinline__ float log_sigmoid(float z) {
    return fminf(z, 0.f) - __logf(1.f + __expf(-fabsf(z)));
}
// sigmoid(z) to full relative precision (the accurate exp; correctly rounded
// reciprocal); exactly 0 or 1 where it saturates.
__device__ __forceinline__ float sigmoid(float z) { return __frcp_rn(1.f + expf(-z)); }

// One token's gates.  ACT = 0: eta = tanh(x) + 1; ACT = 1: eta = 2 sigmoid(x).
template <int ACT>
__device__ __forceinline__ void gate_one(float x, float a, float b, float c, float s,
                                         float mu_min, float& al, float& ml, float& be,
                                         float& et) {
    const float e = 2.f * sigmoid(ACT == 0 ? 2.f * x : x);
    const float u = e * s, u2 = u * u;
    al = log_sigmoid(a) - __logf(1.f + u2);
    be = sigmoid(b) * __frcp_rn(1.f + __frcp_rn(u2));
    ml = fmaxf(log_sigmoid(c), mu_min);
    et = e;
}

// The same with the activation chosen at run time.
__device__ __forceinline__ void gate_one_rt(int act, float x, float a, float b, float c, float s,
                                            float mu_min, float& al, float& ml, float& be,
                                            float& et) {
    if (act == 0) gate_one<0>(x, a, b, c, s, mu_min, al, ml, be, et);
    else gate_one<1>(x, a, b, c, s, mu_min, al, ml, be, et);
}

}  // namespace gate
}  // namespace mdn
