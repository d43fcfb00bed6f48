// B-3a of the backward pass on tcgen05 tensor cores (bf16 inputs, d = 128).
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 7 (the backward pass rebuilds S and M from
// the saved Vtilde).  Per chunk, with S, M the states entering it and dS, dM
// the adjoints of the states leaving it, the six products
//     [dO; dY] [S | M]^T   -> P1 = dO S^T, P2 = dO M^T, P5 = dY S^T, P6 = dY M^T
//     [Vt; 0]  [dS | dM]^T -> P3 = Vt dS^T, P4 = Vt dM^T
// are two groups of eight tcgen05.mma (M 128, N 256, K 128; bf16 operands,
// fp32 accumulators in 512 TMEM columns).  The epilogue forms the parts of dq
// and dk they carry,
//     dq = Diag(alphabar) P1 - Diag(b) P2
//     dk = Diag(Gamma_C) P3 - Diag(w) P4 - Diag(alphabar) P5 + Diag(D2) P6
// and the row sums that feed the gate gradients, exactly as the CUDA-core
// kernel does.  Operands are staged by the threads themselves (fp32 states
// and dY are rounded to bf16 on the way into shared memory), K-major with the
// 128-byte swizzle.
#include "bwd_common.cuh"
#include "mdn_internal.cuh"
#include "tc_common.cuh"

namespace mdn {
namespace {

using namespace sm100;
using namespace tc;

constexpr int kThr = 256;
// shared memory (byte offsets from a 1024-byte aligned base)
constexpr uint32_t SA1 = 0;          // [dO; dY]: 2 K-panels x 128 rows x 128 B
constexpr uint32_t SA2 = 32768;      // [Vt; 0]
constexpr uint32_t SB1 = 65536;      // [S | M] as 256 rows: 2 K-panels x 256 rows x 128 B
constexpr uint32_t SB2 = 131072;     // [dS | dM]
constexpr uint32_t SSUM = 196608;    // fp32 row-sum partials [12][64], then scalars [8][3]
constexpr uint32_t SBAR = SSUM + 3072 + 96;
constexpr uint32_t SMISC = SBAR + 16;
constexpr uint32_t SMEM_BYTES = SMISC + 16 + 1024;  // + alignment slack
constexpr int XS = 129;              // row stride (floats) of the dk exchange tile over SA1

__device__ __forceinline__ size_t tokrow(const BwdArgs& a, int b, int t, int h) {
    return ((size_t)b * a.T + t) * a.H + h;
}

__global__ void __launch_bounds__(kThr, 1)
bwd_state_grads_tc_kernel(BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const size_t chunk = blockIdx.x, crow = chunk * C;
    // row-sum partials, one slot per writer so that the sums are formed in a
    // fixed order: sa from (row kind, column half) in slots 0..3, then sb,
    // sd2, sgl, sw from the two column halves in slots 4..11
    float* part = reinterpret_cast<float*>(sm + SSUM);
    float* wsum = part + 12 * C;                             // [8 warps][3]
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SBAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SMISC);

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    for (int i = tid; i < 12 * C; i += kThr) part[i] = 0.f;
    // rows 64..127 of [Vt; 0]
    for (int i = tid; i < 1024; i += kThr) {
        const int p = i >> 9, w = i & 511;
        *reinterpret_cast<uint4*>(sm + SA2 + p * 16384 + 8192 + w * 16) = make_uint4(0, 0, 0, 0);
    }
    // dO, Vt (bf16 copies) and dY (fp32 -> bf16), 64 rows x 16 chunks of 8 each
    for (int i = tid; i < C * 16; i += kThr) {
        const int r = i >> 4, c16 = i & 15, t = n * C + r;
        const uint32_t off = (c16 >> 3) * 16384 + sw128_off(r, c16 & 7);
        uint4 o = make_uint4(0, 0, 0, 0), v = o, y = o;
        if (t < a.T) {
            const size_t g = tokrow(a, b, t, h) * D + c16 * 8;
            o = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.dout) + g);
            v = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.vt) + g);
            const float4 y0 = *reinterpret_cast<const float4*>(a.dv + g);
            const float4 y1 = *reinterpret_cast<const float4*>(a.dv + g + 4);
            const float yy[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
            y = bf16x8(yy);
        }
        *reinterpret_cast<uint4*>(sm + SA1 + off) = o;
        *reinterpret_cast<uint4*>(sm + SA1 + off + 64 * 128) = y;   // rows 64..127
        *reinterpret_cast<uint4*>(sm + SA2 + off) = v;
    }
    // S, M, dS, dM (fp32 -> bf16), 128 rows x 16 chunks each; the three scalars
    const float* Sn = a.SS + chunk * 2 * D * D;
    const float* Mn = Sn + D * D;
    const float* dSn = a.dSS + chunk * 2 * D * D;
    const float* dMn = dSn + D * D;
    float s1 = 0.f, s2 = 0.f, s3 = 0.f;
    for (int i = tid; i < D * 16; i += kThr) {
        const int row = i >> 4, c16 = i & 15;
        const size_t g = (size_t)row * D + c16 * 8;
        float sv[8], mv[8], dsv[8], dmv[8];
        *reinterpret_cast<float4*>(sv) = *reinterpret_cast<const float4*>(Sn + g);
        *reinterpret_cast<float4*>(sv + 4) = *reinterpret_cast<const float4*>(Sn + g + 4);
        *reinterpret_cast<float4*>(mv) = *reinterpret_cast<const float4*>(Mn + g);
        *reinterpret_cast<float4*>(mv + 4) = *reinterpret_cast<const float4*>(Mn + g + 4);
        *reinterpret_cast<float4*>(dsv) = *reinterpret_cast<const float4*>(dSn + g);
        *reinterpret_cast<float4*>(dsv + 4) = *reinterpret_cast<const float4*>(dSn + g + 4);
        *reinterpret_cast<float4*>(dmv) = *reinterpret_cast<const float4*>(dMn + g);
        *reinterpret_cast<float4*>(dmv + 4) = *reinterpret_cast<const float4*>(dMn + g + 4);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            s1 = fmaf(sv[e], dsv[e], s1);
            s2 = fmaf(mv[e], dsv[e], s2);
            s3 = fmaf(mv[e], dmv[e], s3);
        }
        const uint32_t pan = (c16 >> 3) * 32768;
        st_bf16x8(sm + SB1 + pan + sw128_off(row, c16 & 7), sv);
        st_bf16x8(sm + SB1 + pan + sw128_off(row + 128, c16 & 7), mv);
        st_bf16x8(sm + SB2 + pan + sw128_off(row, c16 & 7), dsv);
        st_bf16x8(sm + SB2 + pan + sw128_off(row + 128, c16 & 7), dmv);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
        s2 += __shfl_xor_sync(0xffffffffu, s2, off);
        s3 += __shfl_xor_sync(0xffffffffu, s3, off);
    }
    if (lane == 0) {
        wsum[warp * 3] = s1;
        wsum[warp * 3 + 1] = s2;
        wsum[warp * 3 + 2] = s3;
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (tid == 0) {
        constexpr uint32_t id = idesc_bf16(128, 256, false, false);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = (ks >> 2) * 16384 + (ks & 3) * 32, kb = (ks >> 2) * 32768 + (ks & 3) * 32;
            mma_bf16(tmem, smem_desc(sbase + SA1 + ko, 16, 1024, kSw128),
                     smem_desc(sbase + SB1 + kb, 16, 1024, kSw128), id, ks > 0);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = (ks >> 2) * 16384 + (ks & 3) * 32, kb = (ks >> 2) * 32768 + (ks & 3) * 32;
            mma_bf16(tmem + 256, smem_desc(sbase + SA2 + ko, 16, 1024, kSw128),
                     smem_desc(sbase + SB2 + kb, 16, 1024, kSw128), id, ks > 0);
        }
        mma_commit(bar);
    }
    const bool ok = __syncthreads_and(mbar_wait(bar, 0));
    tc_fence_after_sync();

    // Epilogue.  Warp w reads TMEM lanes 32 (w % 4) ..; warps w and w + 4 take
    // the two halves of the 128 columns of each product.
    const int quad = warp & 3, half = warp >> 2;
    const int R = quad * 32 + lane;               // TMEM lane: dO rows 0..63, dY rows 64..127
    const uint32_t tq = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    float* X = reinterpret_cast<float*>(sm + SA1);  // dk of the dY rows, [64][XS], over the operands
    const int r = R & 63, t = n * C + r;
    const bool in = t < a.T;
    const size_t grow = in ? tokrow(a, b, t, h) * D : 0;
    const float abar = expf(a.la[crow + r]), bco = a.bco[crow + r];
    const float al = in ? expf(a.alpha_log[tokrow(a, b, t, h)]) : 1.f;
    const float d2 = r > 0 ? a.bco[crow + r - 1] * al : 0.f;
    const float gl = a.gamma[chunk * C * C + (C - 1) * C + r];
    const float et = in ? a.eta[tokrow(a, b, t, h)] : 0.f;
    const float w = et * expf(a.lm[crow + C - 1] - a.lm[crow + r]);
    const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q) + grow;
    const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k) + grow;
    float sa = 0.f, sb = 0.f, sd2 = 0.f, sgl = 0.f, sw = 0.f;
    if (ok && R >= 64) {
        // dY rows: dk part -Diag(alphabar) P5 + Diag(D2) P6, into the exchange tile
#pragma unroll 1
        for (int k0 = half * 64; k0 < half * 64 + 64; k0 += 16) {
            float p5[16], p6[16], kv[16];
            tmem_ld16(tq + k0, p5);
            tmem_ld16(tq + 128 + k0, p6);
            tmem_wait_ld();
            if (in) {
                unpack_bf16x8(*reinterpret_cast<const uint4*>(kg + k0), kv);
                unpack_bf16x8(*reinterpret_cast<const uint4*>(kg + k0 + 8), kv + 8);
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) kv[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                sa = fmaf(-kv[e], p5[e], sa);
                sd2 = fmaf(kv[e], p6[e], sd2);
                p5[e] = fmaf(d2, p6[e], -abar * p5[e]);
            }
            // ordered after the MMAs (their completion was observed) and read after the barrier
#pragma unroll
            for (int e = 0; e < 16; ++e) X[r * XS + k0 + e] = p5[e];
        }
    }
    __syncthreads();
    if (ok && R < 64) {
#pragma unroll 1
        for (int k0 = half * 64; k0 < half * 64 + 64; k0 += 16) {
            float p1[16], p2[16], p3[16], p4[16], kv[16], qh[16];
            tmem_ld16(tq + k0, p1);
            tmem_ld16(tq + 128 + k0, p2);
            tmem_ld16(tq + 256 + k0, p3);
            tmem_ld16(tq + 384 + k0, p4);
            tmem_wait_ld();
            if (in) {  // the TMEM loads above stay warp-uniform
                unpack_bf16x8(*reinterpret_cast<const uint4*>(kg + k0), kv);
                unpack_bf16x8(*reinterpret_cast<const uint4*>(kg + k0 + 8), kv + 8);
                unpack_bf16x8(*reinterpret_cast<const uint4*>(qg + k0), qh);
                unpack_bf16x8(*reinterpret_cast<const uint4*>(qg + k0 + 8), qh + 8);
                float dq[16], dk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    qh[e] -= a.dcorr * kv[e];
                    sa = fmaf(qh[e], p1[e], sa);
                    sb = fmaf(-qh[e], p2[e], sb);
                    sgl = fmaf(kv[e], p3[e], sgl);
                    sw = fmaf(-kv[e], p4[e], sw);
                    dq[e] = fmaf(abar, p1[e], -bco * p2[e]);
                    dk[e] = fmaf(gl, p3[e], -w * p4[e]) + X[r * XS + k0 + e];
                }
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    *reinterpret_cast<float4*>(a.dq + grow + k0 + 4 * e4) =
                        make_float4(dq[4 * e4], dq[4 * e4 + 1], dq[4 * e4 + 2], dq[4 * e4 + 3]);
                    *reinterpret_cast<float4*>(a.dk + grow + k0 + 4 * e4) =
                        make_float4(dk[4 * e4], dk[4 * e4 + 1], dk[4 * e4 + 2], dk[4 * e4 + 3]);
                }
            }
        }
    }
    // row sums of both column halves (and, for sa, of both row kinds)
    if (ok && in) {
        const int kind = R < 64 ? 0 : 1;
        part[(2 * kind + half) * C + r] = sa;
        if (R < 64) {
            part[(4 + half) * C + r] = sb;
            part[(8 + half) * C + r] = sgl;
            part[(10 + half) * C + r] = sw;
        } else {
            part[(6 + half) * C + r] = sd2;
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    float* rec = a.crec_bw + chunk * kBwdRec;
    if (tid < C) {
        const float* p0 = part + tid;
        rec[tid] = (p0[0] + p0[C]) + (p0[2 * C] + p0[3 * C]);
        rec[C + tid] = p0[4 * C] + p0[5 * C];
        rec[2 * C + tid] = p0[6 * C] + p0[7 * C];
        rec[3 * C + tid] = p0[8 * C] + p0[9 * C];
        rec[4 * C + tid] = p0[10 * C] + p0[11 * C];
    }
    if (tid < 3) {
        float acc = 0.f;
        for (int w8 = 0; w8 < 8; ++w8) acc += wsum[w8 * 3 + tid];
        rec[5 * C + tid] = acc;
    }
    if (!ok && tid == 0) atomicOr(a.status + 1, 1u);
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// B-3b on tcgen05: the chunk-local products of the backward pass.
//   stage 1: [dO; dY] Vt^T -> dO Vt^T (lanes 0..63), dY Vt^T (64..127)     (N 64)
//            [Qhat; K] K^T -> Qhat K^T, K K^T                               (N 64)
//   SIMT:    dOVG = (dO Vt^T) o Gamma, dPK = -(dY Vt^T) o Gamma-, the adjoint
//            of Gamma; bf16 operands [dOVG; dPK] and [dOVG^T | (dPK o alpha)^T]
//   stage 2: [dOVG; dPK] K -> dQhat part (lanes 0..63), dP = dPK K (64..127) (N 128)
//            [dOVG^T | (Diag(alpha) dPK)^T] [Qhat; K] -> dK part                (N 128)
//   SIMT:    dq, dk written; the coefficient phase gives the gate gradients.
constexpr uint32_t LA_DY = 0;        // [dO; dY]   K-major, 2 K-panels x 128 rows x 128 B
constexpr uint32_t LA_QK = 32768;    // [Qhat; K]  K-major (its K rows double as B of K K^T)
constexpr uint32_t LB_V = 65536;     // Vt         K-major, 2 K-panels x 64 rows x 128 B
constexpr uint32_t LA_3 = 81920;     // [dOVG; dPK]          K = 64: 1 panel x 128 rows x 128 B
constexpr uint32_t LA_4 = 98304;     // [dOVG^T | dPKa^T; 0] K = 128: 2 panels x 128 rows x 128 B
constexpr uint32_t L_GP = 131072;    // fp32 Gp [64][65]
constexpr uint32_t L_DG = L_GP + 16640;   // fp32 dG [64][65]
constexpr uint32_t L_VEC = L_DG + 16640;  // 12 x 64 floats
constexpr uint32_t L_REC = L_VEC + 3072;  // the chunk record (kBwdRec floats)
constexpr uint32_t L_BAR = L_REC + kBwdRec * 4;
constexpr uint32_t L_MISC = L_BAR + 16;
constexpr uint32_t L_SMEM = L_MISC + 16 + 1024;
constexpr int LAS = 65;                   // row stride of the fp32 C x C matrices

__device__ __forceinline__ void st_bf16(uint8_t* p, float x) {
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(x);
}
// byte offset of element (row, k) in a K-major 128-byte-swizzled tile whose
// K-panels (64 elements) are panel_bytes apart
__device__ __forceinline__ uint32_t kmaj_off(int row, int k, uint32_t panel_bytes) {
    return (k >> 6) * panel_bytes + sw128_off(row, (k & 63) >> 3) + (k & 7) * 2;
}

__global__ void __launch_bounds__(kThr, 1)
bwd_local_grads_tc_kernel(BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const size_t chunk = blockIdx.x, crow = chunk * C;
    float* Gp = reinterpret_cast<float*>(sm + L_GP);
    float* dG = reinterpret_cast<float*>(sm + L_DG);
    const BwdVec v = bwd_vec(reinterpret_cast<float*>(sm + L_VEC));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L_MISC);

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    // operands: dO, dY, Qhat, K, Vt rows (bf16, K-major)
    for (int i = tid; i < C * 16; i += kThr) {
        const int r = i >> 4, c16 = i & 15, t = n * C + r;
        const uint32_t off = (c16 >> 3) * 16384 + sw128_off(r, c16 & 7);
        float o[8] = {0.f}, y[8] = {0.f}, q[8] = {0.f}, k[8] = {0.f}, vt[8] = {0.f};
        if (t < a.T) {
            const size_t g = tokrow(a, b, t, h) * D + c16 * 8;
            unpack_bf16x8(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.dout) + g), o);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + g), q);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.k) + g), k);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.vt) + g), vt);
            const float4 y0 = *reinterpret_cast<const float4*>(a.dv + g);
            const float4 y1 = *reinterpret_cast<const float4*>(a.dv + g + 4);
            y[0] = y0.x; y[1] = y0.y; y[2] = y0.z; y[3] = y0.w;
            y[4] = y1.x; y[5] = y1.y; y[6] = y1.z; y[7] = y1.w;
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] -= a.dcorr * k[e];
        }
        st_bf16x8(sm + LA_DY + off, o);
        st_bf16x8(sm + LA_DY + off + 64 * 128, y);
        st_bf16x8(sm + LA_QK + off, q);
        st_bf16x8(sm + LA_QK + off + 64 * 128, k);
        st_bf16x8(sm + LB_V + (c16 >> 3) * 8192 + sw128_off(r, c16 & 7), vt);
    }
    // rows 64..127 of the second stage-2 operand are zero
    for (int i = tid; i < 1024; i += kThr) {
        const int p = i >> 9, w = i & 511;
        *reinterpret_cast<uint4*>(sm + LA_4 + p * 16384 + 8192 + w * 16) = make_uint4(0, 0, 0, 0);
    }
    if (tid < C) {
        const int r = tid, t = n * C + r;
        const bool in = t < a.T;
        const size_t gi = in ? tokrow(a, b, t, h) : 0;
        v.al[r] = in ? expf(a.alpha_log[gi]) : 1.f;
        v.be[r] = in ? a.beta[gi] : 0.f;
        v.et[r] = in ? a.eta[gi] : 0.f;
        v.la[r] = a.la[crow + r];
        v.lm[r] = a.lm[crow + r];
        v.b[r] = a.bco[crow + r];
        v.da[r] = 0.f;
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        constexpr uint32_t id1 = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ka = (ks >> 2) * 16384 + (ks & 3) * 32;
            const uint32_t kv = (ks >> 2) * 8192 + (ks & 3) * 32;
            mma_bf16(tmem, smem_desc(sbase + LA_DY + ka, 16, 1024, kSw128),
                     smem_desc(sbase + LB_V + kv, 16, 1024, kSw128), id1, ks > 0);
            mma_bf16(tmem + 64, smem_desc(sbase + LA_QK + ka, 16, 1024, kSw128),
                     smem_desc(sbase + LA_QK + 8192 + ka, 16, 1024, kSw128), id1, ks > 0);
        }
        mma_commit(&bars[0]);
    }
    // Gamma without eta, by its column recurrence (overlaps the products)
    if (tid < C) {
        const int i = tid;
        float g = 0.f;
        for (int r = 0; r < C; ++r) {
            if (r < i) {
                Gp[r * LAS + i] = 0.f;
            } else {
                g = (r == i) ? v.be[i] : fmaf(v.al[r], g, v.be[r] * expf(v.lm[r] - v.lm[i]));
                Gp[r * LAS + i] = g;
            }
        }
    }
    bool ok = __syncthreads_and(mbar_wait(&bars[0], 0));
    tc_fence_after_sync();

    // stage-1 epilogue: warp w reads lanes 32 (w % 4) ..; warps w, w + 4 take
    // columns i in [32 half, 32 half + 32)
    const int quad = warp & 3, half = warp >> 2;
    const int R = quad * 32 + lane, r = R & 63;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    float dgm[32];  // dY rows: dA o (P K^T), owed to dG[r - 1][i]
    if (ok) {
        float x1[32], x2[32];
        tmem_ld32(tq + 32 * half, x1);        // dO Vt^T  (dY Vt^T on lanes 64..127)
        tmem_ld32(tq + 64 + 32 * half, x2);   // Qhat K^T (K K^T)
        tmem_wait_ld();
        const float al_r = v.al[r];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int i = 32 * half + e;
            if (R < 64) {
                const float g = v.et[i] * Gp[r * LAS + i];
                const float ovg = i <= r ? x1[e] * g : 0.f;
                dG[r * LAS + i] = i <= r ? x1[e] * x2[e] : 0.f;
                st_bf16(sm + LA_3 + kmaj_off(r, i, 16384), ovg);             // row r of [dOVG; .]
                st_bf16(sm + LA_4 + kmaj_off(i, r, 16384), ovg);             // (dOVG^T)[i][r]
            } else {
                const float pk = i < r ? -x1[e] * v.et[i] * Gp[(r - 1) * LAS + i] : 0.f;
                dgm[e] = i < r ? -x1[e] * al_r * x2[e] : 0.f;
                st_bf16(sm + LA_3 + kmaj_off(64 + r, i, 16384), pk);        // row 64 + r: dPK
                st_bf16(sm + LA_4 + kmaj_off(i, 64 + r, 16384), pk * al_r); // (Diag(alpha) dPK)^T
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (ok && R >= 64) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int i = 32 * half + e;
            if (i < r) dG[(r - 1) * LAS + i] += dgm[e];  // one writer per entry
        }
    }
    const float* rec = a.crec_bw + chunk * kBwdRec;
    if (tid == 0 && ok) {
        constexpr uint32_t id2 = idesc_bf16(128, 128, false, true);
        // [dOVG; dPK] K: B = K (K-dim i = rows 64..127 of the [Qhat; K] tile, N = features)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tmem + 128, smem_desc(sbase + LA_3 + ks * 32, 16, 1024, kSw128),
                     smem_desc(sbase + LA_QK + 8192 + ks * 2048, 16384, 1024, kSw128), id2, ks > 0);
        // [dOVG^T | dPKa^T] [Qhat; K]: B = the whole [Qhat; K] tile, K-dim 128 rows
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + 256,
                     smem_desc(sbase + LA_4 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128),
                     smem_desc(sbase + LA_QK + ks * 2048, 16384, 1024, kSw128), id2, ks > 0);
        mma_commit(&bars[1]);
    }
    __syncthreads();
    if (tid < C) dG[(C - 1) * LAS + tid] += rec[3 * C + tid];  // Gamma_{C,i} in the state update
    ok = __syncthreads_and(ok && mbar_wait(&bars[1], 0));
    tc_fence_after_sync();

    // stage-2 epilogue: lanes 64..127 hold dP = dPK K; lanes 0..63 the dQhat
    // and dK parts; warps w, w + 4 take feature columns [64 half, 64 half + 64)
    float* X = reinterpret_cast<float*>(sm + LA_DY);  // alpha_r dP[r][c], [64][129], over the operands
    const int t = n * C + r;
    const bool in = t < a.T;
    const size_t grow = in ? tokrow(a, b, t, h) * D : 0;
    if (ok && R >= 64) {
        float dar = 0.f;
        const float al_r = v.al[r];
        const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k) + grow;
#pragma unroll 1
        for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
            float dp[16], kv[16];
            tmem_ld16(tq + 128 + c0, dp);
            tmem_wait_ld();
            if (in) {
                unpack_bf16x8(*reinterpret_cast<const uint4*>(kg + c0), kv);
                unpack_bf16x8(*reinterpret_cast<const uint4*>(kg + c0 + 8), kv + 8);
#pragma unroll
                for (int e = 0; e < 16; ++e) dar = fmaf(dp[e], kv[e], dar);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) X[r * 129 + c0 + e] = al_r * dp[e];
        }
        atomicAdd(v.da + r, dar);
    }
    __syncthreads();
    if (ok && R < 64) {
        // The exchange row is read into registers before any global store: X is
        // reached through a generic pointer, so reads of it interleaved with the
        // stores to dq and dk could not be hoisted and serialised the loop.
        float xr[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) xr[e] = X[r * 129 + 64 * half + e];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c0 = 64 * half + 16 * j;
            float dqb[16], dkb[16];
            tmem_ld16(tq + 128 + c0, dqb);
            tmem_ld16(tq + 256 + c0, dkb);
            tmem_wait_ld();
            if (in) {
                float4 q4[4], k4[4];
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {  // every load of the group before any store
                    q4[e4] = *reinterpret_cast<const float4*>(a.dq + grow + c0 + 4 * e4);
                    k4[e4] = *reinterpret_cast<const float4*>(a.dk + grow + c0 + 4 * e4);
                }
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    const float qo[4] = {q4[e4].x, q4[e4].y, q4[e4].z, q4[e4].w};
                    const float ko[4] = {k4[e4].x, k4[e4].y, k4[e4].z, k4[e4].w};
                    float qn[4], kn[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int x = 16 * j + 4 * e4 + e;
                        qn[e] = qo[e] + dqb[4 * e4 + e];
                        kn[e] = ko[e] + dkb[4 * e4 + e] + xr[x] - a.dcorr * qn[e];
                    }
                    *reinterpret_cast<float4*>(a.dq + grow + c0 + 4 * e4) =
                        make_float4(qn[0], qn[1], qn[2], qn[3]);
                    *reinterpret_cast<float4*>(a.dk + grow + c0 + 4 * e4) =
                        make_float4(kn[0], kn[1], kn[2], kn[3]);
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
    if (!ok) {
        if (tid == 0) atomicOr(a.status + 1, 1u);
        return;
    }
    bwd_coeff_phase(a, rec, v, dG, Gp, reinterpret_cast<float*>(sm + L_REC), tid, n, b, h);
}

// ---------------------------------------------------------------------------
// The chunk-only operands of the tensor-core reverse chain (bf16, d = 128).
// With T, Att from B-0, per chunk:
//   U  = [-K^T Diag(alphabar) T^T ; K^T Diag(D2) T^T]   bf16 [256][64]  (A of U dVtilde)
//   TT = [T^T ; 0]                                      bf16 [128][64]  (A of T^T dVtilde = dv)
//   P  = Att^T dO     fp32, slice-major [D/32][64][32]  (dVtilde's chain-free part)
//   E  = Qhat^T Diag(alphabar) dO,  F = Qhat^T Diag(b) dO   fp32 [2][128][128]
//   record: Gamma_{C,r} (64), w_r (64), then alphabar_C, b_C, mubar_C at 192..194
__global__ void __launch_bounds__(kThr, 1)
bwd_chain_prep_kernel(BwdArgs a)
{
    constexpr int KS = D + 1, AS = C + 1;
    extern __shared__ float fsm[];
    float* Ks = fsm;              // [C][D+1]
    float* Qs = Ks + C * KS;      // [C][D+1]  qhat
    float* Os = Qs + C * KS;      // [C][D+1]  dO
    float* Tm = Os + C * KS;      // [C][C+1]  T
    float* At = Tm + C * AS;      // [C][C+1]  Att
    float* ab = At + C * AS;      // [C] alphabar
    float* bb = ab + C;           // [C] b
    float* d2 = bb + C;           // [C] b_{r-1} alpha_r
    const int tid = threadIdx.x;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const size_t chunk = blockIdx.x, crow = chunk * C;
    {   // K, qhat, dO tiles and T, Att: every load of a thread before its stores
        constexpr int U8 = C * D / 8 / kThr;  // 8-element groups per thread and tile
        float kx[U8][8], qx[U8][8], ox[U8][8];
#pragma unroll
        for (int u = 0; u < U8; ++u) {
            const int idx = (tid + kThr * u) * 8, r = idx / D, c = idx % D, t = n * C + r;
            if (t < a.T) {
                const size_t g = tokrow(a, b, t, h) * D + c;
                ld8<__nv_bfloat16>(a.k, g, kx[u]);
                ld8<__nv_bfloat16>(a.q, g, qx[u]);
                ld8<__nv_bfloat16>(a.dout, g, ox[u]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) kx[u][e] = qx[u][e] = ox[u][e] = 0.f;
            }
        }
        constexpr int U4 = C * C / 4 / kThr;
        float4 tx[U4], ax[U4];
#pragma unroll
        for (int u = 0; u < U4; ++u) {
            const int idx = (tid + kThr * u) * 4;
            tx[u] = *reinterpret_cast<const float4*>(a.tmat + chunk * C * C + idx);
            ax[u] = *reinterpret_cast<const float4*>(a.att + chunk * C * C + idx);
        }
#pragma unroll
        for (int u = 0; u < U8; ++u) {
            const int idx = (tid + kThr * u) * 8, r = idx / D, c = idx % D;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                Ks[r * KS + c + e] = kx[u][e];
                Qs[r * KS + c + e] = qx[u][e] - a.dcorr * kx[u][e];
                Os[r * KS + c + e] = ox[u][e];
            }
        }
#pragma unroll
        for (int u = 0; u < U4; ++u) {
            const int idx = (tid + kThr * u) * 4, r = idx / C, i = idx % C;
            const float tv[4] = {tx[u].x, tx[u].y, tx[u].z, tx[u].w};
            const float av[4] = {ax[u].x, ax[u].y, ax[u].z, ax[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                Tm[r * AS + i + e] = tv[e];
                At[r * AS + i + e] = av[e];
            }
        }
    }
    float* rec = a.bc_rec + chunk * 256;
    if (tid < C) {
        const int r = tid, t = n * C + r;
        const bool in = t < a.T;
        ab[r] = expf(a.la[crow + r]);
        bb[r] = a.bco[crow + r];
        const float al = in ? expf(a.alpha_log[tokrow(a, b, t, h)]) : 1.f;
        d2[r] = r > 0 ? a.bco[crow + r - 1] * al : 0.f;
        rec[r] = a.gamma[chunk * C * C + (C - 1) * C + r];
        const float et = in ? a.eta[tokrow(a, b, t, h)] : 0.f;
        rec[C + r] = et * expf(a.lm[crow + C - 1] - a.lm[crow + r]);
        if (r == 0) {
            rec[3 * C] = expf(a.la[crow + C - 1]);
            rec[3 * C + 1] = a.bco[crow + C - 1];
            rec[3 * C + 2] = expf(a.lm[crow + C - 1]);
        }
    }
    __syncthreads();
    {   // U: rows i = ig + 64 e (e < 2) of the S and M halves, columns r = rq + 4 m
        const int ig = tid & 63, rq = tid >> 6;
        float us[2][16], um[2][16];
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int m = 0; m < 16; ++m) us[e][m] = um[e][m] = 0.f;
        for (int r2 = 0; r2 < C; ++r2) {
            const float k0 = Ks[r2 * KS + ig], k1 = Ks[r2 * KS + ig + 64];
            const float as = -ab[r2], ad = d2[r2];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float tv = Tm[(rq + 4 * m) * AS + r2];  // T^T[r2][r] = T[r][r2]
                us[0][m] = fmaf(k0 * as, tv, us[0][m]);
                us[1][m] = fmaf(k1 * as, tv, us[1][m]);
                um[0][m] = fmaf(k0 * ad, tv, um[0][m]);
                um[1][m] = fmaf(k1 * ad, tv, um[1][m]);
            }
        }
        __nv_bfloat16* U = a.bc_u + chunk * 256 * 64;
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const int i = ig + 64 * e, r = rq + 4 * m;
                U[i * 64 + r] = __float2bfloat16_rn(us[e][m]);
                U[(128 + i) * 64 + r] = __float2bfloat16_rn(um[e][m]);
            }
    }
    {   // [T^T; 0]
        __nv_bfloat16* TT = a.bc_tt + chunk * 128 * 64;
        for (int idx = tid; idx < 128 * 64; idx += kThr) {
            const int r = idx >> 6, r2 = idx & 63;
            TT[idx] = __float2bfloat16_rn(r < C ? Tm[r2 * AS + r] : 0.f);
        }
    }
    {   // P = Att^T dO, columns j = tid & 127, rows r = (tid >> 7) + 2 m, slice-major
        const int j = tid & 127, rh = tid >> 7;
        float acc[32];
#pragma unroll
        for (int m = 0; m < 32; ++m) acc[m] = 0.f;
        for (int r2 = 0; r2 < C; ++r2) {
            const float ov = Os[r2 * KS + j];
#pragma unroll
            for (int m = 0; m < 32; ++m) acc[m] = fmaf(At[r2 * AS + rh + 2 * m], ov, acc[m]);
        }
        float* P = a.bc_p + chunk * C * D;
        const int sl = j >> 5, jj = j & 31;
#pragma unroll
        for (int m = 0; m < 32; ++m) P[(sl * C + rh + 2 * m) * 32 + jj] = acc[m];
    }
    // E, F: rows i = ig + 16 u, columns j = jg + 16 v (8 x 8 per thread), one after the other
    const int ig = tid & 15, jg = tid >> 4;
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {
        const float* coef = which == 0 ? ab : bb;
        float acc[8][8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int v = 0; v < 8; ++v) acc[u][v] = 0.f;
        for (int r = 0; r < C; ++r) {
            const float cr = coef[r];
            float qv[8], ov[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) qv[u] = Qs[r * KS + ig + 16 * u] * cr;
#pragma unroll
            for (int v = 0; v < 8; ++v) ov[v] = Os[r * KS + jg + 16 * v];
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(qv[u], ov[v], acc[u][v]);
        }
        float* Mx = a.bc_ef + (chunk * 2 + which) * D * D;
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int v = 0; v < 8; ++v) Mx[(ig + 16 * u) * D + jg + 16 * v] = acc[u][v];
    }
}


}  // namespace

cudaError_t launch_bwd_chain_prep(const BwdArgs& a, cudaStream_t s)
{
    const long long chunks = (long long)a.B * a.H * a.NT;
    const size_t smem = sizeof(float) * (3 * C * (D + 1) + 2 * C * (C + 1) + 3 * C);
    cudaError_t e = cudaFuncSetAttribute(bwd_chain_prep_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps(kBwdChainPrep, s);
    bwd_chain_prep_kernel<<<(unsigned)chunks, kThr, smem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_bwd_state_grads_tc(const BwdArgs& a, cudaStream_t s)
{
    if (a.D != D) return cudaErrorNotSupported;
    const long long chunks = (long long)a.B * a.H * a.NT;
    cudaError_t e = cudaFuncSetAttribute(bwd_state_grads_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    ProfScope ps(kBwdStateGrads, s);
    bwd_state_grads_tc_kernel<<<(unsigned)chunks, kThr, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace mdn

namespace mdn {

cudaError_t launch_bwd_local_grads_tc(const BwdArgs& a, cudaStream_t s)
{
    if (a.D != D) return cudaErrorNotSupported;
    const long long chunks = (long long)a.B * a.H * a.NT;
    cudaError_t e = cudaFuncSetAttribute(bwd_local_grads_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L_SMEM);
    if (e != cudaSuccess) return e;
    ProfScope ps(kBwdLocal, s);
    bwd_local_grads_tc_kernel<<<(unsigned)chunks, kThr, L_SMEM, s>>>(a);
    return cudaGetLastError();
}

}  // namespace mdn
