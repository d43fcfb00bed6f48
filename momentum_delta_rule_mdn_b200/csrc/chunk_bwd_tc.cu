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
constexpr uint32_t SSUM = 196608;    // fp32 row sums [5][64], then scalars [8][3]
constexpr uint32_t SBAR = SSUM + 1280 + 96;
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
    float* sums = reinterpret_cast<float*>(sm + SSUM);       // sa, sb, sd2, sgl, sw x 64 rows
    float* wsum = sums + 5 * C;                              // [8 warps][3]
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
    for (int i = tid; i < 5 * C; i += kThr) sums[i] = 0.f;
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
        atomicAdd(sums + r, sa);
        if (R < 64) {
            atomicAdd(sums + C + r, sb);
            atomicAdd(sums + 3 * C + r, sgl);
            atomicAdd(sums + 4 * C + r, sw);
        } else {
            atomicAdd(sums + 2 * C + r, sd2);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    float* rec = a.crec_bw + chunk * kBwdRec;
    for (int i = tid; i < 5 * C; i += kThr) rec[i] = sums[i];
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

}  // namespace

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
