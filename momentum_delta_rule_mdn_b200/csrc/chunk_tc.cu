// Fused chunkwise MDN forward pass on the 5th-generation tensor cores
// (tcgen05.mma, bf16 operands, fp32 accumulation in TMEM), fed by TMA.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, steps 3-5.  With the chunk form
//     Vtilde = U - Y S + Z M,  U = T V,  Y = T Diag(alphabar_{r-1}) P,
//     Z = T Diag(b_{r-1}) P,   T = (I + (P K^T) o Gamma-)^{-1},
// write X = D1 K S - D2 K M with D1 = Diag(alphabar_r) (= Diag(alphabar_{r-1} alpha_r)),
// D2 = Diag(alpha_r b_{r-1}); then Vtilde = T (V - X) = T Y with Y = V - X.
// The carried-state part of o is Oi = Diag(alphabar) Qhat S - Diag(b) Qhat M and
// the reordered intra-chunk part is (Qhat K^T o Gamma) Vtilde = (Att T) Y.
// The chunk-end update is S' = alphabar_C S - b_C M + K^T Diag(Gamma_{C,.}) T Y,
// M' = mubar_C M - K^T Diag(eta_i mubar_C / mubar_i) T Y.
//
// One CTA owns one (b, h) and 32 of the d_v = 128 columns (columns of S, M and
// Vtilde are independent) and walks the chunks in order with two warpgroups:
//
//   prep group (warps 4-7), chunk p: state-independent work
//     G    = [K; Qhat] [K; Qhat]^T              (M=128, N=128, K=128)  tensor cores
//            lane i < 64 holds k_i.k_r and k_i.qhat_r for all r
//     one pass down each column i: Gamma_{r,i} = alpha_r Gamma_{r-1,i}
//            + eta_i beta_r mubar_r/mubar_i (running product, no subtraction),
//            A_{r,i} = alpha_r k_r.k_i Gamma_{r-1,i},  Att_{r,i} = qhat_r.k_i Gamma_{r,i}
//     T    = (I + A)^{-1}: 16x16 diagonal blocks by substitution, then the
//            off-diagonal blocks by distance, fp32, float4 shared-memory tiles
//     P    = [I; Att] T       -> [T; Att T]      (M=128, N=64,  K=64)
//     R    = K^T [D_G T | -D_w T] -> A2T         (M=128, N=128, K=64)
//   chain group (warps 0-3), chunk n: depends on the state
//     A1   = [K; Qhat] [S | M]                   (M=128, N=64,  K=128)
//     Y    = V - (D1 KS - D2 KM);  Oi = Diag(alphabar) QhatS - Diag(b) QhatM
//     A2   = [A2T_S; A2T_M] Y (two M=128, N=32, K=64); A3 = [T; Att T] Y (M=128, N=32, K=64)
//     S, M <- (alphabar_C S - b_C M, mubar_C M) + A2;  Vtilde = A3[0:64];  o = Oi + A3[64:128]
//
// The prep of chunk n+1 overlaps the chain of chunk n.  The fp32 state lives
// in registers of the chain group (thread i owns row i of S and M); its bf16
// copy in shared memory is the B operand of A1.  Every mbarrier wait is
// bounded: a wait that runs out sets status[1] and the CTA stops.
#include <cudaTypedefs.h>

#include <mutex>

#include "mdn_internal.cuh"
#include "sm100.cuh"

namespace mdn {
namespace {

using namespace sm100;

constexpr int C = 64;         // chunk length
constexpr int D = 128;        // d_k = d_v
constexpr int NS = 32;        // d_v columns per CTA
constexpr int kThreads = 256; // chain group: threads 0-127, prep group: 128-255
constexpr int kRecFloats = 6 * C;
constexpr uint32_t kTmemCols = 512;
constexpr int LDF = 68;       // leading dimension of the fp32 64x64 matrices (16-byte rows)

// Shared memory map (byte offsets from a 1024-byte aligned base).
constexpr uint32_t KQ0 = 0;                 // [K;Qhat], 2 buffers x 2 panels x (128 rows x 128 B)
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t IATT = 2 * KQ_BYTES;     // [I; Att]   128 x 64 bf16, K-major SW128
constexpr uint32_t TB = IATT + 16384;       // T          64 x 64 bf16, rows k (MN-major SW128)
constexpr uint32_t DT = TB + 8192;          // [D_G T | -D_w T], 2 panels of 64 x 64
constexpr uint32_t TAT = DT + 16384;        // [T; Att T] 128 x 64 bf16, K-major SW128
constexpr uint32_t A2T = TAT + 16384;       // [A2T_S | A2T_M], 2 panels of 128 x 64, K-major
constexpr uint32_t ST = A2T + 32768;        // [S | M] bf16, 128 rows x (32 + 32), MN-major SW128
constexpr uint32_t YB = ST + 16384;         // Y 64 x 32 bf16, MN-major SW64
constexpr uint32_t V0 = YB + 4096;          // V slice 64 x 32 bf16 (plain rows), 2 buffers
constexpr uint32_t REC0 = V0 + 8192;        // coefficient records, 2 buffers of 1536 B
constexpr uint32_t VEC0 = REC0 + 2 * 1536;  // derived vectors, 2 buffers of 6 x 64 floats
constexpr uint32_t SCAL0 = VEC0 + 2 * 1536; // alphabar_C, b_C, mubar_C; 2 buffers of 16 B
constexpr uint32_t AM = 190720;             // fp32 [64][LDF]: A (upper blocks: solve scratch)
constexpr uint32_t TM = AM + 64 * LDF * 4;  // fp32 [64][LDF]: T
constexpr uint32_t BARS = TM + 64 * LDF * 4;
constexpr uint32_t MISC = BARS + 128;       // tmem base
constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;  // + alignment slack
static_assert(SCAL0 + 32 <= AM, "shared memory map overlaps");
static_assert(SMEM_BYTES <= 232448, "shared memory map too large");

// derived vectors (floats, per buffer)
constexpr int VA = 0, VD2 = 64, VB = 128, VWG = 192, VWM = 256, VMU = 320;

// TMEM columns
constexpr uint32_t TM_G = 0, TM_P = 128, TM_R = 192, TM_A1 = 320, TM_A2 = 384, TM_A3 = 448;

constexpr uint32_t kTxBytes = KQ_BYTES + 4096 + 1536;  // 2 K + 2 Q boxes, V box, record

// mbarriers
constexpr int B_FULL0 = 0, B_PREP_MMA = 2, B_CHAIN_MMA = 3, B_PREP_READY = 4, B_OPS_FREE = 5;

// named barriers (id 0 is __syncthreads)
constexpr int NB_CHAIN = 1, NB_PREP = 2;

struct TcArgs {
    const float* rec;
    const float* S0;
    const float* M0;
    float* S_T;
    float* M_T;
    __nv_bfloat16* o;
    __nv_bfloat16* vt;
    unsigned* status;
    float* dbg;  // optional intermediate dump (CTA 0, chunk 0); null in normal use
    float dcorr;
    int B, T, H, NT;
};

// Offsets (floats) of the intermediate dump.
constexpr int DBG_G = 0, DBG_A = 16384, DBG_T = 20480, DBG_P = 24576, DBG_R = 32768,
              DBG_A1 = 49152, DBG_Y = 57344, DBG_A2 = 59392, DBG_A3 = 67584, DBG_S = 71680,
              DBG_M = 75776, DBG_VEC = 79872, DBG_FLOATS = 80400;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
// Eight fp32 values -> one 16-byte chunk of bf16 at a shared address.
__device__ __forceinline__ void st_bf16x8(uint32_t addr, const float* x) {
    st_shared_v4(addr, pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                 pack_bf16(x[6], x[7]));
}
__device__ __forceinline__ void named_bar(int id) {
    asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}
// Named barrier over a 128-thread group that also ANDs a predicate.
__device__ __forceinline__ bool named_bar_and(int id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const TcArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool prep_group = warp >= 4;
    const int g = tid & 127;  // thread index inside its group = its TMEM lane
    const int slice = blockIdx.x % (D / NS);
    const int bh = blockIdx.x / (D / NS);
    const int b = bh / a.H, h = bh % a.H;
    const int j0 = slice * NS;

    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);
    float* Am = reinterpret_cast<float*>(sm + AM);
    float* Tm = reinterpret_cast<float*>(sm + TM);

    if (tid == 0) {
        mbar_init(&bars[B_FULL0], 1);
        mbar_init(&bars[B_FULL0 + 1], 1);
        mbar_init(&bars[B_PREP_MMA], 1);
        mbar_init(&bars[B_CHAIN_MMA], 1);
        mbar_init(&bars[B_PREP_READY], 1);
        mbar_init(&bars[B_OPS_FREE], 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    float s[NS], m[NS];
    if (prep_group) {
        if (g < C) {  // identity rows 0..63 of [I; Att], written once
            for (int c = 0; c < 8; ++c) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = (8 * c + e == g) ? 1.f : 0.f;
                st_bf16x8(sbase + IATT + sw128_off(g, c), x);
            }
        }
    } else {
        // entering state: chain thread i owns row i of S and M, columns j0..j0+31
        const size_t row = ((size_t)bh * D + g) * D + j0;
#pragma unroll
        for (int j = 0; j < NS; ++j) {
            s[j] = a.S0 ? a.S0[row + j] : 0.f;
            m[j] = a.M0 ? a.M0[row + j] : 0.f;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            st_bf16x8(sbase + ST + sw128_off(g, c), s + 8 * c);
            st_bf16x8(sbase + ST + sw128_off(g, 4 + c), m + 8 * c);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_sel = static_cast<uint32_t>((warp & 3) * 32) << 16;

    auto issue_loads = [&](int n) {
        const int buf = n & 1;
        const uint32_t kq = KQ0 + buf * KQ_BYTES;
        mbar_arrive_expect_tx(&bars[B_FULL0 + buf], kTxBytes);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_4d(sm + kq + p * 16384, &tm_k, p * 64, h, n * C, b, &bars[B_FULL0 + buf]);
            tma_load_4d(sm + kq + p * 16384 + 8192, &tm_q, p * 64, h, n * C, b,
                        &bars[B_FULL0 + buf]);
        }
        tma_load_4d(sm + V0 + buf * 4096, &tm_v, j0, h, n * C, b, &bars[B_FULL0 + buf]);
        bulk_load(sm + REC0 + buf * 1536, a.rec + ((size_t)bh * a.NT + n) * kRecFloats, 1536,
                  &bars[B_FULL0 + buf]);
    };
    if (tid == 0) {
        if (a.NT > 0) issue_loads(0);
        if (a.NT > 1) issue_loads(1);
    }

    bool ok = true;
    if (prep_group) {
        // ================================================================ prep group
        uint32_t ph = 0;  // parity of the next completion of B_PREP_MMA
        for (int p = 0; p < a.NT; ++p) {
            const int buf = p & 1;
            const uint32_t kq = KQ0 + buf * KQ_BYTES;
            const float* rec = reinterpret_cast<const float*>(sm + REC0 + buf * 1536);
            float* vec = reinterpret_cast<float*>(sm + VEC0 + buf * 1536);
            float* scal = reinterpret_cast<float*>(sm + SCAL0 + buf * 16);
            const bool dump = a.dbg != nullptr && blockIdx.x == 0 && p == 0;
            ok = named_bar_and(NB_PREP, mbar_wait(&bars[B_FULL0 + buf], (p >> 1) & 1));
            if (!ok) break;

            // Qhat = Q - d K in place; per-position vectors
            for (int idx = g; idx < 2 * 512; idx += 128) {
                const int pn = idx >> 9, w = idx & 511, r = w >> 3, c = w & 7;
                const uint32_t ka = sbase + kq + pn * 16384 + sw128_off(r, c);
                const uint32_t qa = sbase + kq + pn * 16384 + sw128_off(r + 64, c);
                uint32_t kw[4], qw[4];
                asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                             : "=r"(kw[0]), "=r"(kw[1]), "=r"(kw[2]), "=r"(kw[3]) : "r"(ka));
                asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                             : "=r"(qw[0]), "=r"(qw[1]), "=r"(qw[2]), "=r"(qw[3]) : "r"(qa));
                float x[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 kk = *reinterpret_cast<const __nv_bfloat162*>(&kw[e]);
                    const __nv_bfloat162 qq = *reinterpret_cast<const __nv_bfloat162*>(&qw[e]);
                    x[2 * e] = __low2float(qq) - a.dcorr * __low2float(kk);
                    x[2 * e + 1] = __high2float(qq) - a.dcorr * __high2float(kk);
                }
                st_bf16x8(qa, x);
            }
            if (g < C) {
                const int r = g;
                const float* la = rec;
                const float* lm = rec + C;
                const float* bb = rec + 2 * C;
                vec[VA + r] = expf(la[r]);
                vec[VD2 + r] = rec[3 * C + r] * (r > 0 ? bb[r - 1] : 0.f);
                vec[VB + r] = bb[r];
                vec[VWM + r] = rec[5 * C + r] * expf(lm[C - 1] - lm[r]);
                vec[VMU + r] = expf(lm[r] - (r > 0 ? lm[r - 1] : 0.f));
                if (r == 0) {
                    scal[0] = expf(la[C - 1]);
                    scal[1] = bb[C - 1];
                    scal[2] = expf(lm[C - 1]);
                }
            }
            fence_proxy_async_smem();
            named_bar(NB_PREP);

            // G = [K; Qhat] [K; Qhat]^T
            if (g == 0) {
                tc_fence_after_sync();
                const uint32_t id = idesc_bf16(128, 128, false, false);
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t ad =
                        smem_desc(sbase + kq + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128);
                    mma_bf16(tmem + TM_G, ad, ad, id, ks > 0);
                }
                mma_commit(&bars[B_PREP_MMA]);
            }
            ok = mbar_wait(&bars[B_PREP_MMA], ph);
            ph ^= 1u;
            tc_fence_after_sync();
            ok = named_bar_and(NB_PREP, ok);
            if (!ok) break;

            // one pass down column i (lanes 0..63): Gamma, A and Att
            if (warp < 6) {
                const int i = g;
                float kk[64], kqv[64];
                tmem_ld32(tmem + lane_sel + TM_G, *reinterpret_cast<float(*)[32]>(kk));
                tmem_ld32(tmem + lane_sel + TM_G + 32, *reinterpret_cast<float(*)[32]>(kk + 32));
                tmem_ld32(tmem + lane_sel + TM_G + 64, *reinterpret_cast<float(*)[32]>(kqv));
                tmem_ld32(tmem + lane_sel + TM_G + 96, *reinterpret_cast<float(*)[32]>(kqv + 32));
                tmem_wait_ld();
                if (dump)
                    for (int j = 0; j < 64; ++j) {
                        a.dbg[DBG_G + i * 128 + j] = kk[j];
                        a.dbg[DBG_G + i * 128 + 64 + j] = kqv[j];
                    }
                const float* al = rec + 3 * C;
                const float* be = rec + 4 * C;
                const float eta_i = rec[5 * C + i];
                float gam = 0.f, f = 1.f;
                const uint32_t att_col = sbase + IATT + ((i & 7) << 1);
#pragma unroll
                for (int r = 0; r < C; ++r) {
                    const float ar = al[r];
                    const float av = (r > i) ? ar * kk[r] * gam : 0.f;
                    if (r == i) {
                        gam = eta_i * be[r];
                        f = 1.f;
                    } else if (r > i) {
                        f *= vec[VMU + r];
                        gam = fmaf(ar, gam, eta_i * be[r] * f);
                    }
                    const float att = (r >= i) ? kqv[r] * gam : 0.f;
                    Am[r * LDF + i] = av;
                    const __nv_bfloat16 hb = __float2bfloat16_rn(att);
                    asm volatile("st.shared.b16 [%0], %1;" ::"r"(att_col + sw128_off(64 + r, i >> 3)),
                                 "h"(*reinterpret_cast<const unsigned short*>(&hb))
                                 : "memory");
                }
                vec[VWG + i] = gam;
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar(NB_PREP);

            // T = (I + A)^{-1}: diagonal 16x16 blocks
            if (g < C) {
                const int blk = g >> 4, c = g & 15, o = 16 * blk;
                float t[16];
#pragma unroll
                for (int r = 0; r < 16; ++r) t[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
                for (int r = 1; r < 16; ++r) {
                    float av[16];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 v4 = lds4(Am + (o + r) * LDF + o + 4 * q4);
                        av[4 * q4] = v4.x;
                        av[4 * q4 + 1] = v4.y;
                        av[4 * q4 + 2] = v4.z;
                        av[4 * q4 + 3] = v4.w;
                    }
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < r; ++k) acc = fmaf(av[k], t[k], acc);
                    if (r > c) t[r] = -acc;
                }
#pragma unroll
                for (int r = 0; r < 16; ++r) Tm[(o + r) * LDF + o + c] = t[r];
            } else {
                // zero the six blocks above the diagonal
                for (int idx = g - C; idx < 6 * 64; idx += 64) {
                    const int blkid = idx >> 6, e = idx & 63;
                    const int bi = blkid < 3 ? 0 : (blkid < 5 ? 1 : 2);
                    const int bj = blkid < 3 ? blkid + 1 : (blkid < 5 ? blkid - 1 : 3);
                    *reinterpret_cast<float4*>(Tm + (16 * bi + (e >> 2)) * LDF + 16 * bj +
                                               4 * (e & 3)) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            named_bar(NB_PREP);
            // off-diagonal blocks by distance L: W = sum_{k=j}^{i-1} A_{i,k} T_{k,j},
            // T_{i,j} = -T_{i,i} W (j = i - L); W goes to block (L-1, i) of Am.
            for (int L = 1; L < 4; ++L) {
                const int tasks = (4 - L) * 64;
                for (int task = g; task < tasks; task += 128) {
                    const int i = L + (task >> 6), j = i - L, r = (task >> 2) & 15, c4 = task & 3;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int kb = j; kb < i; ++kb) {
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const float4 a4 = lds4(Am + (16 * i + r) * LDF + 16 * kb + 4 * k4);
                            const float ae[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float4 t4 =
                                    lds4(Tm + (16 * kb + 4 * k4 + e) * LDF + 16 * j + 4 * c4);
                                acc.x = fmaf(ae[e], t4.x, acc.x);
                                acc.y = fmaf(ae[e], t4.y, acc.y);
                                acc.z = fmaf(ae[e], t4.z, acc.z);
                                acc.w = fmaf(ae[e], t4.w, acc.w);
                            }
                        }
                    }
                    *reinterpret_cast<float4*>(Am + (16 * (L - 1) + r) * LDF + 16 * i + 4 * c4) = acc;
                }
                named_bar(NB_PREP);
                for (int task = g; task < tasks; task += 128) {
                    const int i = L + (task >> 6), j = i - L, r = (task >> 2) & 15, c4 = task & 3;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const float4 a4 = lds4(Tm + (16 * i + r) * LDF + 16 * i + 4 * k4);
                        const float ae[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float4 w4 =
                                lds4(Am + (16 * (L - 1) + 4 * k4 + e) * LDF + 16 * i + 4 * c4);
                            acc.x = fmaf(ae[e], w4.x, acc.x);
                            acc.y = fmaf(ae[e], w4.y, acc.y);
                            acc.z = fmaf(ae[e], w4.z, acc.z);
                            acc.w = fmaf(ae[e], w4.w, acc.w);
                        }
                    }
                    *reinterpret_cast<float4*>(Tm + (16 * i + r) * LDF + 16 * j + 4 * c4) =
                        make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
                }
                named_bar(NB_PREP);
            }
            if (dump && g < C)
                for (int j = 0; j < C; ++j) {
                    a.dbg[DBG_A + g * C + j] = (j < g) ? Am[g * LDF + j] : 0.f;
                    a.dbg[DBG_T + g * C + j] = Tm[g * LDF + j];
                }

            // T (bf16, rows k) and [D_G T | -D_w T]
            {
                const int r = g & 63;
                const bool first = g < 64;
                const float w = first ? vec[VWG + r] : -vec[VWM + r];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 t0 = lds4(Tm + r * LDF + 8 * c);
                    const float4 t1 = lds4(Tm + r * LDF + 8 * c + 4);
                    float x[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[e] = w * x[e];
                    if (first) st_bf16x8(sbase + TB + sw128_off(r, c), x);
                    st_bf16x8(sbase + DT + (first ? 0 : 8192) + sw128_off(r, c), y);
                }
            }
            fence_proxy_async_smem();
            named_bar(NB_PREP);

            // P = [I; Att] T and R = K^T [D_G T | -D_w T]
            if (g == 0) {
                tc_fence_after_sync();
                const uint32_t idp = idesc_bf16(128, 64, false, true);
                const uint32_t idr = idesc_bf16(128, 128, true, true);
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_P, smem_desc(sbase + IATT + ks * 32, 16, 1024, kSw128),
                             smem_desc(sbase + TB + ks * 2048, 8192, 1024, kSw128), idp, ks > 0);
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_R, smem_desc(sbase + kq + ks * 2048, 16384, 1024, kSw128),
                             smem_desc(sbase + DT + ks * 2048, 8192, 1024, kSw128), idr, ks > 0);
                mma_commit(&bars[B_PREP_MMA]);
            }
            ok = mbar_wait(&bars[B_PREP_MMA], ph);
            ph ^= 1u;
            tc_fence_after_sync();
            // the chain must be done reading [T; Att T] and A2T of the previous chunk
            if (p > 0) ok = ok && mbar_wait(&bars[B_OPS_FREE], (p - 1) & 1);
            ok = named_bar_and(NB_PREP, ok);
            if (!ok) break;

            // [T; Att T] and A2T to bf16 operands
            {
                float v[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tmem + lane_sel + TM_P + 32 * half, v);
                    tmem_wait_ld();
                    if (dump)
                        for (int j = 0; j < 32; ++j) a.dbg[DBG_P + g * 64 + 32 * half + j] = v[j];
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        st_bf16x8(sbase + TAT + sw128_off(g, 4 * half + c), v + 8 * c);
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    tmem_ld32(tmem + lane_sel + TM_R + 32 * q4, v);
                    tmem_wait_ld();
                    if (dump)
                        for (int j = 0; j < 32; ++j) a.dbg[DBG_R + g * 128 + 32 * q4 + j] = v[j];
                    const uint32_t panel = A2T + (q4 >> 1) * 16384;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        st_bf16x8(sbase + panel + sw128_off(g, 4 * (q4 & 1) + c), v + 8 * c);
                }
            }
            if (dump && g < C) {
                for (int k = 0; k < 6; ++k) a.dbg[DBG_VEC + k * 64 + g] = vec[k * 64 + g];
                if (g < 3) a.dbg[DBG_VEC + 384 + g] = scal[g];
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar(NB_PREP);
            if (g == 0) mbar_arrive(&bars[B_PREP_READY]);
        }
    } else {
        // ================================================================ chain group
        uint32_t ph = 0;  // parity of the next completion of B_CHAIN_MMA
        const int r = g & 63;
        for (int n = 0; n < a.NT; ++n) {
            const int buf = n & 1;
            const uint32_t kq = KQ0 + buf * KQ_BYTES;
            const float* vec = reinterpret_cast<const float*>(sm + VEC0 + buf * 1536);
            const float* scal = reinterpret_cast<const float*>(sm + SCAL0 + buf * 16);
            const bool dump = a.dbg != nullptr && blockIdx.x == 0 && n == 0;
            ok = named_bar_and(NB_CHAIN, mbar_wait(&bars[B_PREP_READY], n & 1));
            if (!ok) break;
            const float c_ab = vec[VA + r], c_d2 = vec[VD2 + r], c_b = vec[VB + r];
            const float abC = scal[0], bC = scal[1], mbC = scal[2];

            // A1 = [K; Qhat] [S | M]
            if (g == 0) {
                tc_fence_after_sync();
                const uint32_t id = idesc_bf16(128, 64, false, true);
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + TM_A1,
                             smem_desc(sbase + kq + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024,
                                       kSw128),
                             smem_desc(sbase + ST + ks * 2048, 8192, 1024, kSw128), id, ks > 0);
                mma_commit(&bars[B_CHAIN_MMA]);
            }
            ok = mbar_wait(&bars[B_CHAIN_MMA], ph);
            ph ^= 1u;
            tc_fence_after_sync();
            ok = named_bar_and(NB_CHAIN, ok);
            if (!ok) break;

            // Y = V - X (rows 0..63); Oi kept in registers (rows 64..127)
            float oi[NS];
            {
                float x[32], y[32];
                tmem_ld32(tmem + lane_sel + TM_A1, x);
                tmem_ld32(tmem + lane_sel + TM_A1 + 32, y);
                tmem_wait_ld();
                if (dump)
                    for (int j = 0; j < 32; ++j) {
                        a.dbg[DBG_A1 + g * 64 + j] = x[j];
                        a.dbg[DBG_A1 + g * 64 + 32 + j] = y[j];
                    }
                if (g < C) {
                    const __nv_bfloat16* vrow =
                        reinterpret_cast<const __nv_bfloat16*>(sm + V0 + buf * 4096 + r * 64);
                    float yy[NS];
#pragma unroll
                    for (int j = 0; j < NS; ++j)
                        yy[j] = __bfloat162float(vrow[j]) - (c_ab * x[j] - c_d2 * y[j]);
                    if (dump)
                        for (int j = 0; j < NS; ++j) a.dbg[DBG_Y + r * NS + j] = yy[j];
#pragma unroll
                    for (int c = 0; c < 4; ++c) st_bf16x8(sbase + YB + sw64_off(r, c), yy + 8 * c);
                } else {
#pragma unroll
                    for (int j = 0; j < NS; ++j) oi[j] = c_ab * x[j] - c_b * y[j];
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar(NB_CHAIN);

            if (g == 0) {
                // K, Q, V and the record of this buffer are no longer needed
                if (n + 2 < a.NT) issue_loads(n + 2);
                // A2 = [A2T_S; A2T_M] Y and A3 = [T; Att T] Y
                tc_fence_after_sync();
                const uint32_t id = idesc_bf16(128, 32, false, true);
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t yd = smem_desc(sbase + YB + ks * 1024, 4096, 512, kSw64);
                    mma_bf16(tmem + TM_A2, smem_desc(sbase + A2T + ks * 32, 16, 1024, kSw128), yd,
                             id, ks > 0);
                    mma_bf16(tmem + TM_A2 + 32,
                             smem_desc(sbase + A2T + 16384 + ks * 32, 16, 1024, kSw128), yd, id,
                             ks > 0);
                    mma_bf16(tmem + TM_A3, smem_desc(sbase + TAT + ks * 32, 16, 1024, kSw128), yd,
                             id, ks > 0);
                }
                mma_commit(&bars[B_CHAIN_MMA]);
            }
            ok = mbar_wait(&bars[B_CHAIN_MMA], ph);
            ph ^= 1u;
            tc_fence_after_sync();
            if (g == 0 && ok) mbar_arrive(&bars[B_OPS_FREE]);
            ok = named_bar_and(NB_CHAIN, ok);
            if (!ok) break;

            // state update; Vtilde and o
            {
                float dS[32], dM[32], o3[32];
                tmem_ld32(tmem + lane_sel + TM_A2, dS);
                tmem_ld32(tmem + lane_sel + TM_A2 + 32, dM);
                tmem_ld32(tmem + lane_sel + TM_A3, o3);
                tmem_wait_ld();
                if (dump)
                    for (int j = 0; j < 32; ++j) {
                        a.dbg[DBG_A2 + g * 64 + j] = dS[j];
                        a.dbg[DBG_A2 + g * 64 + 32 + j] = dM[j];
                        a.dbg[DBG_A3 + g * 32 + j] = o3[j];
                    }
#pragma unroll
                for (int j = 0; j < NS; ++j) {
                    const float sn = fmaf(abC, s[j], fmaf(-bC, m[j], dS[j]));
                    m[j] = fmaf(mbC, m[j], dM[j]);
                    s[j] = sn;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    st_bf16x8(sbase + ST + sw128_off(g, c), s + 8 * c);
                    st_bf16x8(sbase + ST + sw128_off(g, 4 + c), m + 8 * c);
                }
                if (dump)
                    for (int j = 0; j < NS; ++j) {
                        a.dbg[DBG_S + g * NS + j] = s[j];
                        a.dbg[DBG_M + g * NS + j] = m[j];
                    }
                const int t = n * C + r;
                if (t < a.T) {
                    __nv_bfloat16* dst =
                        (g < C ? a.vt : a.o) + (((size_t)b * a.T + t) * a.H + h) * D + j0;
                    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            w[e] = (g < C) ? o3[8 * c + e] : o3[8 * c + e] + oi[8 * c + e];
                        d4[c] = make_uint4(pack_bf16(w[0], w[1]), pack_bf16(w[2], w[3]),
                                           pack_bf16(w[4], w[5]), pack_bf16(w[6], w[7]));
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar(NB_CHAIN);
        }
        if (ok) {
            const size_t row = ((size_t)bh * D + g) * D + j0;
#pragma unroll
            for (int j = 0; j < NS; ++j) {
                a.S_T[row + j] = s[j];
                a.M_T[row + j] = m[j];
            }
        }
    }

    if (!ok && g == 0) atomicOr(a.status + 1, 1u);
    // Loads that were issued must land before the CTA's shared memory is
    // released; only the last two chunks' buffers can still be in flight.
    if (!ok && tid == 0) {
        for (int n = a.NT - 2; n < a.NT; ++n)
            if (n >= 0) (void)mbar_wait(&bars[B_FULL0 + (n & 1)], (n >> 1) & 1);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 4-D map over a [B, T, H, D] bf16 tensor; box = {box_d, 1, 64, 1}.
bool make_map(CUtensorMap* map, const void* base, int B, int T, int H, int box_d, bool swizzle128)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t s)
{
    if (a.D != D) return cudaErrorNotSupported;
    cudaError_t e = launch_gate_pack(a.alpha_log, a.mu_log, a.beta, a.eta, a.B, a.T, a.H, a.rec, s);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.T, a.H, 64, true) || !make_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_map(&mv, a.v, a.B, a.T, a.H, NS, false))
        return cudaErrorInvalidValue;
    TcArgs t;
    t.rec = a.rec;
    t.S0 = a.S0;
    t.M0 = a.M0;
    t.S_T = a.S_T;
    t.M_T = a.M_T;
    t.o = static_cast<__nv_bfloat16*>(a.o);
    t.vt = static_cast<__nv_bfloat16*>(a.vt);
    t.status = a.status;
    t.dbg = a.dbg;
    t.dcorr = a.dcorr;
    t.B = a.B;
    t.T = a.T;
    t.H = a.H;
    t.NT = a.NT;
    static bool attr_set = false;
    if (!attr_set) {
        e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const long long blocks = (long long)a.B * a.H * (D / NS);
    ProfScope ps(kChunkTc, s);
    chunk_tc_kernel<<<(unsigned)blocks, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, t);
    return cudaGetLastError();
}

}  // namespace mdn
