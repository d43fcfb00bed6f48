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
// Vtilde are independent), and walks the chunks in order.  Per chunk:
//   prep (independent of the state)
//     G    = [K; Qhat] K^T                      (M=128, N=64, K=128)   tensor cores
//     Gamma by its column recurrence, A = alpha_r (K K^T) o Gamma-,
//     Att = (Qhat K^T) o Gamma                                          CUDA cores
//     T = (I + A)^{-1}, blocked 16x16 forward substitution in fp32      CUDA cores
//     P    = [I; Att] T       -> [T; Att T]      (M=128, N=64, K=64)    tensor cores
//     R    = K^T [D_G T | -D_w T] -> A2T         (M=128, N=128, K=64)   tensor cores
//   chain (depends on the state)
//     A1   = [K; Qhat] [S | M]                   (M=128, N=64, K=128)
//     Y    = V - (D1 KS - D2 KM);  Oi = Diag(alphabar) QhatS - Diag(b) QhatM
//     A2   = [A2T_S; A2T_M] Y  (two M=128, N=32, K=64);  A3 = [T; Att T] Y (M=128, N=32, K=64)
//     S, M <- (alphabar_C S - b_C M, mubar_C M) + A2;  Vtilde = A3[0:64];  o = Oi + A3[64:128]
// The fp32 state lives in registers (thread i owns row i of S and M for the
// CTA's 32 columns); its bf16 copy in shared memory is the B operand of A1.
// Every wait on an mbarrier is bounded; a wait that runs out sets status[1]
// and the CTA stops.
#include <cudaTypedefs.h>

#include <mutex>

#include "mdn_internal.cuh"
#include "sm100.cuh"

namespace mdn {
namespace {

using namespace sm100;

constexpr int C = 64;        // chunk length
constexpr int D = 128;       // d_k = d_v
constexpr int NS = 32;       // d_v columns per CTA
constexpr int kThreads = 128;
constexpr int kRecFloats = 6 * C;
constexpr uint32_t kTmemCols = 512;

// Shared memory map (byte offsets from a 1024-byte aligned base).
constexpr uint32_t KQ0 = 0;               // [K;Qhat], 2 feature panels x (128 rows x 128 B)
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t IATT = 2 * KQ_BYTES;   // [I; Att]   128 x 64 bf16, K-major SW128
constexpr uint32_t TB = IATT + 16384;     // T          64 x 64 bf16, rows k (MN-major SW128)
constexpr uint32_t DT = TB + 8192;        // [D_G T | -D_w T], 2 panels of 64 x 64
constexpr uint32_t TAT = DT + 16384;      // [T; Att T] 128 x 64 bf16, K-major SW128
constexpr uint32_t A2T = TAT + 16384;     // [A2T_S | A2T_M], 2 panels of 128 x 64, K-major
constexpr uint32_t ST = A2T + 32768;      // [S | M] bf16, 128 rows x (32 + 32), MN-major SW128
constexpr uint32_t YB = ST + 16384;       // Y 64 x 32 bf16, MN-major SW64
constexpr uint32_t V0 = YB + 4096;        // V slice 64 x 32 bf16 (plain rows), 2 buffers
constexpr uint32_t REC0 = V0 + 8192;      // coefficient records, 2 buffers of 1536 B
constexpr uint32_t VEC = REC0 + 2 * 1536; // abar[64], d2[64], wG[64], wM[64], scalars[8]
constexpr uint32_t GAM = VEC + 1280;      // fp32 [64][65]: Gamma, then T
constexpr uint32_t AMAT = GAM + 16640;    // fp32 [64][65]: A (upper blocks: solve scratch)
constexpr uint32_t BARS = AMAT + 16640;   // mbarriers: full[2], mma
constexpr uint32_t MISC = BARS + 32;      // tmem base, abort flag
constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;  // + alignment slack
constexpr int LD = C + 1;                 // leading dimension of the fp32 matrices

// TMEM columns
constexpr uint32_t TM_G = 0, TM_P = 64, TM_R = 128, TM_A1 = 256, TM_A2 = 320, TM_A3 = 384;

constexpr uint32_t kTxBytes = KQ_BYTES + 4096 + 1536;  // 2 K + 2 Q boxes, V box, record

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
constexpr int DBG_G = 0, DBG_GAM = 8192, DBG_A = 12288, DBG_T = 16384, DBG_P = 20480,
              DBG_R = 28672, DBG_A1 = 45056, DBG_Y = 53248, DBG_A2 = 55296, DBG_A3 = 63488,
              DBG_S = 67584, DBG_M = 71680, DBG_VEC = 75776, DBG_FLOATS = 76096;

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

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const TcArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int slice = blockIdx.x % (D / NS);
    const int bh = blockIdx.x / (D / NS);
    const int b = bh / a.H, h = bh % a.H;
    const int j0 = slice * NS;

    uint64_t* full = reinterpret_cast<uint64_t*>(sm + BARS);
    uint64_t* mbar = full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);
    float* abar_v = reinterpret_cast<float*>(sm + VEC);
    float* d2_v = abar_v + C;
    float* wG_v = d2_v + C;
    float* wM_v = wG_v + C;
    float* scal = wM_v + C;  // alphabar_C, b_C, mubar_C
    float* Gm = reinterpret_cast<float*>(sm + GAM);   // Gamma, later T
    float* Am = reinterpret_cast<float*>(sm + AMAT);

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(mbar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // Identity rows 0..63 of [I; Att] (written once).
    if (tid < C) {
        const int r = tid;
        for (int c = 0; c < 8; ++c) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = (8 * c + e == r) ? 1.f : 0.f;
            st_bf16x8(sbase + IATT + sw128_off(r, c), x);
        }
    }
    // Entering state: thread i owns row i of S and M for columns j0..j0+31.
    float s[NS], m[NS];
    {
        const size_t row = ((size_t)bh * D + tid) * D + j0;
#pragma unroll
        for (int j = 0; j < NS; ++j) {
            s[j] = a.S0 ? a.S0[row + j] : 0.f;
            m[j] = a.M0 ? a.M0[row + j] : 0.f;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            st_bf16x8(sbase + ST + sw128_off(tid, c), s + 8 * c);
            st_bf16x8(sbase + ST + sw128_off(tid, 4 + c), m + 8 * c);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_sel = static_cast<uint32_t>(warp * 32) << 16;

    auto issue_loads = [&](int n, int buf) {
        const uint32_t kq = KQ0 + buf * KQ_BYTES;
        mbar_arrive_expect_tx(&full[buf], kTxBytes);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_4d(sm + kq + p * 16384, &tm_k, p * 64, h, n * C, b, &full[buf]);
            tma_load_4d(sm + kq + p * 16384 + 8192, &tm_q, p * 64, h, n * C, b, &full[buf]);
        }
        tma_load_4d(sm + V0 + buf * 4096, &tm_v, j0, h, n * C, b, &full[buf]);
        bulk_load(sm + REC0 + buf * 1536, a.rec + ((size_t)bh * a.NT + n) * kRecFloats, 1536,
                  &full[buf]);
    };

    bool ok = true;
    uint32_t mma_phase = 0;
    int issued = 0;  // chunks whose loads were issued
    if (tid == 0 && a.NT > 0) { issue_loads(0, 0); }
    issued = a.NT > 0 ? 1 : 0;

    auto wait_mma = [&]() -> bool {
        const bool w = mbar_wait(mbar, mma_phase);
        mma_phase ^= 1u;
        tc_fence_after_sync();
        return w;
    };

    for (int n = 0; n < a.NT && ok; ++n) {
        const int buf = n & 1;
        const uint32_t kq = KQ0 + buf * KQ_BYTES;
        const float* rec = reinterpret_cast<const float*>(sm + REC0 + buf * 1536);
        if (tid == 0 && n + 1 < a.NT) issue_loads(n + 1, buf ^ 1);
        if (n + 1 < a.NT) issued = n + 2;
        ok = __syncthreads_and(mbar_wait(&full[buf], (n >> 1) & 1));
        if (!ok) break;

        // ---- step 1: Qhat = Q - d K in place; per-position vectors; Gamma columns
        if (tid >= C) {
            for (int idx = tid - C; idx < 2 * 512; idx += C) {
                const int p = idx >> 9, w = idx & 511, r = w >> 3, c = w & 7;
                const uint32_t ka = sbase + kq + p * 16384 + sw128_off(r, c);
                const uint32_t qa = sbase + kq + p * 16384 + sw128_off(r + 64, c);
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
        } else {
            const int r = tid;
            const float* la = rec;
            const float* lm = rec + C;
            const float* bb = rec + 2 * C;
            const float* al = rec + 3 * C;
            const float* be = rec + 4 * C;
            const float* et = rec + 5 * C;
            abar_v[r] = expf(la[r]);
            d2_v[r] = al[r] * (r > 0 ? bb[r - 1] : 0.f);
            wM_v[r] = et[r] * expf(lm[C - 1] - lm[r]);
            if (r == 0) {
                scal[0] = expf(la[C - 1]);
                scal[1] = bb[C - 1];
                scal[2] = expf(lm[C - 1]);
            }
            // Column r of Gamma: Gamma_{t,r} = alpha_t Gamma_{t-1,r} + eta_r beta_t mubar_t/mubar_r
            const float eta_i = et[r], lm_i = lm[r];
            float g = 0.f;
            for (int t = 0; t < C; ++t) {
                g = (t >= r) ? fmaf(al[t], g, eta_i * be[t] * expf(lm[t] - lm_i)) : 0.f;
                Gm[t * LD + r] = g;
            }
            wG_v[r] = g;
        }
        fence_proxy_async_smem();
        __syncthreads();
        const bool dump = a.dbg != nullptr && blockIdx.x == 0 && n == 0;
        if (dump && tid < C) {
            for (int i = 0; i < C; ++i) a.dbg[DBG_GAM + tid * C + i] = Gm[tid * LD + i];
            a.dbg[DBG_VEC + tid] = abar_v[tid];
            a.dbg[DBG_VEC + C + tid] = d2_v[tid];
            a.dbg[DBG_VEC + 2 * C + tid] = wG_v[tid];
            a.dbg[DBG_VEC + 3 * C + tid] = wM_v[tid];
            if (tid < 3) a.dbg[DBG_VEC + 4 * C + tid] = scal[tid];
        }

        // ---- step 2: G = [K; Qhat] K^T
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t id = idesc_bf16(128, 64, false, false);
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = kq + (ks >> 2) * 16384 + (ks & 3) * 32;
                const uint64_t ad = smem_desc(sbase + off, 16, 1024, kSw128);
                mma_bf16(tmem + TM_G, ad, ad, id, ks > 0);
            }
            mma_commit(mbar);
        }
        ok = __syncthreads_and(wait_mma());
        if (!ok) break;

        // ---- step 3: A (rows 0..63) and Att (rows 64..127)
        {
            float g[64];
            tmem_ld32(tmem + lane_sel + TM_G, *reinterpret_cast<float(*)[32]>(g));
            tmem_ld32(tmem + lane_sel + TM_G + 32, *reinterpret_cast<float(*)[32]>(g + 32));
            tmem_wait_ld();
            if (dump)
                for (int i = 0; i < C; ++i) a.dbg[DBG_G + tid * C + i] = g[i];
            if (tid < C) {
                const int r = tid;
                const float ar = rec[3 * C + r];
                for (int i = 0; i < C; ++i)
                    Am[r * LD + i] = (i < r) ? ar * g[i] * Gm[(r - 1) * LD + i] : 0.f;
            } else {
                const int r = tid - C;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = 8 * c + e;
                        x[e] = (i <= r) ? g[i] * Gm[r * LD + i] : 0.f;
                    }
                    st_bf16x8(sbase + IATT + sw128_off(tid, c), x);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- step 4: T = (I + A)^{-1} into Gm (blocked by 16)
        float* Tm = Gm;
        if (tid < C) {
            const int blk = tid >> 4, c = tid & 15, o = 16 * blk;
            float t[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) t[r] = (r == c) ? 1.f : 0.f;
#pragma unroll
            for (int r = 1; r < 16; ++r) {
                if (r > c) {
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < r; ++k) acc = fmaf(Am[(o + r) * LD + o + k], t[k], acc);
                    t[r] = -acc;
                }
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tm[(o + r) * LD + o + c] = t[r];
        } else {
            // zero the blocks above the diagonal
            for (int idx = tid - C; idx < 6 * 256; idx += C) {
                const int blkid = idx >> 8, e = idx & 255;
                const int bi = blkid < 3 ? 0 : (blkid < 5 ? 1 : 2);
                const int bj = blkid < 3 ? blkid + 1 : (blkid < 5 ? blkid - 1 : 3);
                Tm[(16 * bi + (e >> 4)) * LD + 16 * bj + (e & 15)] = 0.f;
            }
        }
        __syncthreads();
        // Off-diagonal blocks, by distance L from the diagonal:
        //   W = sum_{k=j}^{i-1} A_{i,k} T_{k,j};  T_{i,j} = -T_{i,i} W,  j = i - L.
        // W goes to the (unused) block (L-1, i) above the diagonal of Am.
        for (int L = 1; L < 4; ++L) {
            const int nblk = 4 - L;
            for (int idx = tid; idx < nblk * 256; idx += kThreads) {
                const int i = L + (idx >> 8), j = i - L, r = (idx >> 4) & 15, c = idx & 15;
                float acc = 0.f;
                for (int kb = j; kb < i; ++kb) {
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        acc = fmaf(Am[(16 * i + r) * LD + 16 * kb + k],
                                   Tm[(16 * kb + k) * LD + 16 * j + c], acc);
                }
                Am[(16 * (L - 1) + r) * LD + 16 * i + c] = acc;
            }
            __syncthreads();
            for (int idx = tid; idx < nblk * 256; idx += kThreads) {
                const int i = L + (idx >> 8), j = i - L, r = (idx >> 4) & 15, c = idx & 15;
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    acc = fmaf(Tm[(16 * i + r) * LD + 16 * i + k],
                               Am[(16 * (L - 1) + k) * LD + 16 * i + c], acc);
                Tm[(16 * i + r) * LD + 16 * j + c] = -acc;
            }
            __syncthreads();
        }

        if (dump && tid < C)
            for (int i = 0; i < C; ++i) {
                a.dbg[DBG_A + tid * C + i] = Am[tid * LD + i];
                a.dbg[DBG_T + tid * C + i] = Tm[tid * LD + i];
            }

        // ---- step 5: T (bf16, rows k) and [D_G T | -D_w T]
        if (tid < C) {
            const int r = tid;
            const float wg = wG_v[r], wm = -wM_v[r];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float x[8], y[8], z[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    x[e] = Tm[r * LD + 8 * c + e];
                    y[e] = wg * x[e];
                    z[e] = wm * x[e];
                }
                st_bf16x8(sbase + TB + sw128_off(r, c), x);
                st_bf16x8(sbase + DT + sw128_off(r, c), y);
                st_bf16x8(sbase + DT + 8192 + sw128_off(r, c), z);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- step 6: P = [I; Att] T and R = K^T [D_G T | -D_w T]
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t idp = idesc_bf16(128, 64, false, true);
            const uint32_t idr = idesc_bf16(128, 128, true, true);
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + TM_P, smem_desc(sbase + IATT + ks * 32, 16, 1024, kSw128),
                         smem_desc(sbase + TB + ks * 2048, 8192, 1024, kSw128), idp, ks > 0);
            }
            for (int ks = 0; ks < 4; ++ks) {
                mma_bf16(tmem + TM_R, smem_desc(sbase + kq + ks * 2048, 16384, 1024, kSw128),
                         smem_desc(sbase + DT + ks * 2048, 8192, 1024, kSw128), idr, ks > 0);
            }
            mma_commit(mbar);
        }
        ok = __syncthreads_and(wait_mma());
        if (!ok) break;

        // ---- step 7: [T; Att T] and A2T to bf16 operands
        {
            float v[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(tmem + lane_sel + TM_P + 32 * half, v);
                tmem_wait_ld();
                if (dump)
                    for (int i = 0; i < 32; ++i) a.dbg[DBG_P + tid * 64 + 32 * half + i] = v[i];
#pragma unroll
                for (int c = 0; c < 4; ++c) st_bf16x8(sbase + TAT + sw128_off(tid, 4 * half + c), v + 8 * c);
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                tmem_ld32(tmem + lane_sel + TM_R + 32 * q4, v);
                tmem_wait_ld();
                if (dump)
                    for (int i = 0; i < 32; ++i) a.dbg[DBG_R + tid * 128 + 32 * q4 + i] = v[i];
                const uint32_t panel = A2T + (q4 >> 1) * 16384;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    st_bf16x8(sbase + panel + sw128_off(tid, 4 * (q4 & 1) + c), v + 8 * c);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- step 8 (chain): A1 = [K; Qhat] [S | M]
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t id = idesc_bf16(128, 64, false, true);
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = kq + (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_bf16(tmem + TM_A1, smem_desc(sbase + off, 16, 1024, kSw128),
                         smem_desc(sbase + ST + ks * 2048, 8192, 1024, kSw128), id, ks > 0);
            }
            mma_commit(mbar);
        }
        ok = __syncthreads_and(wait_mma());
        if (!ok) break;

        // ---- step 9: Y = V - X (rows 0..63); Oi kept in registers (rows 64..127)
        float oi[NS];
        {
            float x[32], y[32];
            tmem_ld32(tmem + lane_sel + TM_A1, x);
            tmem_ld32(tmem + lane_sel + TM_A1 + 32, y);
            tmem_wait_ld();
            if (dump)
                for (int i = 0; i < 32; ++i) {
                    a.dbg[DBG_A1 + tid * 64 + i] = x[i];
                    a.dbg[DBG_A1 + tid * 64 + 32 + i] = y[i];
                }
            if (tid < C) {
                const int r = tid;
                const float da = abar_v[r], d2 = d2_v[r];
                const __nv_bfloat16* vrow =
                    reinterpret_cast<const __nv_bfloat16*>(sm + V0 + buf * 4096 + r * 64);
                float yy[NS];
#pragma unroll
                for (int j = 0; j < NS; ++j)
                    yy[j] = __bfloat162float(vrow[j]) - (da * x[j] - d2 * y[j]);
                if (dump)
                    for (int j = 0; j < NS; ++j) a.dbg[DBG_Y + r * NS + j] = yy[j];
#pragma unroll
                for (int c = 0; c < 4; ++c) st_bf16x8(sbase + YB + sw64_off(r, c), yy + 8 * c);
            } else {
                const int r = tid - C;
                const float da = abar_v[r], db = rec[2 * C + r];
#pragma unroll
                for (int j = 0; j < NS; ++j) oi[j] = da * x[j] - db * y[j];
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        // ---- step 10: A2 = [A2T_S; A2T_M] Y and A3 = [T; Att T] Y
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t id = idesc_bf16(128, 32, false, true);
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t yd = smem_desc(sbase + YB + ks * 1024, 4096, 512, kSw64);
                mma_bf16(tmem + TM_A2, smem_desc(sbase + A2T + ks * 32, 16, 1024, kSw128), yd, id,
                         ks > 0);
                mma_bf16(tmem + TM_A2 + 32,
                         smem_desc(sbase + A2T + 16384 + ks * 32, 16, 1024, kSw128), yd, id,
                         ks > 0);
                mma_bf16(tmem + TM_A3, smem_desc(sbase + TAT + ks * 32, 16, 1024, kSw128), yd, id,
                         ks > 0);
            }
            mma_commit(mbar);
        }
        ok = __syncthreads_and(wait_mma());
        if (!ok) break;

        // ---- step 11: state update; Vtilde and o
        {
            float dS[32], dM[32], o3[32];
            tmem_ld32(tmem + lane_sel + TM_A2, dS);
            tmem_ld32(tmem + lane_sel + TM_A2 + 32, dM);
            tmem_ld32(tmem + lane_sel + TM_A3, o3);
            tmem_wait_ld();
            if (dump)
                for (int i = 0; i < 32; ++i) {
                    a.dbg[DBG_A2 + tid * 64 + i] = dS[i];
                    a.dbg[DBG_A2 + tid * 64 + 32 + i] = dM[i];
                    a.dbg[DBG_A3 + tid * 32 + i] = o3[i];
                }
            const float abC = scal[0], bC = scal[1], mbC = scal[2];
#pragma unroll
            for (int j = 0; j < NS; ++j) {
                const float sn = fmaf(abC, s[j], fmaf(-bC, m[j], dS[j]));
                m[j] = fmaf(mbC, m[j], dM[j]);
                s[j] = sn;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                st_bf16x8(sbase + ST + sw128_off(tid, c), s + 8 * c);
                st_bf16x8(sbase + ST + sw128_off(tid, 4 + c), m + 8 * c);
            }
            if (dump)
                for (int j = 0; j < NS; ++j) {
                    a.dbg[DBG_S + tid * NS + j] = s[j];
                    a.dbg[DBG_M + tid * NS + j] = m[j];
                }
            const int r = tid & (C - 1);
            const int t = n * C + r;
            if (t < a.T) {
                __nv_bfloat16* dst = (tid < C ? a.vt : a.o) +
                                     (((size_t)b * a.T + t) * a.H + h) * D + j0;
                uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        w[e] = (tid < C) ? o3[8 * c + e] : o3[8 * c + e] + oi[8 * c + e];
                    d4[c] = make_uint4(pack_bf16(w[0], w[1]), pack_bf16(w[2], w[3]),
                                       pack_bf16(w[4], w[5]), pack_bf16(w[6], w[7]));
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
    }

    if (ok) {
        const size_t row = ((size_t)bh * D + tid) * D + j0;
#pragma unroll
        for (int j = 0; j < NS; ++j) {
            a.S_T[row + j] = s[j];
            a.M_T[row + j] = m[j];
        }
    } else {
        if (tid == 0) atomicOr(a.status + 1, 1u);
        // Let loads already issued land before the CTA's shared memory goes away.
        for (int k = 0; k < issued && k < a.NT; ++k) (void)mbar_wait(&full[k & 1], (k >> 1) & 1);
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
