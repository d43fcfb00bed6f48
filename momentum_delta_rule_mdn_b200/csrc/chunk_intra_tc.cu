// K-2 on sm_100a: the intra-chunk part of the chunkwise MDN forward pass,
// one CTA per chunk, all chunks in parallel.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, steps 3-5.  Per chunk (positions r, i inside it):
//   Qhat   = Q - d K
//   G      = [K; Qhat] [K; Qhat]^T     tcgen05.mma, M=128, N=128, K=128, bf16 in, fp32 in TMEM
//            lane i < 64: k_i.k_r (cols 0..63);  lane 64+r: qhat_r.k_i (cols 0..63)
//   Gamma  down each column i by Gamma_{r,i} = alpha_r Gamma_{r-1,i} + eta_i beta_r mubar_r/mubar_i
//          (mubar_r/mubar_i as a running product of mu: non-negative terms only)
//   A      = (P K^T) o Gamma-:  A_{r,i} = alpha_r k_r.k_i Gamma_{r-1,i}  (i < r)
//   Att    = (Qhat K^T) o Gamma:  Att_{r,i} = qhat_r.k_i Gamma_{r,i}  (i <= r)
//   T      = (I + A)^{-1}: 16x16 diagonal blocks by forward substitution, then the
//            off-diagonal blocks by distance from the diagonal, fp32
//   P      = [I; Att] T = [T; Att T]                    (M=128, N=64,  K=64)
//   R      = K^T [Diag(Gamma_C) T | -Diag(w) T]          (M=128, N=128, K=64)
//            with w_r = eta_r mubar_C / mubar_r
// and writes, per chunk, the operands of the sequential inter-chunk kernel in
// bf16: Qhat [64 x 128], [T; Att T] [128 x 64], A2T = [R_S; R_M] [256 x 64],
// plus the per-position coefficients alphabar_r, alpha_r b_{r-1}, b_r and the
// chunk scalars alphabar_C, b_C, mubar_C (fp32).
#include "mdn_internal.cuh"
#include "tc_common.cuh"

namespace mdn {
namespace {

using namespace sm100;
using namespace tc;

constexpr int kThreads = 128;
constexpr uint32_t KQ = 0;                   // [K; Qhat], 2 feature panels x (128 rows x 128 B)
constexpr uint32_t GM = 32768;               // fp32 [64][LDF] Gamma;  later [D_G T | -D_w T] bf16
constexpr uint32_t AM = GM + 64 * LDF * 4;   // fp32 [64][LDF] A (upper blocks: scratch); later T bf16
constexpr uint32_t TMF = AM + 64 * LDF * 4;  // fp32 [64][LDF] T
constexpr uint32_t IATT = TMF + 64 * LDF * 4;// [I; Att] 128 x 64 bf16, K-major SW128
constexpr uint32_t REC = IATT + 16384;       // record rows 0..5
constexpr uint32_t VEC = REC + 1536;         // mu_r, w_r, Gamma_{C,r}
constexpr uint32_t BARS = VEC + 768;
constexpr uint32_t MISC = BARS + 16;
constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;
constexpr uint32_t DT = GM;                  // aliases: written after Gamma and A are dead
constexpr uint32_t TB = AM;
static_assert(GM % 1024 == 0 && AM % 1024 == 0 && IATT % 1024 == 0, "operand alignment");
static_assert(SMEM_BYTES <= 116 * 1024, "two CTAs per SM");
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t TM_G = 0, TM_P = 0, TM_R = 128;  // P reuses G's columns once G is read
constexpr uint32_t kTxBytes = 32768;
// staging of the outputs for the TMA stores (regions dead by then)
constexpr uint32_t STG_TAT = IATT;           // 128 x 64 bf16
constexpr uint32_t STG_A2T = GM;             // 256 x 64 bf16 (spans GM and AM)
static_assert(STG_A2T + 32768 <= TMF, "A2T staging overlaps T");

struct IntraArgs {
    const float* alpha_log;  // [B, T, H] gates
    const float* mu_log;
    const float* beta;
    const float* eta;
    __nv_bfloat16* qhat;   // [chunks][64][128]
    __nv_bfloat16* tat;    // [chunks][128][64]
    __nv_bfloat16* a2t;    // [chunks][256][64]
    float* crec;           // [chunks][256]
    unsigned* status;
    float* dbg;            // diagnostics: phase clocks of CTA 0 (null in normal use)
    float dcorr;
    int T, H, NT;
};

__global__ void __launch_bounds__(kThreads)
chunk_intra_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_tat,
                   const __grid_constant__ CUtensorMap tm_a2t, const IntraArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const long long chunk = blockIdx.x;
    const int n = (int)(chunk % a.NT);
    const long long bh = chunk / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);
    float* Gm = reinterpret_cast<float*>(sm + GM);
    float* Am = reinterpret_cast<float*>(sm + AM);
    float* Tm = reinterpret_cast<float*>(sm + TMF);
    float* rec = reinterpret_cast<float*>(sm + REC);
    float* mu = reinterpret_cast<float*>(sm + VEC);
    float* wv = mu + C;    // w_r = eta_r mubar_C / mubar_r
    float* wg = wv + C;    // Gamma_{C,r}
    PhaseClock clk;
    clk.start((a.dbg && chunk == 0 && tid == 0) ? a.dbg : nullptr);
#ifdef MDN_PHASE_CLOCKS
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    const uint64_t t_begin = global_timer_ns();
#endif

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
        mbar_arrive_expect_tx(&bars[0], kTxBytes);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_4d(sm + KQ + p * 16384, &tm_k, p * 64, h, n * C, b, &bars[0]);
            tma_load_4d(sm + KQ + p * 16384 + 8192, &tm_q, p * 64, h, n * C, b, &bars[0]);
        }
    }
    if (warp == 3) {
        // per-position coefficients: la, lm, b, alpha, beta, eta (positions past T are
        // steps that leave the state unchanged)
        const int lane = tid & 31;
        const int t0 = n * C + 2 * lane;
        float ga[2] = {0.f, 0.f}, gm[2] = {0.f, 0.f}, gb[2] = {0.f, 0.f}, ge[2] = {0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (t0 + e < a.T) {
                const size_t gi = ((size_t)b * a.T + t0 + e) * a.H + h;
                ga[e] = a.alpha_log[gi];
                gm[e] = a.mu_log[gi];
                gb[e] = a.beta[gi];
                ge[e] = a.eta[gi];
            }
        }
        float la[2], lm[2], lc[2];
        chunk_log_coeffs(ga, gm, gb, lane, la, lm, lc);
        float2* r2 = reinterpret_cast<float2*>(rec) + lane;
        r2[0] = make_float2(la[0], la[1]);
        r2[32] = make_float2(lm[0], lm[1]);
        r2[64] = make_float2(expf(la[0] + lc[0]), expf(la[1] + lc[1]));
        r2[96] = make_float2(expf(ga[0]), expf(ga[1]));
        r2[128] = make_float2(gb[0], gb[1]);
        r2[160] = make_float2(ge[0], ge[1]);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid < C) {  // identity rows 0..63 of [I; Att]
        for (int c = 0; c < 8; ++c) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = (8 * c + e == tid) ? 1.f : 0.f;
            st_bf16x8(sm + IATT + sw128_off(tid, c), x);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_sel = static_cast<uint32_t>(warp * 32) << 16;

    bool ok = __syncthreads_and(mbar_wait(&bars[0], 0));
    clk.lap(0);
    if (ok) {
        // Qhat = Q - d K in place (rows 64..127 of both panels) and to global memory
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int idx = tid + 128 * u;
            const int pn = idx >> 9, w = idx & 511, r = w >> 3, c = w & 7;
            const uint4 kw = *reinterpret_cast<const uint4*>(sm + KQ + pn * 16384 + sw128_off(r, c));
            uint8_t* qp = sm + KQ + pn * 16384 + sw128_off(r + 64, c);
            float kx[8], qx[8];
            unpack_bf16x8(kw, kx);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(qp), qx);
#pragma unroll
            for (int e = 0; e < 8; ++e) qx[e] -= a.dcorr * kx[e];
            *reinterpret_cast<uint4*>(qp) = bf16x8(qx);
        }
        if (tid < C) {
            const int r = tid;
            const float* la = rec;
            const float* lm = rec + C;
            const float* bb = rec + 2 * C;
            mu[r] = expf(lm[r] - (r > 0 ? lm[r - 1] : 0.f));
            wv[r] = rec[5 * C + r] * expf(lm[C - 1] - lm[r]);
            float* cr = a.crec + chunk * 256;
            cr[r] = expf(la[r]);
            cr[C + r] = rec[3 * C + r] * (r > 0 ? bb[r - 1] : 0.f);
            cr[2 * C + r] = bb[r];
            if (r == 0) {
                cr[3 * C] = expf(la[C - 1]);
                cr[3 * C + 1] = bb[C - 1];
                cr[3 * C + 2] = expf(lm[C - 1]);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        clk.lap(1);
        if (tid == 0) {
            // Qhat (rows 64..127 of both panels) to global memory
            tma_store_3d(&tm_qh, 0, 0, (int)chunk, sm + KQ + 8192);
            tma_store_3d(&tm_qh, 64, 0, (int)chunk, sm + KQ + 16384 + 8192);
            bulk_commit_group();
            tc_fence_after_sync();
            const uint32_t id = idesc_bf16(128, 128, false, false);
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad =
                    smem_desc(sbase + KQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128);
                mma_bf16(tmem + TM_G, ad, ad, id, ks > 0);
            }
            mma_commit(&bars[1]);
        }
        ok = mbar_wait(&bars[1], 0);
        tc_fence_after_sync();
        ok = __syncthreads_and(ok);
        clk.lap(2);
    }
    if (ok) {
        // lane i < 64: k_i.k_r;  lane 64 + r: qhat_r.k_i   (columns 0..63)
        float gv[64];
        tmem_ld32(tmem + lane_sel + TM_G, *reinterpret_cast<float(*)[32]>(gv));
        tmem_ld32(tmem + lane_sel + TM_G + 32, *reinterpret_cast<float(*)[32]>(gv + 32));
        tmem_wait_ld();
        if (tid < C) {
            // column i of Gamma and A
            const int i = tid;
            const float* al = rec + 3 * C;
            const float* be = rec + 4 * C;
            const float eta_i = rec[5 * C + i];
            float gam = 0.f, f = 1.f;
#pragma unroll
            for (int r4 = 0; r4 < C; r4 += 4) {
                const float4 a4 = lds4(al + r4), b4 = lds4(be + r4), m4 = lds4(mu + r4);
                const float ar_[4] = {a4.x, a4.y, a4.z, a4.w};
                const float br_[4] = {b4.x, b4.y, b4.z, b4.w};
                const float mr_[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = r4 + e;
                    Am[r * LDF + i] = (r > i) ? ar_[e] * gv[r] * gam : 0.f;
                    f = (r > i) ? f * mr_[e] : 1.f;
                    gam = (r >= i) ? fmaf(ar_[e], gam, eta_i * br_[e] * f) : 0.f;
                    Gm[r * LDF + i] = gam;
                }
            }
            wg[i] = gam;  // Gamma_{C,i}
        } else {
            // zero the six blocks of T above the diagonal
            for (int idx = tid - C; idx < 6 * 64; idx += 64) {
                const int blkid = idx >> 6, e = idx & 63;
                const int bi = blkid < 3 ? 0 : (blkid < 5 ? 1 : 2);
                const int bj = blkid < 3 ? blkid + 1 : (blkid < 5 ? blkid - 1 : 3);
                *reinterpret_cast<float4*>(Tm + (16 * bi + (e >> 2)) * LDF + 16 * bj + 4 * (e & 3)) =
                    make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        __syncthreads();
        clk.lap(3);
        if (tid >= C) {
            // row r of Att into rows 64..127 of [I; Att]
            const int r = tid - C;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 g0 = lds4(Gm + r * LDF + 8 * c), g1 = lds4(Gm + r * LDF + 8 * c + 4);
                const float gr[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = (8 * c + e <= r) ? gv[8 * c + e] * gr[e] : 0.f;
                st_bf16x8(sm + IATT + sw128_off(tid, c), x);
            }
        } else {
            // diagonal 16x16 blocks of T by forward substitution, one column per thread
            const int blk = tid >> 4, c = tid & 15, o = 16 * blk;
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
        }
        __syncthreads();
        clk.lap(4);
        // Off-diagonal blocks by distance L: W = sum_{k=j}^{i-1} A_{i,k} T_{k,j},
        // T_{i,j} = -T_{i,i} W (j = i - L).  W goes to block (L-1, i) of Am.  A
        // thread owns a 2 x 4 tile of a block.
        for (int L = 1; L < 4; ++L) {
            const int tasks = (4 - L) * 32;
            const int task = tid;
            const bool mine = task < tasks;
            const int i = L + (task >> 5), j = i - L, r0 = 2 * ((task >> 2) & 7), c4 = task & 3;
            if (mine) {
                float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
                for (int kb = j; kb < i; ++kb) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const float4 a0 = lds4(Am + (16 * i + r0) * LDF + 16 * kb + 4 * k4);
                        const float4 a1 = lds4(Am + (16 * i + r0 + 1) * LDF + 16 * kb + 4 * k4);
                        const float x0[4] = {a0.x, a0.y, a0.z, a0.w};
                        const float x1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float4 t4 = lds4(Tm + (16 * kb + 4 * k4 + e) * LDF + 16 * j + 4 * c4);
                            acc0.x = fmaf(x0[e], t4.x, acc0.x);
                            acc0.y = fmaf(x0[e], t4.y, acc0.y);
                            acc0.z = fmaf(x0[e], t4.z, acc0.z);
                            acc0.w = fmaf(x0[e], t4.w, acc0.w);
                            acc1.x = fmaf(x1[e], t4.x, acc1.x);
                            acc1.y = fmaf(x1[e], t4.y, acc1.y);
                            acc1.z = fmaf(x1[e], t4.z, acc1.z);
                            acc1.w = fmaf(x1[e], t4.w, acc1.w);
                        }
                    }
                }
                float* w = Am + (16 * (L - 1) + r0) * LDF + 16 * i + 4 * c4;
                *reinterpret_cast<float4*>(w) = acc0;
                *reinterpret_cast<float4*>(w + LDF) = acc1;
            }
            __syncthreads();
            if (mine) {
                float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const float4 t0 = lds4(Tm + (16 * i + r0) * LDF + 16 * i + 4 * k4);
                    const float4 t1 = lds4(Tm + (16 * i + r0 + 1) * LDF + 16 * i + 4 * k4);
                    const float x0[4] = {t0.x, t0.y, t0.z, t0.w};
                    const float x1[4] = {t1.x, t1.y, t1.z, t1.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 w4 =
                            lds4(Am + (16 * (L - 1) + 4 * k4 + e) * LDF + 16 * i + 4 * c4);
                        acc0.x = fmaf(x0[e], w4.x, acc0.x);
                        acc0.y = fmaf(x0[e], w4.y, acc0.y);
                        acc0.z = fmaf(x0[e], w4.z, acc0.z);
                        acc0.w = fmaf(x0[e], w4.w, acc0.w);
                        acc1.x = fmaf(x1[e], w4.x, acc1.x);
                        acc1.y = fmaf(x1[e], w4.y, acc1.y);
                        acc1.z = fmaf(x1[e], w4.z, acc1.z);
                        acc1.w = fmaf(x1[e], w4.w, acc1.w);
                    }
                }
                float* t = Tm + (16 * i + r0) * LDF + 16 * j + 4 * c4;
                *reinterpret_cast<float4*>(t) = make_float4(-acc0.x, -acc0.y, -acc0.z, -acc0.w);
                *reinterpret_cast<float4*>(t + LDF) = make_float4(-acc1.x, -acc1.y, -acc1.z, -acc1.w);
            }
            __syncthreads();
        }
        clk.lap(5);
        // T (bf16, rows k) and [Diag(Gamma_C) T | -Diag(w) T]; thread = (row, half)
        {
            const int r = tid & 63, hf = tid >> 6;
            const float wr = hf ? -wv[r] : wg[r];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 t0 = lds4(Tm + r * LDF + 8 * c), t1 = lds4(Tm + r * LDF + 8 * c + 4);
                float x[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                if (hf == 0) st_bf16x8(sm + TB + sw128_off(r, c), x);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] *= wr;
                st_bf16x8(sm + DT + hf * 8192 + sw128_off(r, c), x);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        clk.lap(6);
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t idp = idesc_bf16(128, 64, false, true);
            const uint32_t idr = idesc_bf16(128, 128, true, true);
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_P, smem_desc(sbase + IATT + ks * 32, 16, 1024, kSw128),
                         smem_desc(sbase + TB + ks * 2048, 8192, 1024, kSw128), idp, ks > 0);
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_R, smem_desc(sbase + KQ + ks * 2048, 16384, 1024, kSw128),
                         smem_desc(sbase + DT + ks * 2048, 8192, 1024, kSw128), idr, ks > 0);
            mma_commit(&bars[1]);
        }
        ok = mbar_wait(&bars[1], 1);
        tc_fence_after_sync();
        ok = __syncthreads_and(ok);
        clk.lap(7);
    }
    if (ok) {
        // [T; Att T] row = lane and the two A2T rows (lane, 128 + lane) into the
        // swizzled staging tiles, then TMA stores
        float v[64];
        tmem_ld32(tmem + lane_sel + TM_P, *reinterpret_cast<float(*)[32]>(v));
        tmem_ld32(tmem + lane_sel + TM_P + 32, *reinterpret_cast<float(*)[32]>(v + 32));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 8; ++c) st_bf16x8(sm + STG_TAT + sw128_off(tid, c), v + 8 * c);
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
            tmem_ld32(tmem + lane_sel + TM_R + 64 * q2, *reinterpret_cast<float(*)[32]>(v));
            tmem_ld32(tmem + lane_sel + TM_R + 64 * q2 + 32, *reinterpret_cast<float(*)[32]>(v + 32));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 8; ++c)
                st_bf16x8(sm + STG_A2T + q2 * 16384 + sw128_off(tid, c), v + 8 * c);
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_3d(&tm_tat, 0, 0, (int)chunk, sm + STG_TAT);
            tma_store_3d(&tm_a2t, 0, 0, (int)chunk, sm + STG_A2T);
            tma_store_3d(&tm_a2t, 0, 128, (int)chunk, sm + STG_A2T + 16384);
            bulk_commit_group();
        }
        clk.lap(8);
    }
    if (!ok && tid == 0) {
        atomicOr(a.status + 1, 1u);
        (void)mbar_wait(&bars[0], 0);  // the loads must land before shared memory goes away
    }
    clk.flush();
    if (tid == 0) bulk_wait_group_all();  // the stores have read their shared-memory tiles
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
#ifdef MDN_PHASE_CLOCKS
    if (a.dbg && tid == 0 && chunk < 4096) {
        double* tl = reinterpret_cast<double*>(a.dbg + 64);
        tl[3 * chunk] = (double)t_begin;
        tl[3 * chunk + 1] = (double)global_timer_ns();
        tl[3 * chunk + 2] = (double)smid;
    }
#endif
}

}  // namespace

cudaError_t launch_chunk_intra_tc(const ChunkArgs& a, cudaStream_t s)
{
    const long long chunks = (long long)a.B * a.H * a.NT;
    CUtensorMap mq, mk, mqh, mtat, ma2t;
    if (!make_token_map(&mq, a.q, a.B, a.T, a.H, 64, true) ||
        !make_token_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_chunk_map(&mqh, a.qhat, chunks, C, D, C) ||
        !make_chunk_map(&mtat, a.tat, chunks, 2 * C, C, 2 * C) ||
        !make_chunk_map(&ma2t, a.a2t, chunks, 2 * D, C, 128))
        return cudaErrorInvalidValue;
    IntraArgs t;
    t.alpha_log = a.alpha_log;
    t.mu_log = a.mu_log;
    t.beta = a.beta;
    t.eta = a.eta;
    t.qhat = a.qhat;
    t.tat = a.tat;
    t.a2t = a.a2t;
    t.crec = a.crec;
    t.status = a.status;
    t.dbg = a.dbg ? a.dbg + 80512 : nullptr;
    t.dcorr = a.dcorr;
    t.T = a.T;
    t.H = a.H;
    t.NT = a.NT;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunk_intra_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    ProfScope ps(kIntraTc, s);
    chunk_intra_kernel<<<(unsigned)chunks, kThreads, SMEM_BYTES, s>>>(mq, mk, mqh, mtat, ma2t, t);
    return cudaGetLastError();
}

}  // namespace mdn
