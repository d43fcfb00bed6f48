// K-3 on sm_100a: sequential state passing over the chunks, with the
// carried-state and intra-chunk parts of o, on tcgen05 tensor cores fed by TMA.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 4.  With the chunk form
//     Vtilde = U - Y S + Z M,  U = T V,  Y = T Diag(alphabar_{r-1}) P,  Z = T Diag(b_{r-1}) P,
// write X = D1 K S - D2 K M with D1 = Diag(alphabar_r) (= Diag(alphabar_{r-1} alpha_r)) and
// D2 = Diag(alpha_r b_{r-1}); then Vtilde = T (V - X) = T Y with Y = V - X.  The
// carried-state part of o is Oi = Diag(alphabar) Qhat S - Diag(b) Qhat M, the
// reordered intra-chunk part (Qhat K^T o Gamma) Vtilde = (Att T) Y, and the
// chunk-end update S' = alphabar_C S - b_C M + K^T Diag(Gamma_{C,.}) T Y,
// M' = mubar_C M - K^T Diag(eta_i mubar_C / mubar_i) T Y.
//
// One CTA owns one (b, h) and 32 of the d_v = 128 columns (columns of S, M and
// Vtilde are independent) and walks the chunks in order with two warpgroups.
// T and Att come from the intra-chunk kernel.
//
//   operand group (warps 4-7), chunk p, ahead of the chain:
//     Qhat = Q - d K (in place);  [D_G T | -D_w T]
//     P  = [I; Att] T              -> [T; Att T]  (M=128, N=64,  K=64)
//     R  = K^T [D_G T | -D_w T]    -> A2T         (M=128, N=128, K=64)
//   chain group (warps 0-3), chunk n:
//     A1 = [K; Qhat] [S | M]                      (M=128, N=64,  K=128)
//     Y  = V - (D1 KS - D2 KM);   Oi = Diag(alphabar) QhatS - Diag(b) QhatM
//     A2 = [A2T_S; A2T_M] Y   (two M=128, N=32, K=64)
//     S, M <- (alphabar_C S - b_C M, mubar_C M) + A2
//     A3 = [T; Att T] Y (M=128, N=32, K=64):  Vtilde = A3[0:64], o = Oi + A3[64:128]
// The critical path of a chunk is A1 -> Y -> A2 -> state; the stores of chunk
// n-1 run while A1 of chunk n executes.  The fp32 state lives in the chain
// group's registers (thread i owns row i of S and M); its bf16 copy in shared
// memory is the B operand of A1.  Every mbarrier wait is bounded; a wait that
// runs out sets status[1] and the CTA stops.
#include "mdn_internal.cuh"
#include "tc_common.cuh"

namespace mdn {
namespace {

using namespace sm100;
using namespace tc;

constexpr int NS = 32;         // d_v columns per CTA
constexpr int kThreads = 256;  // chain group: threads 0-127, operand group: 128-255
constexpr uint32_t kTmemCols = 512;

// Shared memory map (byte offsets from a 1024-byte aligned base).
constexpr uint32_t KQ0 = 0;                 // [K;Qhat], 2 buffers x 2 panels x (128 rows x 128 B)
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t IATT0 = 2 * KQ_BYTES;    // [I; Att] 128 x 64 bf16 (K-major SW128), 2 buffers
constexpr uint32_t TB0 = IATT0 + 2 * 16384; // T 64 x 64 bf16, rows k (MN-major SW128), 2 buffers
constexpr uint32_t DT = TB0 + 2 * 8192;     // [D_G T | -D_w T], 2 panels of 64 x 64
constexpr uint32_t TAT = DT + 16384;        // [T; Att T] 128 x 64 bf16, K-major SW128
constexpr uint32_t A2T = TAT + 16384;       // [A2T_S | A2T_M], 2 panels of 128 x 64, K-major
constexpr uint32_t ST = A2T + 32768;        // [S | M] bf16, 128 rows x (32 + 32), MN-major SW128
constexpr uint32_t YB = ST + 16384;         // Y 64 x 32 bf16, MN-major SW64
constexpr uint32_t V0 = YB + 4096;          // V slice 64 x 32 bf16 (plain rows), 2 buffers
constexpr uint32_t REC0 = V0 + 8192;        // coefficient records, 2 buffers
constexpr uint32_t VEC0 = REC0 + 2 * kRecBytes;  // abar, d2, b (3 x 64 floats), 2 buffers
constexpr uint32_t SCAL0 = VEC0 + 2 * 768;  // alphabar_C, b_C, mubar_C; 2 buffers of 16 B
constexpr uint32_t BARS = SCAL0 + 32;
constexpr uint32_t MISC = BARS + 128;
constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory map too large");
constexpr int VA = 0, VD2 = 64, VB = 128;

// TMEM columns
constexpr uint32_t TM_P = 0, TM_R = 64, TM_A1 = 192, TM_A2 = 256, TM_A3 = 320;

constexpr uint32_t kTxBytes = KQ_BYTES + 4096 + 8192 + 8192 + kRecBytes;

// mbarriers
constexpr int B_FULL0 = 0, B_QREADY0 = 2, B_OPS_READY = 4, B_OPS_FREE = 5, B_PREP_MMA = 6,
              B_M1 = 7, B_M2 = 8, B_M3 = 9;
// named barriers (id 0 is __syncthreads)
constexpr int NB_CHAIN = 1, NB_OPS = 2;

struct InterArgs {
    const float* rec;
    const float* S0;
    const float* M0;
    float* S_T;
    float* M_T;
    __nv_bfloat16* o;
    __nv_bfloat16* vt;
    unsigned* status;
    float* dbg;  // diagnostics: CTA 0 dumps its first chunk's intermediates and phase clocks
    float dcorr;
    int T, H, NT;
};

// Offsets (floats) of the diagnostic dump.
constexpr int DBG_P = 24576, DBG_R = 32768, DBG_A1 = 49152, DBG_Y = 57344, DBG_A2 = 59392,
              DBG_A3 = 67584, DBG_S = 71680, DBG_M = 75776, DBG_VEC = 79872, DBG_CLK = 80400;

__global__ void __launch_bounds__(kThreads, 1)
chunk_inter_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_t,
                   const __grid_constant__ CUtensorMap tm_att, const InterArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool ops_group = warp >= 4;
    const int g = tid & 127;  // thread index inside its group = its TMEM lane
    const int slice = blockIdx.x % (D / NS);
    const int bh = blockIdx.x / (D / NS);
    const int b = bh / a.H, h = bh % a.H;
    const int j0 = slice * NS;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);

    if (tid == 0) {
        for (int k = 0; k < 10; ++k) mbar_init(&bars[k], 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    float s[NS], m[NS];
    if (ops_group) {
        if (g < C) {  // identity rows 0..63 of both [I; Att] buffers, written once
            for (int c = 0; c < 8; ++c) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = (8 * c + e == g) ? 1.f : 0.f;
                st_bf16x8(sm + IATT0 + sw128_off(g, c), x);
                st_bf16x8(sm + IATT0 + 16384 + sw128_off(g, c), x);
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
            st_bf16x8(sm + ST + sw128_off(g, c), s + 8 * c);
            st_bf16x8(sm + ST + sw128_off(g, 4 + c), m + 8 * c);
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
        uint64_t* fb = &bars[B_FULL0 + buf];
        const uint32_t kq = KQ0 + buf * KQ_BYTES;
        const long long chunk = (long long)bh * a.NT + n;
        mbar_arrive_expect_tx(fb, kTxBytes);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_4d(sm + kq + p * 16384, &tm_k, p * 64, h, n * C, b, fb);
            tma_load_4d(sm + kq + p * 16384 + 8192, &tm_q, p * 64, h, n * C, b, fb);
        }
        tma_load_4d(sm + V0 + buf * 4096, &tm_v, j0, h, n * C, b, fb);
        tma_load_3d(sm + TB0 + buf * 8192, &tm_t, 0, 0, (int)chunk, fb);
        tma_load_3d(sm + IATT0 + buf * 16384 + 8192, &tm_att, 0, 0, (int)chunk, fb);
        bulk_load(sm + REC0 + buf * kRecBytes, a.rec + chunk * kRecFloats, kRecBytes, fb);
    };
    if (tid == 0) {
        if (a.NT > 0) issue_loads(0);
        if (a.NT > 1) issue_loads(1);
    }

    bool ok = true;
    if (ops_group) {
        // ================================================================ operand group
        uint32_t ph = 0;  // parity of the next completion of B_PREP_MMA
        PhaseClock clk;
        clk.start((a.dbg && blockIdx.x == 0 && g == 0) ? a.dbg + DBG_CLK : nullptr);
        for (int p = 0; p < a.NT; ++p) {
            const int buf = p & 1;
            const uint32_t kq = KQ0 + buf * KQ_BYTES;
            const float* rec = reinterpret_cast<const float*>(sm + REC0 + buf * kRecBytes);
            float* vec = reinterpret_cast<float*>(sm + VEC0 + buf * 768);
            float* scal = reinterpret_cast<float*>(sm + SCAL0 + buf * 16);
            const bool dump = a.dbg != nullptr && blockIdx.x == 0 && p == 0;
            ok = named_bar_and(NB_OPS, 128, mbar_wait(&bars[B_FULL0 + buf], (p >> 1) & 1));
            if (!ok) break;
            clk.lap(0);

            // Qhat = Q - d K in place
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int idx = g + 128 * u;
                const int pn = idx >> 9, w = idx & 511, r = w >> 3, c = w & 7;
                const uint4 kw = *reinterpret_cast<const uint4*>(sm + kq + pn * 16384 + sw128_off(r, c));
                uint8_t* qp = sm + kq + pn * 16384 + sw128_off(r + 64, c);
                float kx[8], qx[8];
                unpack_bf16x8(kw, kx);
                unpack_bf16x8(*reinterpret_cast<const uint4*>(qp), qx);
#pragma unroll
                for (int e = 0; e < 8; ++e) qx[e] -= a.dcorr * kx[e];
                st_bf16x8(qp, qx);
            }
            // per-position vectors, and [D_G T | -D_w T] (thread = row, panel)
            {
                const int r = g & 63;
                const float* la = rec;
                const float* lm = rec + C;
                const float* bb = rec + 2 * C;
                if (g < C) {
                    vec[VA + r] = expf(la[r]);
                    vec[VD2 + r] = rec[3 * C + r] * (r > 0 ? bb[r - 1] : 0.f);
                    vec[VB + r] = bb[r];
                    if (r == 0) {
                        scal[0] = expf(la[C - 1]);
                        scal[1] = bb[C - 1];
                        scal[2] = expf(lm[C - 1]);
                    }
                }
                const float w = (g < C) ? rec[6 * C + r] : -rec[5 * C + r] * expf(lm[C - 1] - lm[r]);
                const uint8_t* tb = sm + TB0 + buf * 8192;
                uint8_t* dt = sm + DT + (g < C ? 0 : 8192);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float x[8];
                    unpack_bf16x8(*reinterpret_cast<const uint4*>(tb + sw128_off(r, c)), x);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] *= w;
                    st_bf16x8(dt + sw128_off(r, c), x);
                }
            }
            fence_proxy_async_smem();
            named_bar(NB_OPS, 128);
            if (g == 0) {
                mbar_arrive(&bars[B_QREADY0 + buf]);
                // P = [I; Att] T and R = K^T [D_G T | -D_w T]
                tc_fence_after_sync();
                const uint32_t idp = idesc_bf16(128, 64, false, true);
                const uint32_t idr = idesc_bf16(128, 128, true, true);
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_P,
                             smem_desc(sbase + IATT0 + buf * 16384 + ks * 32, 16, 1024, kSw128),
                             smem_desc(sbase + TB0 + buf * 8192 + ks * 2048, 8192, 1024, kSw128),
                             idp, ks > 0);
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_R, smem_desc(sbase + kq + ks * 2048, 16384, 1024, kSw128),
                             smem_desc(sbase + DT + ks * 2048, 8192, 1024, kSw128), idr, ks > 0);
                mma_commit(&bars[B_PREP_MMA]);
            }
            clk.lap(1);
            ok = mbar_wait(&bars[B_PREP_MMA], ph);
            ph ^= 1u;
            tc_fence_after_sync();
            clk.lap(2);
            // the chain must be done reading [T; Att T] and A2T of the previous chunk
            if (p > 0) ok = ok && mbar_wait(&bars[B_OPS_FREE], (p - 1) & 1);
            ok = named_bar_and(NB_OPS, 128, ok);
            if (!ok) break;
            clk.lap(3);

            // [T; Att T] and A2T to bf16 operands (thread = TMEM lane = operand row)
            {
                float v[64];
                tmem_ld32(tmem + lane_sel + TM_P, *reinterpret_cast<float(*)[32]>(v));
                tmem_ld32(tmem + lane_sel + TM_P + 32, *reinterpret_cast<float(*)[32]>(v + 32));
                tmem_wait_ld();
                if (dump)
                    for (int j = 0; j < 64; ++j) a.dbg[DBG_P + g * 64 + j] = v[j];
#pragma unroll
                for (int c = 0; c < 8; ++c) st_bf16x8(sm + TAT + sw128_off(g, c), v + 8 * c);
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    tmem_ld32(tmem + lane_sel + TM_R + 64 * q2, *reinterpret_cast<float(*)[32]>(v));
                    tmem_ld32(tmem + lane_sel + TM_R + 64 * q2 + 32,
                              *reinterpret_cast<float(*)[32]>(v + 32));
                    tmem_wait_ld();
                    if (dump)
                        for (int j = 0; j < 64; ++j) a.dbg[DBG_R + g * 128 + 64 * q2 + j] = v[j];
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        st_bf16x8(sm + A2T + q2 * 16384 + sw128_off(g, c), v + 8 * c);
                }
            }
            if (dump && g < C) {
                for (int k = 0; k < 3; ++k) a.dbg[DBG_VEC + k * 64 + g] = vec[k * 64 + g];
                if (g < 3) a.dbg[DBG_VEC + 384 + g] = scal[g];
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar(NB_OPS, 128);
            if (g == 0) mbar_arrive(&bars[B_OPS_READY]);
            clk.lap(4);
        }
    } else {
        // ================================================================ chain group
        const int r = g & 63;
        PhaseClock clk;
        clk.start((a.dbg && blockIdx.x == 0 && g == 0) ? a.dbg + DBG_CLK + 16 : nullptr);
        float oi[NS];
        // Vtilde and o of chunk n (its A3 product has been issued)
        auto store_outputs = [&](int n) -> bool {
            if (!mbar_wait(&bars[B_M3], n & 1)) return false;
            tc_fence_after_sync();
            float o3[32];
            tmem_ld32(tmem + lane_sel + TM_A3, o3);
            tmem_wait_ld();
            if (a.dbg != nullptr && blockIdx.x == 0 && n == 0)
                for (int j = 0; j < 32; ++j) a.dbg[DBG_A3 + g * 32 + j] = o3[j];
            const int t = n * C + r;
            if (t < a.T) {
                __nv_bfloat16* dst = (g < C ? a.vt : a.o) + (((size_t)b * a.T + t) * a.H + h) * D + j0;
                uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        w[e] = (g < C) ? o3[8 * c + e] : o3[8 * c + e] + oi[8 * c + e];
                    d4[c] = bf16x8(w);
                }
            }
            return true;
        };

        for (int n = 0; n < a.NT; ++n) {
            const int buf = n & 1;
            const uint32_t kq = KQ0 + buf * KQ_BYTES;
            const float* vec = reinterpret_cast<const float*>(sm + VEC0 + buf * 768);
            const float* scal = reinterpret_cast<const float*>(sm + SCAL0 + buf * 16);
            const bool dump = a.dbg != nullptr && blockIdx.x == 0 && n == 0;
            ok = named_bar_and(NB_CHAIN, 128, mbar_wait(&bars[B_QREADY0 + buf], (n >> 1) & 1));
            if (!ok) break;
            clk.lap(0);
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
                mma_commit(&bars[B_M1]);
            }
            // outputs of the previous chunk while A1 runs; then the operand
            // group may overwrite [T; Att T] and A2T
            if (n > 0) {
                ok = store_outputs(n - 1);
                if (g == 0 && ok) mbar_arrive(&bars[B_OPS_FREE]);
            }
            ok = mbar_wait(&bars[B_M1], n & 1) && ok;
            tc_fence_after_sync();
            ok = named_bar_and(NB_CHAIN, 128, ok);
            if (!ok) break;
            clk.lap(1);

            // Y = V - X (rows 0..63); Oi kept in registers (rows 64..127)
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
                    const uint4* vrow = reinterpret_cast<const uint4*>(sm + V0 + buf * 4096 + r * 64);
                    float yy[NS];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float vv[8];
                        unpack_bf16x8(vrow[c], vv);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = 8 * c + e;
                            yy[j] = vv[e] - (c_ab * x[j] - c_d2 * y[j]);
                        }
                    }
                    if (dump)
                        for (int j = 0; j < NS; ++j) a.dbg[DBG_Y + r * NS + j] = yy[j];
#pragma unroll
                    for (int c = 0; c < 4; ++c) st_bf16x8(sm + YB + sw64_off(r, c), yy + 8 * c);
                } else {
#pragma unroll
                    for (int j = 0; j < NS; ++j) oi[j] = c_ab * x[j] - c_b * y[j];
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            ok = named_bar_and(NB_CHAIN, 128, mbar_wait(&bars[B_OPS_READY], n & 1));
            if (!ok) break;
            clk.lap(2);

            if (g == 0) {
                // K, Q, V, T, Att and the record of this buffer are no longer needed
                if (n + 2 < a.NT) issue_loads(n + 2);
                tc_fence_after_sync();
                const uint32_t id = idesc_bf16(128, 32, false, true);
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t yd = smem_desc(sbase + YB + ks * 1024, 4096, 512, kSw64);
                    mma_bf16(tmem + TM_A2, smem_desc(sbase + A2T + ks * 32, 16, 1024, kSw128), yd,
                             id, ks > 0);
                    mma_bf16(tmem + TM_A2 + 32,
                             smem_desc(sbase + A2T + 16384 + ks * 32, 16, 1024, kSw128), yd, id,
                             ks > 0);
                }
                mma_commit(&bars[B_M2]);
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t yd = smem_desc(sbase + YB + ks * 1024, 4096, 512, kSw64);
                    mma_bf16(tmem + TM_A3, smem_desc(sbase + TAT + ks * 32, 16, 1024, kSw128), yd,
                             id, ks > 0);
                }
                mma_commit(&bars[B_M3]);
            }
            ok = mbar_wait(&bars[B_M2], n & 1);
            tc_fence_after_sync();
            ok = named_bar_and(NB_CHAIN, 128, ok);
            if (!ok) break;
            clk.lap(3);

            // state update
            {
                float dS[32], dM[32];
                tmem_ld32(tmem + lane_sel + TM_A2, dS);
                tmem_ld32(tmem + lane_sel + TM_A2 + 32, dM);
                tmem_wait_ld();
                if (dump)
                    for (int j = 0; j < 32; ++j) {
                        a.dbg[DBG_A2 + g * 64 + j] = dS[j];
                        a.dbg[DBG_A2 + g * 64 + 32 + j] = dM[j];
                    }
#pragma unroll
                for (int j = 0; j < NS; ++j) {
                    const float sn = fmaf(abC, s[j], fmaf(-bC, m[j], dS[j]));
                    m[j] = fmaf(mbC, m[j], dM[j]);
                    s[j] = sn;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    st_bf16x8(sm + ST + sw128_off(g, c), s + 8 * c);
                    st_bf16x8(sm + ST + sw128_off(g, 4 + c), m + 8 * c);
                }
                if (dump)
                    for (int j = 0; j < NS; ++j) {
                        a.dbg[DBG_S + g * NS + j] = s[j];
                        a.dbg[DBG_M + g * NS + j] = m[j];
                    }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_bar(NB_CHAIN, 128);
            clk.lap(4);
        }
        if (ok && a.NT > 0) ok = store_outputs(a.NT - 1);
        ok = named_bar_and(NB_CHAIN, 128, ok);
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

}  // namespace

cudaError_t launch_chunk_inter_tc(const ChunkArgs& a, cudaStream_t s)
{
    CUtensorMap mq, mk, mv, mt, matt;
    const long long chunks = (long long)a.B * a.H * a.NT;
    if (!make_token_map(&mq, a.q, a.B, a.T, a.H, 64, true) ||
        !make_token_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_token_map(&mv, a.v, a.B, a.T, a.H, NS, false) || !make_mat_map(&mt, a.tmat, chunks) ||
        !make_mat_map(&matt, a.att, chunks))
        return cudaErrorInvalidValue;
    InterArgs t;
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
    t.T = a.T;
    t.H = a.H;
    t.NT = a.NT;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunk_inter_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const long long blocks = (long long)a.B * a.H * (D / NS);
    ProfScope ps(kInterTc, s);
    chunk_inter_kernel<<<(unsigned)blocks, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, mt, matt, t);
    return cudaGetLastError();
}

// The tensor-core path: coefficients, then the intra-chunk kernel, then the
// sequential inter-chunk kernel, all on stream s.
cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t s)
{
    if (a.D != D) return cudaErrorNotSupported;
    cudaError_t e = launch_gate_pack(a.alpha_log, a.mu_log, a.beta, a.eta, a.B, a.T, a.H, a.rec, s);
    if (e != cudaSuccess) return e;
    if ((e = launch_chunk_intra_tc(a, s)) != cudaSuccess) return e;
    return launch_chunk_inter_tc(a, s);
}

}  // namespace mdn
