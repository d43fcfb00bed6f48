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
// One CTA owns one (b, h) and NS (32 or 64) of the d_v = 128 columns (columns
// of S, M and Vtilde are independent) and walks the chunks in order.  The
// intra-chunk kernel has prepared Qhat, [T; Att T] and A2T = [K^T Diag(Gamma_C) T;
// -K^T Diag(w) T] for every chunk.  Per chunk n:
//     A1 = [K; Qhat] [S | M]                      (M=128, N=2 NS, K=128)
//     Y  = V - (D1 KS - D2 KM)
//     A2 = [A2T_S; A2T_M] Y   (two M=128, N=NS, K=64)
//     S, M <- (alphabar_C S - b_C M, mubar_C M) + A2
//     A3 = [T; Att T] Y  (M=128, N=NS, K=64):
//     Vtilde = A3[0:64],  o = Diag(alphabar) QhatS - Diag(b) QhatM + A3[64:128]
// A tcgen05.mma of N <= 128 costs about the same whatever N is, so a wider
// slice does more work per instruction; NS = 64 halves the CTAs per head
// and the operand traffic for the same chain length.
// Only A1 -> Y -> A2 -> state is sequential; the warps are specialised so
// that nothing else sits on that chain:
//   warp 0      one lane issues every tcgen05.mma and commit
//   warp 1      one lane issues every TMA load, up to two chunks ahead
//   16 chain warps: warp w owns TMEM lanes 32(w%4).. and NH columns (8 at
//               NS = 32, 16 at NS = 64: the epilogues on the chain are short
//               per thread); it holds those columns of one row of S and M in fp32 registers
//               for the whole sequence (their bf16 copy in shared memory is
//               the B operand of A1); the warps on lanes 0..63 also form Y
//   4 output warps: Vtilde and o of chunk n from A3 and A1, written to
//               global memory while the chain runs on
// Hand-offs are mbarriers only (no CTA-wide barrier inside the loop).  TMEM
// holds A1 and A3 twice (chunk parity) so the outputs of chunk n can be read
// while chunk n+1 computes.  Every wait is bounded; a wait that runs out
// raises the CTA's abort flag, every role leaves its loop, in-flight copies
// and MMAs are drained, and status[1] is set.
#include <algorithm>

#include "inter_common.cuh"

namespace mdn {
namespace {

using namespace sm100;
using namespace tc;
using namespace inter;

constexpr int kChainWarp0 = 2;   // warps 0, 1: MMA issue, loads

// Per-width layout.  NS = d_v columns per CTA (32 or 64).
template <int NS>
struct Cfg {
    static constexpr int NH = NS == 32 ? 8 : 16;      // columns per chain thread
    static constexpr int CW = 4 * (NS / NH);          // chain warps: 4 lane quadrants x NS/NH column groups
    static constexpr int kOutWarp0 = kChainWarp0 + CW;
    static constexpr int kThreads = (kOutWarp0 + 4) * 32;
    // one CTA per SM; registers are granted to warps in groups of four
    static constexpr int kMaxRegs = (65536 / (((kThreads / 32 + 3) / 4) * 128)) & ~7;
    static constexpr int NVC = NS == 32 ? 4 : 2;      // V / coefficient slots
    static constexpr uint32_t kTmemCols = NS == 32 ? 256 : 512;
    // shared memory (byte offsets from a 1024-byte aligned base)
    static constexpr uint32_t KQ0 = 0;                // [K; Qhat], 2 slots x 2 panels x (128 rows x 128 B)
    static constexpr uint32_t FB0 = 2 * 32768;        // [T; Att T] (16 KB), [A2T_S | A2T_M] (2 x 16 KB), 2 slots
    static constexpr uint32_t FB_BYTES = 49152;
    static constexpr uint32_t ST = FB0 + 2 * FB_BYTES;  // [S | M] bf16, 128 rows, MN-major 128-byte swizzle
    static constexpr uint32_t ST_BYTES = 128 * 2 * NS * 2;
    static constexpr uint32_t YB = ST + ST_BYTES;      // Y 64 rows x NS bf16, MN-major (64 / 128-byte swizzle)
    static constexpr uint32_t YB_BYTES = 64 * NS * 2;
    static constexpr uint32_t V0 = YB + YB_BYTES;      // V slice 64 rows x NS bf16 (plain rows), NVC slots
    static constexpr uint32_t V_BYTES = 64 * NS * 2;
    static constexpr uint32_t CR0 = V0 + NVC * V_BYTES;  // chunk coefficients (256 floats), NVC slots
    static constexpr uint32_t BARS = CR0 + NVC * 1024;
    static constexpr uint32_t MISC = BARS + 256;
    static constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;  // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory map too large");
    static_assert(ST % 1024 == 0 && YB % 1024 == 0 && V0 % 16 == 0, "operand alignment");
    // TMEM columns: A1 (KS | KM, QhatS | QhatM) in two slots, A2 (dS | dM), A3 in two slots
    static constexpr uint32_t TM_A1 = 0, TM_A2 = 4 * NS, TM_A3 = 6 * NS;
    static constexpr uint32_t kTxVC = V_BYTES + 1024;
    // byte offset of 16-byte chunk c (8 columns) of row i of S, resp. M, in ST
    __device__ static __forceinline__ uint32_t s_off(int i, int c) { return sw128_off(i, c); }
    __device__ static __forceinline__ uint32_t m_off(int i, int c) {
        return NS == 32 ? sw128_off(i, 4 + c) : 16384 + sw128_off(i, c);
    }
    // byte offset of chunk c of row r of Y in YB
    __device__ static __forceinline__ uint32_t y_off(int r, int c) {
        return NS == 32 ? sw64_off(r, c) : sw128_off(r, c);
    }
};

constexpr uint32_t kTxKQ = 32768;   // K, Qhat
constexpr uint32_t kTxFB = 49152;   // [T; Att T], A2T

// mbarriers (index into the array at BARS)
constexpr int B_FKQ = 0;   // [2] K, Qhat landed
constexpr int B_FFB = 2;   // [2] [T; Att T], A2T landed
constexpr int B_FVC = 4;   // [4] V, coefficients landed
constexpr int B_EVC = 8;   // [4] V, coefficients slot released (chain + output warps)
constexpr int B_M1 = 12;   // [2] A1 complete
constexpr int B_M2 = 14;   //     A2 complete
constexpr int B_M3 = 15;   // [2] A3 complete (and every earlier MMA)
constexpr int B_YR = 17;   //     Y written (the chain warps on lanes 0..63)
constexpr int B_SR = 18;   //     next state written (every chain warp)
constexpr int B_OD = 19;   // [2] A1 / A3 slot read by the output warps (4 warps)
constexpr int B_FIN = 21;  //     every MMA complete (exit)
constexpr int kBars = 22;

// N (8 or 16) consecutive columns of this thread's TMEM lane.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* v) {
    if constexpr (N == 16) tmem_ld16(taddr, v);
    else tmem_ld8(taddr, v);
}

template <int NS>
__global__ void __launch_bounds__(Cfg<NS>::kThreads) __maxnreg__(Cfg<NS>::kMaxRegs)
chunk_inter_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_qh,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_tat,
                   const __grid_constant__ CUtensorMap tm_a2t, const InterArgs a)
{
    using L = Cfg<NS>;
    constexpr int CW = L::CW;
    constexpr int NH = L::NH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lid = tid & 31;
    const int quad = warp & 3;                   // TMEM lane quadrant this warp may access
    const int lane = (quad << 5) | lid;          // TMEM lane = operand row
    const int slice = blockIdx.x % (D / NS);
    const Chain ch = chain_of(a, blockIdx.x / (D / NS));
    const int b = ch.b, h = ch.h;
    const int j0 = slice * NS;
    const int NT = ch.nt;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 4);

    if (tid == 0) {
        for (int k = 0; k < kBars; ++k) {
            uint32_t count = 1;  // TMA (expect_tx) and tcgen05.commit barriers
            if (k >= B_EVC && k < B_EVC + 4) count = CW + 4;
            if (k == B_YR) count = CW / 2;
            if (k == B_OD || k == B_OD + 1) count = 4;
            if (k == B_SR) count = CW;
            mbar_init(&bars[k], count);
        }
        mbar_fence_init();
        *abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    // chain warps: the entering state, row `lane`, columns j0 + NH hc ..
    const bool chain = warp >= kChainWarp0 && warp < L::kOutWarp0;
    const int hc = (warp - kChainWarp0) >> 2;  // column group of a chain warp
    float s[NH], m[NH];
    if (chain) {
        const size_t row = ((size_t)ch.sh * D + lane) * D + j0 + NH * hc;
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            s[j] = a.S0 ? a.S0[row + j] : 0.f;
            m[j] = a.M0 ? a.M0[row + j] : 0.f;
        }
#pragma unroll
        for (int c = 0; c < NH / 8; ++c) {
            st_bf16x8(sm + L::ST + L::s_off(lane, hc * (NH / 8) + c), s + 8 * c);
            st_bf16x8(sm + L::ST + L::m_off(lane, hc * (NH / 8) + c), m + 8 * c);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quad * 32) << 16);  // this warp's lane base
#ifdef MDN_PHASE_CLOCKS
    const uint64_t t_start = global_timer_ns();
#endif

    if (warp == 0) {
        // ------------------------------------------------------------ MMA issue
        if (lid == 0) {
            PhaseClock clk;
            clk.start((a.dbg && blockIdx.x == 0) ? a.dbg : nullptr);
            const uint64_t d_kq0 = smem_desc(sbase + L::KQ0, 16, 1024, kSw128);
            // B of A1: [S | M], N = 2 NS; for NS = 64 the S and M halves are two 128-byte panels
            const uint64_t d_st = smem_desc(sbase + L::ST, NS == 32 ? 8192 : 16384, 1024, kSw128);
            const uint64_t d_fb0 = smem_desc(sbase + L::FB0, 16, 1024, kSw128);
            const uint64_t d_y = NS == 32 ? smem_desc(sbase + L::YB, 4096, 512, kSw64)
                                          : smem_desc(sbase + L::YB, 8192, 1024, kSw128);
            constexpr uint32_t ystep = (16 * NS * 2) >> 4;  // 16 rows of Y
            constexpr uint32_t id1 = idesc_bf16(128, 2 * NS, false, true);
            constexpr uint32_t id2 = idesc_bf16(128, NS, false, true);
            // K, Qhat of chunk n and the A1 / A3 slot of chunk n are waited for
            // while chunk n - 1 waits for its Y, so that only the state hand-off
            // separates the last product of one chunk from the first of the next.
            bool ready = NT > 0 && wait_bar(&bars[B_FKQ], 0, abort_flag);
            for (int n = 0; n < NT && ready; ++n) {
                const int s2 = n & 1;
                clk.lap(0);
                if (n >= 1 && !wait_bar(&bars[B_SR], (n - 1) & 1, abort_flag)) break;
                clk.lap(1);
                tc_fence_after_sync();
                const uint64_t dkq = d_kq0 + s2 * (32768 >> 4);
                const uint32_t a1 = tmem + L::TM_A1 + 2 * NS * s2;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(a1, dkq + (((ks >> 2) * 16384 + (ks & 3) * 32) >> 4),
                             d_st + ks * (2048 >> 4), id1, ks > 0);
                mma_commit(&bars[B_M1 + s2]);
                clk.lap(2);
                if (!wait_bar(&bars[B_FFB + s2], (n >> 1) & 1, abort_flag)) break;
                if (n + 1 < NT) {
                    const int t2 = (n + 1) & 1;
                    if (!wait_bar(&bars[B_FKQ + t2], ((n + 1) >> 1) & 1, abort_flag)) break;
                    if (n >= 1 && !wait_bar(&bars[B_OD + t2], ((n - 1) >> 1) & 1, abort_flag)) break;
                }
                clk.lap(3);
                if (!wait_bar(&bars[B_YR], n & 1, abort_flag)) break;
                clk.lap(4);
                tc_fence_after_sync();
                const uint64_t dfb = d_fb0 + s2 * (L::FB_BYTES >> 4);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t yd = d_y + ks * ystep;
                    mma_bf16(tmem + L::TM_A2, dfb + (16384 >> 4) + ks * 2, yd, id2, ks > 0);
                    mma_bf16(tmem + L::TM_A2 + NS, dfb + (32768 >> 4) + ks * 2, yd, id2, ks > 0);
                }
                mma_commit(&bars[B_M2]);
                clk.lap(5);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + L::TM_A3 + NS * s2, dfb + ks * 2, d_y + ks * ystep, id2, ks > 0);
                mma_commit(&bars[B_M3 + s2]);
                clk.lap(6);
            }
            clk.flush();
            // every issued MMA has completed before TMEM and shared memory are released
            mma_commit(&bars[B_FIN]);
            (void)mbar_wait(&bars[B_FIN], 0);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ TMA loads
        if (lid == 0) {
            PhaseClock clk;
            clk.start((a.dbg && blockIdx.x == 0) ? a.dbg + 20 : nullptr);
            int issued_kq = 0, issued_fb = 0, issued_vc = 0;
            for (int n = 0; n < NT; ++n) {
                const int s2 = n & 1, sv = n % L::NVC;
                const long long chunk = ch.chunk0 + n;
                if (n >= 2 && !wait_bar(&bars[B_M1 + s2], ((n - 2) >> 1) & 1, abort_flag)) break;
                // the operands of chunk n are in global memory
                if (!wait_ready(a.ready + chunk, abort_flag)) break;
                fence_proxy_async_global();
                clk.lap(0);
                uint64_t* fb = &bars[B_FKQ + s2];
                mbar_arrive_expect_tx(fb, kTxKQ);
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    uint8_t* dst = sm + L::KQ0 + s2 * 32768 + p * 16384;
                    tma_load_4d(dst, &tm_k, p * 64, h, (ch.n0 + n) * C, b, fb);
                    tma_load_3d(dst + 8192, &tm_qh, p * 64, 0, (int)chunk, fb);
                }
                issued_kq = n + 1;
                if (n >= 2 && !wait_bar(&bars[B_M3 + s2], ((n - 2) >> 1) & 1, abort_flag)) break;
                clk.lap(1);
                fb = &bars[B_FFB + s2];
                mbar_arrive_expect_tx(fb, kTxFB);
                uint8_t* dst = sm + L::FB0 + s2 * L::FB_BYTES;
                tma_load_3d(dst, &tm_tat, 0, 0, (int)chunk, fb);
                tma_load_3d(dst + 16384, &tm_a2t, 0, 0, (int)chunk, fb);
                tma_load_3d(dst + 32768, &tm_a2t, 0, 128, (int)chunk, fb);
                issued_fb = n + 1;
                if (n >= L::NVC &&
                    !wait_bar(&bars[B_EVC + sv], ((n / L::NVC) - 1) & 1, abort_flag))
                    break;
                clk.lap(2);
                fb = &bars[B_FVC + sv];
                mbar_arrive_expect_tx(fb, L::kTxVC);
                tma_load_4d(sm + L::V0 + sv * L::V_BYTES, &tm_v, j0, h, (ch.n0 + n) * C, b, fb);
                bulk_load(sm + L::CR0 + sv * 1024, a.crec + chunk * 256, 1024, fb);
                issued_vc = n + 1;
            }
            clk.flush();
            // Copies that were issued must land before shared memory is
            // released (after an abort some were never consumed).  A phase
            // that has completed passes at once.
            for (int n = issued_kq - 2; n < issued_kq; ++n)
                if (n >= 0) (void)mbar_wait(&bars[B_FKQ + (n & 1)], (n >> 1) & 1);
            for (int n = issued_fb - 2; n < issued_fb; ++n)
                if (n >= 0) (void)mbar_wait(&bars[B_FFB + (n & 1)], (n >> 1) & 1);
            for (int n = issued_vc - L::NVC; n < issued_vc; ++n)
                if (n >= 0) (void)mbar_wait(&bars[B_FVC + n % L::NVC], (n / L::NVC) & 1);
        }
        __syncwarp();
    } else if (chain) {
        // ------------------------------------------------------------ chain epilogues
        const bool ypart = quad < 2;  // lanes 0..63: rows of K, so this warp forms Y
        const int r = lane & 63;
        PhaseClock clk;
        clk.start((a.dbg && blockIdx.x == 0 && warp == kChainWarp0 + 2 && lid == 0) ? a.dbg + 40 : nullptr);
        for (int n = 0; n < NT; ++n) {
            const int s2 = n & 1, sv = n % L::NVC;
            if (!warp_wait(&bars[B_FVC + sv], (n / L::NVC) & 1, abort_flag)) break;
            clk.lap(0);
            const float* cr = reinterpret_cast<const float*>(sm + L::CR0 + sv * 1024);
            const float abC = cr[3 * C], bC = cr[3 * C + 1], mbC = cr[3 * C + 2];
            if (ypart) {
                const float c_ab = cr[r], c_d2 = cr[C + r];
                const uint4* vrow =
                    reinterpret_cast<const uint4*>(sm + L::V0 + sv * L::V_BYTES + r * (NS * 2)) + hc * (NH / 8);
                if (!warp_wait(&bars[B_M1 + s2], (n >> 1) & 1, abort_flag)) break;
                clk.lap(1);
                tc_fence_after_sync();
                const uint32_t a1 = tq + L::TM_A1 + 2 * NS * s2 + NH * hc;
                float x[NH], y[NH];
                tmem_ld_cols<NH>(a1, x);
                tmem_ld_cols<NH>(a1 + NS, y);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < NH / 8; ++c) {
                    float vv[8];
                    unpack_bf16x8(vrow[c], vv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) vv[e] -= fmaf(c_ab, x[8 * c + e], -c_d2 * y[8 * c + e]);
                    st_bf16x8(sm + L::YB + L::y_off(r, hc * (NH / 8) + c), vv);
                }
                clk.lap(2);
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lid == 0) {
                    mbar_arrive(&bars[B_YR]);
                    mbar_arrive(&bars[B_EVC + sv]);
                }
                clk.lap(3);
            } else {
                __syncwarp();
                if (lid == 0) mbar_arrive(&bars[B_EVC + sv]);
            }
            if (!warp_wait(&bars[B_M2], n & 1, abort_flag)) break;
            clk.lap(4);
            tc_fence_after_sync();
            {
                float dS[NH], dM[NH];
                tmem_ld_cols<NH>(tq + L::TM_A2 + NH * hc, dS);
                tmem_ld_cols<NH>(tq + L::TM_A2 + NS + NH * hc, dM);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < NH; ++j) {
                    const float sn = fmaf(abC, s[j], fmaf(-bC, m[j], dS[j]));
                    m[j] = fmaf(mbC, m[j], dM[j]);
                    s[j] = sn;
                }
            }
#pragma unroll
            for (int c = 0; c < NH / 8; ++c) {
                st_bf16x8(sm + L::ST + L::s_off(lane, hc * (NH / 8) + c), s + 8 * c);
                st_bf16x8(sm + L::ST + L::m_off(lane, hc * (NH / 8) + c), m + 8 * c);
            }
            clk.lap(5);
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lid == 0) mbar_arrive(&bars[B_SR]);
            clk.lap(6);
        }
        clk.flush();
    } else {
        // ------------------------------------------------------------ outputs
        const bool orow = quad >= 2;  // lanes 64..127: rows of o; lanes 0..63: rows of Vtilde
        const int r = lane & 63;
        __nv_bfloat16* const out = orow ? a.o : a.vt;
        for (int n = 0; n < NT; ++n) {
            const int s2 = n & 1, sv = n % L::NVC;
            if (!warp_wait(&bars[B_FVC + sv], (n / L::NVC) & 1, abort_flag)) break;
            const float* cr = reinterpret_cast<const float*>(sm + L::CR0 + sv * 1024);
            const float c_ab = cr[r], c_b = cr[2 * C + r];
            __syncwarp();
            if (lid == 0) mbar_arrive(&bars[B_EVC + sv]);
            if (!warp_wait(&bars[B_M3 + s2], (n >> 1) & 1, abort_flag)) break;
            tc_fence_after_sync();
            const int t = n * C + r;  // token of the chain
            uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)(ch.out0 + t) * a.H + h) * D + j0);
#pragma unroll 1
            for (int q16 = 0; q16 < NS / 16; ++q16) {
                float x[16], y[16];
                if (orow) {
                    tmem_ld16(tq + L::TM_A1 + 2 * NS * s2 + 16 * q16, x);       // Qhat S
                    tmem_ld16(tq + L::TM_A1 + 2 * NS * s2 + NS + 16 * q16, y);  // Qhat M
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) x[j] = fmaf(c_ab, x[j], -c_b * y[j]);
                    tmem_ld16(tq + L::TM_A3 + NS * s2 + 16 * q16, y);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) x[j] += y[j];
                } else {
                    tmem_ld16(tq + L::TM_A3 + NS * s2 + 16 * q16, x);
                    tmem_wait_ld();
                }
                if (t < ch.len) {
                    dst[2 * q16] = bf16x8(x);
                    dst[2 * q16 + 1] = bf16x8(x + 8);
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lid == 0) mbar_arrive(&bars[B_OD + s2]);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    const bool ok = *abort_flag == 0;
    if (chain && ok) {
        const size_t row = ((size_t)ch.sh * D + lane) * D + j0 + NH * hc;
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            a.S_T[row + j] = s[j];
            a.M_T[row + j] = m[j];
        }
    }
    if (!ok && tid == 0) atomicOr(a.status + 1, 1u);
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, L::kTmemCols);
    }
#ifdef MDN_PHASE_CLOCKS
    if (a.dbg && tid == 0 && blockIdx.x < 1024) {
        double* tl = reinterpret_cast<double*>(a.dbg + 30000);
        tl[2 * blockIdx.x] = (double)t_start;
        tl[2 * blockIdx.x + 1] = (double)global_timer_ns();
    }
#endif
}

template <int NS>
cudaError_t launch_inter(const ChunkArgs& a, cudaStream_t s)
{
    using L = Cfg<NS>;
    CUtensorMap mk, mqh, mv, mtat, ma2t;
    const long long chunks = (long long)a.B * a.H * a.NT;
    if (!make_token_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_chunk_map(&mqh, a.qhat, chunks, C, D, C) ||
        !make_token_map(&mv, a.v, a.B, a.T, a.H, NS, false) ||
        !make_chunk_map(&mtat, a.tat, chunks, 2 * C, C, 2 * C) ||
        !make_chunk_map(&ma2t, a.a2t, chunks, 2 * D, C, 128))
        return cudaErrorInvalidValue;
    const InterArgs t = inter_args(a);
    cudaError_t e = cudaFuncSetAttribute(chunk_inter_kernel<NS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const long long chains = a.cu_chunks ? (long long)a.nseq * a.H : (long long)a.B * a.H;
    const long long blocks = chains * (D / NS);
    ProfScope ps(kInterTc, s);
    // Programmatic dependent launch: the CTAs may start while the intra-chunk
    // kernel (launched just before on s) still runs; each chunk is read only
    // after its ready flag.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(L::kThreads);
    cfg.dynamicSmemBytes = L::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, chunk_inter_kernel<NS>, mk, mqh, mv, mtat, ma2t, t);
}

}  // namespace

// The tensor-core path: the intra-chunk kernel, then the sequential
// inter-chunk kernel as its programmatic dependent, both on stream s.
//
// Reserved SMs for the chains, and the chunk limit of the intra-chunk CTAs
// on them.  The inter-chunk kernel's CTAs can only start on SMs that the
// intra-chunk kernel (two CTAs per SM) has left, and each chain then takes
// one chunk of its head per step.  With the intra-chunk CTAs on the chains'
// SMs limited to L chunks, the chains start after about L chunk times while
// the CTAs on the other SMs (U of them) produce the remaining chunks, which
// the chunk-major order makes the last ones the chains need.  An
// intra-chunk chunk costs about r chain steps (two CTAs per SM, ~17k cycles;
// a 32-column chain step ~3.3k, a 64-column one ~4.6k), so L minimises
//     L r + max(NT, rest / U r + 1),   rest = chunks - 2 SMs L.
// For whole-head chains (~9k cycles a step) r = 6 is not that ratio but the
// value that measured best on the 1.3B-layer workload: both kernels are then
// bound by SM time, not by the chain, and the plan keeps the intra-chunk
// kernel on every SM until nearly all chunks are done.
struct Reserve {
    int sms = 0;    // CTAs on SMs 0 .. sms-1 are limited
    int limit = 1;
};
static Reserve plan_reserve(long long chunks, long long ctas, int sms, int nt, int ns)
{
    Reserve rv;
    if (ctas > sms) return rv;
    const double r = ns == 32 ? 5.0 : ns == 64 ? 3.7 : 6.0;
    const long long U = 2LL * (sms - ctas), per_round = 2LL * sms;
    const int lmax = (int)((chunks + per_round - 1) / per_round);
    double best = 0.0;
    for (int L = 1; L <= lmax; ++L) {
        const long long rest = chunks - per_round * L;
        if (rest > 0 && U == 0) continue;
        const double t = L * r + std::max((double)nt, rest > 0 ? (double)rest / U * r + 1.0 : 0.0);
        if (rv.sms == 0 || t < best) {
            best = t;
            rv.sms = (int)ctas;
            rv.limit = L;
        }
    }
    return rv;
}

// Chain width (ns = 0 chooses).  A chain step costs about 3.1k cycles with
// 32-column slices, 4.8k with 64 and 9k with the whole head: the epilogues of
// one CTA move data in proportion to its width, and that, not the tensor
// pipe, bounds the step.  So four 32-column slices per head when they all fit
// on the SMs at once (the shortest chain); otherwise one CTA per head, which
// takes the least SM time per chunk (9k against 4 x 3.1k or 2 x 4.8k) and
// leaves the fewest waves.  Packed sequences keep 32 up to four waves, else
// 64 (their chains end at different times), and reserve SMs (one chunk
// each) for the chains of the longest sequence, which start first.
cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t s, int ns)
{
    if (a.D != D) return cudaErrorNotSupported;
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long heads = a.cu_chunks ? (long long)a.nseq * a.H : (long long)a.B * a.H;
    const long long room = sms - sms / 4;  // SMs the chain may take beside the intra kernel
    if (ns == 0) {
        // packed sequences: the chains are ordered longest first, and the
        // longest one is the critical path; 32-column slices (the shortest
        // step) while the slices fit in four waves, else 64
        if (a.cu_chunks) ns = heads * 4 <= 4LL * sms ? 32 : 64;
        else ns = heads * 4 <= sms ? 32 : 128;
    }
    const long long ctas = heads * (D / ns);
    Reserve rv;
    if (a.cu_chunks) {
        // SMs from the start for the chains of the longest sequence (the
        // first H slices' worth of CTAs); the intra-chunk kernel keeps the
        // rest, so that it produces that sequence's chunks faster than its
        // chains take them; the other chains follow as SMs free up
        const long long first = (long long)a.H * (D / ns);
        long long want = first < ctas ? first : ctas;
        if (want > room) want = room;
        rv.sms = (int)want;
    } else {
        rv = plan_reserve(heads * a.NT, ctas, sms, a.NT, ns);
    }
    if (!a.test_no_intra && (e = launch_chunk_intra_tc(a, s, rv.sms, rv.limit)) != cudaSuccess)
        return e;
    if (ns == 128) return launch_inter_head(a, s);
    return ns == 64 ? launch_inter<64>(a, s) : launch_inter<32>(a, s);
}

}  // namespace mdn
