// The reverse chain of the backward pass on tcgen05 (bf16 inputs, d = 128):
// the adjoints (dS, dM) of the states walked back over the chunks.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 7 (training keeps Vtilde; the backward pass
// runs from it).  Per chunk, from the adjoints of the states leaving it:
//     dVtilde = Att^T dO + Diag(Gamma_C) K dS - Diag(w) K dM
//     dY      = T^T dVtilde                                       (= dv)
//     dS     <- alphabar_C dS + E - K^T Diag(alphabar) dY
//     dM     <- -b_C dS + mubar_C dM - F + K^T Diag(D2) dY
// with E = Qhat^T Diag(alphabar) dO, F = Qhat^T Diag(b) dO.  Folding T into
// U = [-K^T Diag(alphabar) T^T ; K^T Diag(D2) T^T] (chunk data, formed with
// Att^T dO, E, F and T by a parallel kernel first), a chunk is
//     A1 = [K; Qhat] [dS | dM]           (M 128, N 2 NS, K 128; lanes 0..63 used)
//     dVtilde = Att^T dO + Diag(Gamma_C) A1_S - Diag(w) A1_M      (epilogue)
//     A2 = U dVtilde                     (two M 128, N NS, K 64)
//     dS, dM <- (alphabar_C dS + E, -b_C dS + mubar_C dM - F) + A2   (epilogue)
//   with E = Qhat^T Diag(alphabar) dO and -F = Qhat^T (-Diag(b) dO) issued into
//   A2's accumulators right after A1 (one product of M 128, N 2 NS, K 64, A
//   MN-major from the Qhat rows of the [K; Qhat] tile), while the chain warps
//   form dVtilde
//     A3 = T^T dVtilde = dY              (M 128 with rows 64..127 unused, N NS, K 64;
//                                         off the chain; T^T MN-major from T's rows)
// This is the shape of the forward pass's inter-chunk kernel, whose warp
// roles, hand-offs and bounded waits this kernel keeps: one lane issues the
// MMAs, one lane the TMA and bulk loads (two chunks ahead), 16 chain warps
// hold rows of dS and dM in fp32 registers, 8 columns each (their bf16 copy is
// A1's B operand), 4 output warps write dv.  NS = 32: four CTAs per head.
// The adjoints leaving each chunk are stored in bf16 as the state products'
// operand image (state_img_off), which those products copy in whole.
#include "mdn_internal.cuh"
#include "tc_common.cuh"

namespace mdn {
namespace {

using namespace sm100;
using namespace tc;

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
    static constexpr int NVC = 2;                     // P, E/F operand and coefficient slots
    static constexpr uint32_t kTmemCols = NS == 32 ? 256 : 512;
    // shared memory (byte offsets from a 1024-byte aligned base)
    static constexpr uint32_t KQ0 = 0;                // [K; Qhat], 2 slots x 2 panels x (128 rows x 128 B)
    static constexpr uint32_t FB0 = 2 * 32768;        // T (8 KB of a 16 KB part), [U_S | U_M] (2 x 16 KB), 2 slots
    static constexpr uint32_t FB_BYTES = 49152;
    static constexpr uint32_t ST = FB0 + 2 * FB_BYTES;  // [S | M] bf16, 128 rows, MN-major 128-byte swizzle
    static constexpr uint32_t ST_BYTES = 128 * 2 * NS * 2;
    static constexpr uint32_t YB = ST + ST_BYTES;      // Y 64 rows x NS bf16, MN-major (64 / 128-byte swizzle)
    static constexpr uint32_t YB_BYTES = 64 * NS * 2;
    static constexpr uint32_t V0 = YB + YB_BYTES;      // Att^T dO slice 64 rows x NS bf16, NVC slots
    static constexpr uint32_t V_BYTES = 64 * NS * 2;
    static constexpr uint32_t E0 = V0 + NVC * V_BYTES;   // Diag(alphabar) dO, -Diag(b) dO slices, NVC slots
    static constexpr uint32_t E_BYTES = 2 * 64 * NS * 2;  // (bf16, 64 rows x NS, MN-major: B of E, F)
    static constexpr uint32_t CR0 = E0 + NVC * E_BYTES;  // chunk coefficients (256 floats), NVC slots
    static constexpr uint32_t BARS = CR0 + NVC * 1024;
    static constexpr uint32_t MISC = BARS + 256;
    static constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;  // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory map too large");
    static_assert(ST % 1024 == 0 && YB % 1024 == 0 && V0 % 16 == 0 && E0 % 1024 == 0, "operand alignment");
    // TMEM columns: A1 (KS | KM, QhatS | QhatM) in two slots, A2 (dS | dM), A3 in two slots
    static constexpr uint32_t TM_A1 = 0, TM_A2 = 4 * NS, TM_A3 = 6 * NS;
    static constexpr uint32_t kTxVC = V_BYTES + E_BYTES + 1024;
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
constexpr uint32_t kTxFB = 8192 + 32768;  // T (64 x 64), U

// mbarriers (index into the array at BARS); as in the inter-chunk kernel
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
constexpr int B_MQ = 22;   // [2] A1 and the E / F products complete: the [K; Qhat] slot is free
constexpr int kBars = 24;

struct ChainArgs {
    const float* crec;      // [chunks][256]: Gamma_C, w, ..., alphabar_C, b_C, mubar_C at 192..194
    const __nv_bfloat16* pp;  // [chunks][D/32][64][32]  Att^T dO by slice (bf16)
    const uint8_t* eo;      // [chunks][D/32][2][4096 B]  Diag(alphabar) dO, -Diag(b) dO by slice
    const float* dS_T;      // cotangents of S_T, M_T (may be null)
    const float* dM_T;
    float* dS0;
    float* dM0;
    uint8_t* dss_img;       // [chunks][kStateImgBytes]: adjoints of the states leaving each chunk (bf16)
    float* dv;              // [B, T, H, D] fp32
    uint8_t* dy_img;        // [chunks][kDyImgBytes]: dv of each chunk in bf16 (operand image)
    unsigned* status;
    int T, H, NT;
    const int* cu_seqlens;  // unused here (one batch row per sequence)
    const int* cu_chunks;
    const int* seq_order;   // unused here
};

constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s

// Per-phase cycle sums of CTA 0's MMA lane (slots 0..19), TMA lane (20..39)
// and first chain warp (40..59), in diagnostic builds (MDN_PHASE_CLOCKS, the
// buffer set by mdn_diag_chain_clock); null otherwise.
#ifdef MDN_PHASE_CLOCKS
__device__ float* g_chain_clk = nullptr;
__device__ __forceinline__ float* chain_clk(int slot) {
    return (blockIdx.x == 0 && g_chain_clk) ? g_chain_clk + slot : nullptr;
}
#else
__device__ __forceinline__ float* chain_clk(int) { return nullptr; }
#endif

// Wait for the phase of `bar` with this parity.  Gives up when another role
// has raised the abort flag, or after ~1 s (then raises it itself).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitNs || i > (1u << 26)) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}
// N (8 or 16) consecutive columns of this thread's TMEM lane.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* v) {
    if constexpr (N == 16) tmem_ld16(taddr, v);
    else tmem_ld8(taddr, v);
}

// Warp-uniform form: every lane waits, and the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag));
}

template <int NS>
__global__ void __launch_bounds__(Cfg<NS>::kThreads) __maxnreg__(Cfg<NS>::kMaxRegs)
chunk_bwd_chain_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_qh,
                       const __grid_constant__ CUtensorMap tm_tat, const __grid_constant__ CUtensorMap tm_a2t,
                       const ChainArgs a)
{
    using L = Cfg<NS>;
    static_assert(NS == 32, "the E/F operand slices are laid out for 32 columns");
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
            s[j] = a.dS_T ? a.dS_T[row + j] : 0.f;
            m[j] = a.dM_T ? a.dM_T[row + j] : 0.f;
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

    if (warp == 0) {
        // ------------------------------------------------------------ MMA issue
        if (lid == 0) {
            PhaseClock clk;
            clk.start(chain_clk(0));
            const uint64_t d_kq0 = smem_desc(sbase + L::KQ0, 16, 1024, kSw128);
            // B of A1: [S | M], N = 2 NS; for NS = 64 the S and M halves are two 128-byte panels
            const uint64_t d_st = smem_desc(sbase + L::ST, NS == 32 ? 8192 : 16384, 1024, kSw128);
            const uint64_t d_fb0 = smem_desc(sbase + L::FB0, 16, 1024, kSw128);
            const uint64_t d_y = NS == 32 ? smem_desc(sbase + L::YB, 4096, 512, kSw64)
                                          : smem_desc(sbase + L::YB, 8192, 1024, kSw128);
            constexpr uint32_t ystep = (16 * NS * 2) >> 4;  // 16 rows of Y
            constexpr uint32_t id1 = idesc_bf16(128, 2 * NS, false, true);
            constexpr uint32_t id2 = idesc_bf16(128, NS, false, true);
            constexpr uint32_t idef = idesc_bf16(128, NS, true, true);  // Qhat^T: MN-major A
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
                // E = Qhat^T Diag(alphabar) dO and -F = Qhat^T (-Diag(b) dO) into the
                // accumulators of A2 (read by the last state epilogue, which has
                // signalled), while the chain warps form dVtilde
                {
                    const int sv = n % L::NVC;
                    if (!wait_bar(&bars[B_FVC + sv], (n / L::NVC) & 1, abort_flag)) break;
                    const uint32_t qh = sbase + L::KQ0 + s2 * 32768 + 8192;
                    const uint32_t eo = sbase + L::E0 + sv * L::E_BYTES;
                    // one product of N = 2 NS: B = [Diag(alphabar) dO | -Diag(b) dO] (the two
                    // 32-column MN atoms 4096 B apart), D = the [dS | dM] accumulators
                    constexpr uint32_t idef2 = idesc_bf16(128, 2 * NS, true, true);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t aq = smem_desc(qh + ks * 2048, 16384, 1024, kSw128);
                        mma_bf16(tmem + L::TM_A2, aq, smem_desc(eo + ks * 1024, 4096, 512, kSw64), idef2, ks > 0);
                    }
                    mma_commit(&bars[B_MQ + s2]);  // the last reads of this [K; Qhat] slot
                }
                clk.lap(2);
                if (!wait_bar(&bars[B_FFB + s2], (n >> 1) & 1, abort_flag)) break;
                clk.lap(3);
                if (!wait_bar(&bars[B_YR], n & 1, abort_flag)) break;
                clk.lap(4);
                tc_fence_after_sync();
                const uint64_t dfb = d_fb0 + s2 * (L::FB_BYTES >> 4);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t yd = d_y + ks * ystep;
                    mma_bf16(tmem + L::TM_A2, dfb + (16384 >> 4) + ks * 2, yd, id2, true);
                    mma_bf16(tmem + L::TM_A2 + NS, dfb + (32768 >> 4) + ks * 2, yd, id2, true);
                }
                mma_commit(&bars[B_M2]);
                clk.lap(5);
                // A3 = T^T dVtilde: T^T is the MN-major form of T's row-major rows (M-panel 0;
                // the output rows of panel 1, from the rest of the slot, are not read)
                const uint32_t tt = sbase + L::FB0 + s2 * L::FB_BYTES;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + L::TM_A3 + NS * s2, smem_desc(tt + ks * 2048, 8192, 1024, kSw128),
                             d_y + ks * ystep, idef, ks > 0);
                mma_commit(&bars[B_M3 + s2]);
                clk.lap(6);
                // K, Qhat of chunk n + 1 and the A1 / A3 slot it reuses (read by the
                // output warps of chunk n - 1), waited for while the chain warps
                // form the state of chunk n + 1
                if (n + 1 < NT) {
                    const int t2 = (n + 1) & 1;
                    if (!wait_bar(&bars[B_FKQ + t2], ((n + 1) >> 1) & 1, abort_flag)) break;
                    if (n >= 1 && !wait_bar(&bars[B_OD + t2], ((n - 1) >> 1) & 1, abort_flag)) break;
                }
                clk.lap(7);
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
            clk.start(chain_clk(20));
            int issued_kq = 0, issued_fb = 0, issued_vc = 0;
            for (int n = 0; n < NT; ++n) {
                const int s2 = n & 1, sv = n % L::NVC;
                const int mm = NT - 1 - n;  // chunks are walked backwards
                const long long chunk = ch.chunk0 + mm;
                // the slot's previous chunk (n - 2) has been read by A1 and by E, F
                if (n >= 2 && !wait_bar(&bars[B_MQ + s2], ((n - 2) >> 1) & 1, abort_flag)) break;
                clk.lap(0);
                uint64_t* fb = &bars[B_FKQ + s2];
                mbar_arrive_expect_tx(fb, kTxKQ);
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    uint8_t* dst = sm + L::KQ0 + s2 * 32768 + p * 16384;
                    tma_load_4d(dst, &tm_k, p * 64, h, (ch.n0 + mm) * C, b, fb);
                    tma_load_3d(dst + 8192, &tm_qh, p * 64, 0, (int)chunk, fb);
                }
                issued_kq = n + 1;
                // the chunk's slices of Att^T dO, of the scaled dO and its
                // coefficients first: the chain warps need them before anything
                // else of the chunk, and their slot frees before the T / U slot
                if (n >= L::NVC &&
                    !wait_bar(&bars[B_EVC + sv], ((n / L::NVC) - 1) & 1, abort_flag))
                    break;
                clk.lap(1);
                fb = &bars[B_FVC + sv];
                mbar_arrive_expect_tx(fb, L::kTxVC);
                bulk_load(sm + L::V0 + sv * L::V_BYTES, a.pp + (chunk * (D / NS) + slice) * 64 * NS,
                          L::V_BYTES, fb);
                bulk_load(sm + L::E0 + sv * L::E_BYTES, a.eo + (chunk * (D / NS) + slice) * L::E_BYTES,
                          L::E_BYTES, fb);
                bulk_load(sm + L::CR0 + sv * 1024, a.crec + chunk * 256, 1024, fb);
                issued_vc = n + 1;
                if (n >= 2 && !wait_bar(&bars[B_M3 + s2], ((n - 2) >> 1) & 1, abort_flag)) break;
                clk.lap(2);
                fb = &bars[B_FFB + s2];
                mbar_arrive_expect_tx(fb, kTxFB);
                uint8_t* dst = sm + L::FB0 + s2 * L::FB_BYTES;
                tma_load_3d(dst, &tm_tat, 0, 0, (int)chunk, fb);
                tma_load_3d(dst + 16384, &tm_a2t, 0, 0, (int)chunk, fb);
                tma_load_3d(dst + 32768, &tm_a2t, 0, 128, (int)chunk, fb);
                issued_fb = n + 1;
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
        clk.start(warp == kChainWarp0 + 2 && lid == 0 ? chain_clk(40) : nullptr);
        for (int n = 0; n < NT; ++n) {
            const int s2 = n & 1, sv = n % L::NVC;
            const long long chunk = ch.chunk0 + (NT - 1 - n);
            if (!warp_wait(&bars[B_FVC + sv], (n / L::NVC) & 1, abort_flag)) break;
            clk.lap(0);
            const float* cr = reinterpret_cast<const float*>(sm + L::CR0 + sv * 1024);
            const float abC = cr[3 * C], bC = cr[3 * C + 1], mbC = cr[3 * C + 2];
            if (ypart) {
                const float c_g = cr[r], c_w = cr[C + r];
                const uint4* prow = reinterpret_cast<const uint4*>(
                    sm + L::V0 + sv * L::V_BYTES + (r * NS + NH * hc) * 2);
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
                    float vv[8];  // dVtilde = Att^T dO + Gamma_C K dS - w K dM
                    unpack_bf16x8(prow[c], vv);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        vv[e] += fmaf(c_g, x[8 * c + e], -c_w * y[8 * c + e]);
                    st_bf16x8(sm + L::YB + L::y_off(r, hc * (NH / 8) + c), vv);
                }
                clk.lap(2);
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lid == 0) mbar_arrive(&bars[B_YR]);
                clk.lap(3);
            }
            // the adjoints of the states leaving this chunk, kept (bf16, as the
            // state products' operand image) for the chunk-local gradients;
            // stored once Y is on its way (the stores' issue stalls would
            // otherwise delay Y)
            {
                uint8_t* dst = a.dss_img + (size_t)chunk * kStateImgBytes;
#pragma unroll
                for (int c = 0; c < NH / 8; ++c) {
                    const int g = (j0 + NH * hc) / 8 + c;
                    st_bf16x8(dst + state_img_off(lane, g), s + 8 * c);
                    st_bf16x8(dst + state_img_off(lane + D, g), m + 8 * c);
                }
            }
            clk.lap(7);
            if (!warp_wait(&bars[B_M2], n & 1, abort_flag)) break;
            // the products of this chunk (E and F among them) have read the
            // slot: it may be refilled
            if (lid == 0) mbar_arrive(&bars[B_EVC + sv]);
            clk.lap(4);
            tc_fence_after_sync();
            {
                float dS[NH], dM[NH];
                tmem_ld_cols<NH>(tq + L::TM_A2 + NH * hc, dS);
                tmem_ld_cols<NH>(tq + L::TM_A2 + NS + NH * hc, dM);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < NH; ++j) {
                    // dS holds E + U_S dVtilde, dM holds -F + U_M dVtilde
                    const float sn = fmaf(abC, s[j], dS[j]);
                    m[j] = fmaf(mbC, m[j], fmaf(-bC, s[j], dM[j]));
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
        const bool yrow = quad < 2;  // lanes 0..63: rows of dY (lanes 64..127 of A3 are zero)
        const int r = lane & 63;
        for (int n = 0; n < NT; ++n) {
            const int s2 = n & 1, sv = n % L::NVC;
            if (!warp_wait(&bars[B_FVC + sv], (n / L::NVC) & 1, abort_flag)) break;
            __syncwarp();
            if (lid == 0) mbar_arrive(&bars[B_EVC + sv]);
            if (!warp_wait(&bars[B_M3 + s2], (n >> 1) & 1, abort_flag)) break;
            tc_fence_after_sync();
            if (yrow) {
                const int t = (NT - 1 - n) * C + r;  // token of the chain
                float* dst = a.dv + ((size_t)(ch.out0 + t) * a.H + h) * D + j0;
                // dY in bf16 as the chunk-local kernels' operand image (2 panels of
                // 64 rows x 128 B, 128-byte swizzle; zero past the end of the sequence)
                uint8_t* im = a.dy_img + (size_t)(ch.chunk0 + (NT - 1 - n)) * kDyImgBytes;
#pragma unroll 1
                for (int q16 = 0; q16 < NS / 16; ++q16) {
                    float x[16];
                    tmem_ld16(tq + L::TM_A3 + NS * s2 + 16 * q16, x);
                    tmem_wait_ld();
                    const bool keep = t < ch.len;
                    if (keep) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<float4*>(dst + 16 * q16 + 4 * q) =
                                make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = keep ? x[e] : 0.f;
                    const int c = j0 + 16 * q16;
                    uint8_t* row = im + (c >> 6) * 8192;
                    st_bf16x8(row + sw128_off(r, (c & 63) >> 3), x);
                    st_bf16x8(row + sw128_off(r, ((c & 63) >> 3) + 1), x + 8);
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
            a.dS0[row + j] = s[j];
            a.dM0[row + j] = m[j];
        }
    }
    if (!ok && tid == 0) atomicOr(a.status + 1, 1u);
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

}  // namespace

#ifdef MDN_PHASE_CLOCKS
extern "C" int mdn_diag_chain_clock(float* p)
{
    return cudaMemcpyToSymbol(g_chain_clk, &p, sizeof(p)) == cudaSuccess ? 0 : 1;
}
#endif

cudaError_t launch_bwd_chain_tc(const BwdArgs& a, cudaStream_t s)
{
    constexpr int NS = 32;
    using L = Cfg<NS>;
    if (a.D != D) return cudaErrorNotSupported;
    CUtensorMap mk, mqh, mtt, mu;
    const long long chunks = (long long)a.B * a.H * a.NT;
    if (!make_token_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_chunk_map(&mqh, a.bc_qh, chunks, C, D, C) ||
        !make_chunk_map(&mtt, a.bc_tt, chunks, C, C, C) ||
        !make_chunk_map(&mu, a.bc_u, chunks, 2 * D, C, 128))
        return cudaErrorInvalidValue;
    ChainArgs t;
    t.crec = a.bc_rec;
    t.pp = a.bc_p;
    t.eo = a.bc_eo;
    t.dS_T = a.dS_T;
    t.dM_T = a.dM_T;
    t.dS0 = a.dS0;
    t.dM0 = a.dM0;
    t.dss_img = a.dss_img;
    t.dv = a.dv;
    t.dy_img = a.dy_img;
    t.status = a.status;
    t.T = a.T;
    t.H = a.H;
    t.NT = a.NT;
    t.cu_seqlens = nullptr;
    t.cu_chunks = nullptr;
    t.seq_order = nullptr;
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_chain_kernel<NS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)a.B * a.H * (D / NS);
    ProfScope ps(kBwdChain, s);
    chunk_bwd_chain_kernel<NS><<<(unsigned)blocks, L::kThreads, L::SMEM_BYTES, s>>>(mk, mqh, mtt, mu, t);
    return cudaGetLastError();
}

}  // namespace mdn
