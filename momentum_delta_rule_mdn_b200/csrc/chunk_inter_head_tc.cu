// K-3 on sm_100a with one CTA per head: sequential state passing over the
// chunks for all d_v = 128 columns of S, M and Vtilde at once, with the
// carried-state and intra-chunk parts of o, on tcgen05 tensor cores fed by TMA.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 4.  The chunk algebra is the one of the
// column-slice kernel (chunk_inter_tc.cu): with X = D1 K S - D2 K M
// (D1 = Diag(alphabar_r), D2 = Diag(alpha_r b_{r-1})), Y = V - X and
// Vtilde = T Y; o = Diag(alphabar) Qhat S - Diag(b) Qhat M + (Att T) Y; and the
// chunk-end update S' = alphabar_C S - b_C M + A2T_S Y, M' = mubar_C M + A2T_M Y
// with the intra-chunk kernel's A2T = [K^T Diag(Gamma_C) T; -K^T Diag(w) T].
//
// A whole head per CTA makes every product wide: A1 = [K; Qhat] [S | M] is
// M = 128, N = 256 (a tcgen05.mma of N = 256 does twice the work of one of
// N <= 128 for about twice the time, where the narrower slices pay the same
// issue cost for less), and the chunk operands are loaded once per head
// instead of once per slice.  TMEM (512 columns) holds:
//   columns   0..255  A1 of the current chunk: lanes 0..63 K S | K M,
//                     lanes 64..127 Qhat S | Qhat M
//   columns 256..511  the state S | M (lane i = row i of d_k), fp32, kept
//                     between chunks already scaled for the next update:
//                     S' = alphabar_C S - b_C M, M' = mubar_C M, so that A2
//                     accumulates onto it: S_{n+1} = S' + A2T_S Y, M_{n+1} = M' + A2T_M Y
// Per chunk n:
//   A1 = [K; Qhat] [S | M]                     (N = 256, K = 128)
//   Y  = V - (D1 KS - D2 KM)                    lanes 0..63, into shared memory; those
//                                               lanes' columns 0..127 are then cleared
//   Oi = Diag(alphabar) QhatS - Diag(b) QhatM   lanes 64..127, written over columns 0..127
//   A2: state += [A2T_S; A2T_M] Y              (two M = 128, N = 128, K = 64)
//   A3: columns 0..127 += [T; Att T] Y         -> lanes 0..63 Vtilde, lanes 64..127 o
// Only A1 -> Y -> A2 -> state is sequential.  Warps:
//   warp 0        one lane issues every tcgen05.mma and commit
//   warp 1        one lane issues every TMA load and bulk copy
//   16 chain warps  warp w reads TMEM lanes 32(w%4).. and 32 columns; the eight on
//                 lanes 0..63 form Y, the eight on lanes 64..127 form Oi; after
//                 A2 all sixteen read the state once, write its bf16 copy (the B
//                 operand of the next A1) and store it back rescaled in TMEM
//   8 output warps  Vtilde and o of chunk n from A3, read out of TMEM (which
//                 frees it for the next A1) before they go to global memory
// Hand-offs are mbarriers only; every wait is bounded (as in the slice
// kernel: a wait that runs out raises the CTA's abort flag, every role leaves
// its loop, copies and MMAs in flight are drained, and status[1] is set).
#include "inter_common.cuh"

namespace mdn {
namespace {

using namespace sm100;
using namespace tc;
using namespace inter;

constexpr int kChainWarp0 = 2;                 // warps 0, 1: MMA issue, loads
constexpr int kOutWarp0 = kChainWarp0 + 16;    // 16 chain warps
constexpr int kWarps = kOutWarp0 + 8;          // 8 output warps
constexpr int kThreads = kWarps * 32;

// Shared memory (byte offsets from a 1024-byte aligned base).
constexpr uint32_t KQ0 = 0;             // [K; Qhat], 2 slots x 2 feature panels x (128 rows x 128 B)
constexpr uint32_t FB = 65536;          // [T; Att T] (16 KB), A2T_S (16 KB), A2T_M (16 KB)
constexpr uint32_t ST = FB + 49152;     // [S | M] bf16, MN-major: 4 panels of 64 columns x 128 rows
constexpr uint32_t YB = ST + 65536;     // Y bf16, MN-major: 2 panels of 64 columns x 64 rows
constexpr uint32_t VB = YB + 16384;     // V: 2 boxes of 64 columns x 64 rows (128-byte swizzle)
constexpr uint32_t CR0 = VB + 16384;    // chunk records (256 floats), 4 slots
constexpr uint32_t BARS = CR0 + 4096;
constexpr uint32_t MISC = BARS + 256;
constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory map too large");
static_assert(FB % 1024 == 0 && ST % 1024 == 0 && YB % 1024 == 0 && VB % 1024 == 0,
              "operand alignment");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TM_A1 = 0, TM_S = 256, TM_M = 384;
constexpr uint32_t kTxKQ = 32768, kTxFB = 49152, kTxV = 16384, kTxCR = 1024;

// mbarriers (index into the array at BARS)
constexpr int B_FKQ = 0;   // [2] K, Qhat landed
constexpr int B_FFB = 2;   //     [T; Att T], A2T landed
constexpr int B_FV = 3;    //     V landed
constexpr int B_FCR = 4;   // [4] chunk record landed
constexpr int B_ECR = 8;   // [4] chunk record released (16 chain warps)
constexpr int B_M1 = 12;   // [2] A1 complete (per K/Qhat slot)
constexpr int B_M2 = 14;   //     A2 complete
constexpr int B_M3 = 15;   //     A3 complete (and every earlier MMA)
constexpr int B_YR = 16;   //     Y written, K-row columns cleared (8 warps)
constexpr int B_OI = 17;   //     Oi written (8 warps)
constexpr int B_SR = 18;   //     bf16 state for the next A1 written (16 warps)
constexpr int B_PS = 19;   //     fp32 state rescaled for the next A2 (16 warps)
constexpr int B_OD = 20;   //     A3 read by the output warps (8 warps)
constexpr int B_FIN = 21;  //     every MMA complete (exit)
constexpr int kBars = 22;

__global__ void __launch_bounds__(kThreads, 1)
chunk_inter_head_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_qh,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_tat,
                        const __grid_constant__ CUtensorMap tm_a2t, const InterArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lid = tid & 31;
    const int quad = warp & 3;            // TMEM lane quadrant this warp may access
    const int lane = (quad << 5) | lid;   // TMEM lane
    const Chain ch = chain_of(a, blockIdx.x);
    const int b = ch.b, h = ch.h, NT = ch.nt;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + MISC + 4);
    const bool chain = warp >= kChainWarp0 && warp < kOutWarp0;
    const int grp = (warp - kChainWarp0) >> 2;  // chain warp: columns 32 grp .. 32 grp + 31

    if (tid == 0) {
        for (int k = 0; k < kBars; ++k) {
            uint32_t count = 1;  // TMA (expect_tx) and tcgen05.commit barriers
            if (k >= B_ECR && k < B_ECR + 4) count = 16;
            if (k == B_YR || k == B_OI || k == B_OD) count = 8;
            if (k == B_SR || k == B_PS) count = 16;
            mbar_init(&bars[k], count);
        }
        mbar_fence_init();
        *abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
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
        if (lid == 0 && NT > 0) {
            PhaseClock clk;
            clk.start((a.dbg && blockIdx.x == 0) ? a.dbg : nullptr);
            const uint64_t d_kq0 = smem_desc(sbase + KQ0, 16, 1024, kSw128);
            const uint64_t d_st = smem_desc(sbase + ST, 16384, 1024, kSw128);
            const uint64_t d_fb = smem_desc(sbase + FB, 16, 1024, kSw128);
            const uint64_t d_y = smem_desc(sbase + YB, 8192, 1024, kSw128);
            constexpr uint32_t id1 = idesc_bf16(128, 256, false, true);
            constexpr uint32_t id2 = idesc_bf16(128, 128, false, true);
            for (int n = 0; n < NT; ++n) {
                const int s2 = n & 1;
                clk.lap(0);
                if (!wait_bar(&bars[B_FKQ + s2], (n >> 1) & 1, abort_flag)) break;
                if (!wait_bar(&bars[B_SR], n & 1, abort_flag)) break;
                if (n >= 1 && !wait_bar(&bars[B_OD], (n - 1) & 1, abort_flag)) break;
                clk.lap(1);
                tc_fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tmem + TM_A1,
                             d_kq0 + ((s2 * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32) >> 4),
                             d_st + ((ks * 2048) >> 4), id1, ks > 0);
                mma_commit(&bars[B_M1 + s2]);
                clk.lap(2);
                if (!wait_bar(&bars[B_FFB], n & 1, abort_flag)) break;
                if (!wait_bar(&bars[B_PS], n & 1, abort_flag)) break;
                if (!wait_bar(&bars[B_YR], n & 1, abort_flag)) break;
                clk.lap(3);
                tc_fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t yd = d_y + ((ks * 2048) >> 4);
                    mma_bf16(tmem + TM_S, d_fb + ((16384 + ks * 32) >> 4), yd, id2, 1);
                    mma_bf16(tmem + TM_M, d_fb + ((32768 + ks * 32) >> 4), yd, id2, 1);
                }
                mma_commit(&bars[B_M2]);
                clk.lap(4);
                if (!wait_bar(&bars[B_OI], n & 1, abort_flag)) break;
                tc_fence_after_sync();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + TM_A1, d_fb + ((ks * 32) >> 4), d_y + ((ks * 2048) >> 4), id2,
                             1);
                mma_commit(&bars[B_M3]);
                clk.lap(5);
            }
            clk.flush();
        }
        if (lid == 0) {
            // every issued MMA has completed before TMEM and shared memory are released
            mma_commit(&bars[B_FIN]);
            (void)mbar_wait(&bars[B_FIN], 0);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ TMA loads
        if (lid == 0) {
            int issued_kq = 0, issued_cr = 0, issued_v = 0, issued_fb = 0;
            for (int n = 0; n < NT; ++n) {
                const long long chunk = ch.chunk0 + n;
                const int s2 = n & 1, sc = n & 3;
                // the operands of chunk n are in global memory
                if (!wait_ready(a.ready + chunk, abort_flag)) break;
                fence_proxy_async_global();
                // K, Qhat: the slot's previous chunk (n - 2) has been read by its A1
                if (n >= 2 && !wait_bar(&bars[B_M1 + s2], ((n - 2) >> 1) & 1, abort_flag)) break;
                uint64_t* fb = &bars[B_FKQ + s2];
                mbar_arrive_expect_tx(fb, kTxKQ);
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    uint8_t* dst = sm + KQ0 + s2 * 32768 + p * 16384;
                    tma_load_4d(dst, &tm_k, p * 64, h, (ch.n0 + n) * C, b, fb);
                    tma_load_3d(dst + 8192, &tm_qh, p * 64, 0, (int)chunk, fb);
                }
                issued_kq = n + 1;
                // chunk record: its slot's previous chunk (n - 4) has been released
                if (n >= 4 && !wait_bar(&bars[B_ECR + sc], ((n - 4) >> 2) & 1, abort_flag)) break;
                fb = &bars[B_FCR + sc];
                mbar_arrive_expect_tx(fb, kTxCR);
                bulk_load(sm + CR0 + sc * 1024, a.crec + chunk * 256, kTxCR, fb);
                issued_cr = n + 1;
                // V: the previous chunk's Y has been formed from it
                if (n >= 1 && !wait_bar(&bars[B_YR], (n - 1) & 1, abort_flag)) break;
                fb = &bars[B_FV];
                mbar_arrive_expect_tx(fb, kTxV);
#pragma unroll
                for (int p = 0; p < 2; ++p)
                    tma_load_4d(sm + VB + p * 8192, &tm_v, p * 64, h, (ch.n0 + n) * C, b, fb);
                issued_v = n + 1;
                // [T; Att T], A2T: the previous chunk's A2 and A3 have completed
                if (n >= 1 && !wait_bar(&bars[B_M3], (n - 1) & 1, abort_flag)) break;
                fb = &bars[B_FFB];
                mbar_arrive_expect_tx(fb, kTxFB);
                tma_load_3d(sm + FB, &tm_tat, 0, 0, (int)chunk, fb);
                tma_load_3d(sm + FB + 16384, &tm_a2t, 0, 0, (int)chunk, fb);
                tma_load_3d(sm + FB + 32768, &tm_a2t, 0, 128, (int)chunk, fb);
                issued_fb = n + 1;
            }
            // Copies that were issued must land before shared memory is
            // released (after an abort some were never consumed).  A phase
            // that has completed passes at once.
            for (int n = issued_kq - 2; n < issued_kq; ++n)
                if (n >= 0) (void)mbar_wait(&bars[B_FKQ + (n & 1)], (n >> 1) & 1);
            for (int n = issued_cr - 4; n < issued_cr; ++n)
                if (n >= 0) (void)mbar_wait(&bars[B_FCR + (n & 3)], (n >> 2) & 1);
            if (issued_v > 0) (void)mbar_wait(&bars[B_FV], (issued_v - 1) & 1);
            if (issued_fb > 0) (void)mbar_wait(&bars[B_FFB], (issued_fb - 1) & 1);
        }
        __syncwarp();
    } else if (chain) {
        // ------------------------------------------------------------ chain epilogues
        const size_t row = ((size_t)ch.sh * D + lane) * D + 32 * grp;  // state row `lane`
        const int pan = grp >> 1;           // 64-column panel of the columns 32 grp ..
        const int c16 = (grp & 1) * 4;      // their first 16-byte chunk in a 128-byte row
        const uint32_t s_col = TM_S + 32 * grp, m_col = TM_M + 32 * grp;
        bool ok = true;
        PhaseClock clk;  // diagnostics: a Y warp (quad 0) and an Oi warp (quad 2) of CTA 0
        clk.start((a.dbg && blockIdx.x == 0 && lid == 0 && grp == 0 && (quad == 0 || quad == 2))
                      ? a.dbg + (quad == 0 ? 20 : 40) : nullptr);
        // the entering state: its bf16 copy, and the fp32 state rescaled for chunk 0
        if (NT > 0) {
            ok = warp_wait(&bars[B_FCR], 0, abort_flag);
            if (ok) {
                const float* cr = reinterpret_cast<const float*>(sm + CR0);
                const float abC = cr[3 * C], bC = cr[3 * C + 1], mbC = cr[3 * C + 2];
#pragma unroll 1
                for (int p = 0; p < 2; ++p) {
                    float s[16], m[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        s[j] = a.S0 ? a.S0[row + 16 * p + j] : 0.f;
                        m[j] = a.M0 ? a.M0[row + 16 * p + j] : 0.f;
                    }
                    const int cc = c16 + 2 * p;
                    st_bf16x8(sm + ST + pan * 16384 + sw128_off(lane, cc), s);
                    st_bf16x8(sm + ST + pan * 16384 + sw128_off(lane, cc + 1), s + 8);
                    st_bf16x8(sm + ST + (2 + pan) * 16384 + sw128_off(lane, cc), m);
                    st_bf16x8(sm + ST + (2 + pan) * 16384 + sw128_off(lane, cc + 1), m + 8);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        s[j] = fmaf(abC, s[j], -bC * m[j]);
                        m[j] *= mbC;
                    }
                    tmem_st16(tq + s_col + 16 * p, s);
                    tmem_st16(tq + m_col + 16 * p, m);
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                if (lid == 0) {
                    mbar_arrive(&bars[B_SR]);
                    mbar_arrive(&bars[B_PS]);
                }
            }
        } else if (a.S_T) {
            // an empty chain (a packed sequence without tokens): S_T = S0, M_T = M0
#pragma unroll 4
            for (int j = 0; j < 32; ++j) {
                a.S_T[row + j] = a.S0 ? a.S0[row + j] : 0.f;
                a.M_T[row + j] = a.M0 ? a.M0[row + j] : 0.f;
            }
        }
        for (int n = 0; n < NT && ok; ++n) {
            const int s2 = n & 1, sc = n & 3;
            const float* cr = reinterpret_cast<const float*>(sm + CR0 + sc * 1024);
            clk.lap(0);
            if (!warp_wait(&bars[B_FCR + sc], (n >> 2) & 1, abort_flag)) break;
            if (quad < 2) {
                // ---- Y = V - (D1 KS - D2 KM) for rows 0..63, then clear those columns
                const int r = lane;
                const float c_ab = cr[r], c_d2 = cr[C + r];
                if (!warp_wait(&bars[B_FV], n & 1, abort_flag)) break;
                clk.lap(1);
                if (!warp_wait(&bars[B_M1 + s2], (n >> 1) & 1, abort_flag)) break;
                clk.lap(2);
                tc_fence_after_sync();
#pragma unroll 1
                for (int p = 0; p < 2; ++p) {
                    const uint32_t col = TM_A1 + 32 * grp + 16 * p;
                    const int cc = c16 + 2 * p;
                    float x[16], y[16], v[16];
                    tmem_ld16(tq + col, x);
                    tmem_ld16(tq + col + 128, y);
                    unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + VB + pan * 8192 +
                                                                  sw128_off(r, cc)), v);
                    unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + VB + pan * 8192 +
                                                                  sw128_off(r, cc + 1)), v + 8);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[e] -= fmaf(c_ab, x[e], -c_d2 * y[e]);
                    st_bf16x8(sm + YB + pan * 8192 + sw128_off(r, cc), v);
                    st_bf16x8(sm + YB + pan * 8192 + sw128_off(r, cc + 1), v + 8);
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = 0.f;
                    tmem_st16(tq + col, x);
                }
                clk.lap(3);
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before_sync();
                __syncwarp();
                clk.lap(4);
                if (lid == 0) {
                    mbar_arrive(&bars[B_YR]);
                    mbar_arrive(&bars[B_ECR + sc]);
                }
            } else {
                // ---- Oi = Diag(alphabar) QhatS - Diag(b) QhatM for rows 64..127, in place
                const int r = lane - 64;
                const float c_ab = cr[r], c_b = cr[2 * C + r];
                clk.lap(1);
                if (!warp_wait(&bars[B_M1 + s2], (n >> 1) & 1, abort_flag)) break;
                clk.lap(2);
                tc_fence_after_sync();
#pragma unroll 1
                for (int p = 0; p < 2; ++p) {
                    const uint32_t col = TM_A1 + 32 * grp + 16 * p;
                    float x[16], y[16];
                    tmem_ld16(tq + col, x);
                    tmem_ld16(tq + col + 128, y);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = fmaf(c_ab, x[e], -c_b * y[e]);
                    tmem_st16(tq + col, x);
                }
                clk.lap(3);
                tmem_wait_st();
                tc_fence_before_sync();
                __syncwarp();
                clk.lap(4);
                if (lid == 0) {
                    mbar_arrive(&bars[B_OI]);
                    mbar_arrive(&bars[B_ECR + sc]);
                }
            }
            // ---- the state after chunk n
            clk.lap(5);
            if (!warp_wait(&bars[B_M2], n & 1, abort_flag)) break;
            clk.lap(6);
            tc_fence_after_sync();
            if (n + 1 == NT) {
                // S_T, M_T (nothing reads the bf16 copy or the rescaled state any more)
#pragma unroll 1
                for (int p = 0; p < 2; ++p) {
                    float s[16], m[16];
                    tmem_ld16(tq + s_col + 16 * p, s);
                    tmem_ld16(tq + m_col + 16 * p, m);
                    tmem_wait_ld();
                    float4* so = reinterpret_cast<float4*>(a.S_T + row + 16 * p);
                    float4* mo = reinterpret_cast<float4*>(a.M_T + row + 16 * p);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        so[q4] = make_float4(s[4 * q4], s[4 * q4 + 1], s[4 * q4 + 2], s[4 * q4 + 3]);
                        mo[q4] = make_float4(m[4 * q4], m[4 * q4 + 1], m[4 * q4 + 2], m[4 * q4 + 3]);
                    }
                }
                break;
            }
            // bf16 copy for the next A1, and the fp32 state rescaled in place for
            // the next A2 (chunk n + 1's record was loaded with its K, Qhat), from
            // one read of the state
            const int sn = (n + 1) & 3;
            if (!warp_wait(&bars[B_FCR + sn], ((n + 1) >> 2) & 1, abort_flag)) break;
            const float* crn = reinterpret_cast<const float*>(sm + CR0 + sn * 1024);
            const float abC = crn[3 * C], bC = crn[3 * C + 1], mbC = crn[3 * C + 2];
            clk.lap(7);
#pragma unroll 1
            for (int p = 0; p < 2; ++p) {
                float s[16], m[16];
                tmem_ld16(tq + s_col + 16 * p, s);
                tmem_ld16(tq + m_col + 16 * p, m);
                tmem_wait_ld();
                const int cc = c16 + 2 * p;
                st_bf16x8(sm + ST + pan * 16384 + sw128_off(lane, cc), s);
                st_bf16x8(sm + ST + pan * 16384 + sw128_off(lane, cc + 1), s + 8);
                st_bf16x8(sm + ST + (2 + pan) * 16384 + sw128_off(lane, cc), m);
                st_bf16x8(sm + ST + (2 + pan) * 16384 + sw128_off(lane, cc + 1), m + 8);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    s[j] = fmaf(abC, s[j], -bC * m[j]);
                    m[j] *= mbC;
                }
                tmem_st16(tq + s_col + 16 * p, s);
                tmem_st16(tq + m_col + 16 * p, m);
            }
            clk.lap(8);
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lid == 0) mbar_arrive(&bars[B_SR]);
            clk.lap(9);
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (lid == 0) mbar_arrive(&bars[B_PS]);
            clk.lap(10);
        }
        clk.flush();
    } else {
        // ------------------------------------------------------------ outputs
        const int half = (warp - kOutWarp0) >> 2;  // columns 64 half .. 64 half + 63
        const bool orow = quad >= 2;               // lanes 64..127: rows of o; 0..63: of Vtilde
        const int r = lane & 63;
        __nv_bfloat16* const out = orow ? a.o : a.vt;
        PhaseClock clk;  // diagnostics: one output warp of CTA 0
        clk.start((a.dbg && blockIdx.x == 0 && lid == 0 && warp == kOutWarp0) ? a.dbg + 60 : nullptr);
        for (int n = 0; n < NT; ++n) {
            clk.lap(0);
            if (!warp_wait(&bars[B_M3], n & 1, abort_flag)) break;
            clk.lap(1);
            tc_fence_after_sync();
            // read the 64 columns and pack them to bf16 first: the TMEM columns
            // are released (for the next chunk's A1) before the global stores
            uint32_t pk[32];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                float x[16], y[16];
                tmem_ld16(tq + TM_A1 + 64 * half + 32 * p, x);
                tmem_ld16(tq + TM_A1 + 64 * half + 32 * p + 16, y);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    pk[16 * p + e] = pack_bf16(x[2 * e], x[2 * e + 1]);
                    pk[16 * p + 8 + e] = pack_bf16(y[2 * e], y[2 * e + 1]);
                }
            }
            clk.lap(2);
            tc_fence_before_sync();
            __syncwarp();
            if (lid == 0) mbar_arrive(&bars[B_OD]);
            // Transpose 16-byte chunks within each group of eight lanes (three
            // butterfly exchanges): lane 8 o + j then holds chunk j of rows
            // 8 o .. 8 o + 7 of the warp, so that one store instruction writes four
            // whole 128-byte rows instead of 32 scattered 16-byte pieces.
            uint4 ch16[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                ch16[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            const int j8 = lid & 7;
#pragma unroll
            for (int m = 4; m >= 1; m >>= 1) {
                const bool hi = (j8 & m) != 0;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    if (c & m) continue;
                    const uint4 snd = hi ? ch16[c] : ch16[c | m];
                    uint4 rcv;
                    rcv.x = __shfl_xor_sync(0xffffffffu, snd.x, m);
                    rcv.y = __shfl_xor_sync(0xffffffffu, snd.y, m);
                    rcv.z = __shfl_xor_sync(0xffffffffu, snd.z, m);
                    rcv.w = __shfl_xor_sync(0xffffffffu, snd.w, m);
                    if (hi) ch16[c] = rcv;
                    else ch16[c | m] = rcv;
                }
            }
            const int rbase = (r & ~31) + (lid & ~7);  // first row of this lane's group of eight
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int t = n * C + rbase + k;  // token of the chain
                if (t < ch.len)
                    reinterpret_cast<uint4*>(out + ((size_t)(ch.out0 + t) * a.H + h) * D +
                                             64 * half)[j8] = ch16[k];
            }
            clk.lap(3);
        }
        clk.flush();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (*abort_flag != 0 && tid == 0) atomicOr(a.status + 1, 1u);
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
#ifdef MDN_PHASE_CLOCKS
    if (a.dbg && tid == 0 && blockIdx.x < 1024) {
        double* tl = reinterpret_cast<double*>(a.dbg + 30000);
        tl[2 * blockIdx.x] = (double)t_start;
        tl[2 * blockIdx.x + 1] = (double)global_timer_ns();
    }
#endif
}

}  // namespace

// One CTA per chain (head, or packed sequence and head), launched as the
// programmatic dependent of the intra-chunk kernel on the same stream.
cudaError_t launch_inter_head(const ChunkArgs& a, cudaStream_t s)
{
    CUtensorMap mk, mqh, mv, mtat, ma2t;
    const long long chunks = (long long)a.B * a.H * a.NT;
    if (!make_token_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_chunk_map(&mqh, a.qhat, chunks, C, D, C) ||
        !make_token_map(&mv, a.v, a.B, a.T, a.H, 64, true) ||
        !make_chunk_map(&mtat, a.tat, chunks, 2 * C, C, 2 * C) ||
        !make_chunk_map(&ma2t, a.a2t, chunks, 2 * D, C, 128))
        return cudaErrorInvalidValue;
    const InterArgs t = inter_args(a);
    cudaError_t e = cudaFuncSetAttribute(chunk_inter_head_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const long long chains = a.cu_chunks ? (long long)a.nseq * a.H : (long long)a.B * a.H;
    ProfScope ps(kInterTc, s);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)chains);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, chunk_inter_head_kernel, mk, mqh, mv, mtat, ma2t, t);
}

}  // namespace mdn
