// B-3a of the backward pass on tcgen05 tensor cores (bf16 inputs, d = 128).
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, step 7 (the backward pass rebuilds S and M from
// the saved Vtilde).  Per chunk, with S, M the states entering it and dS, dM
// the adjoints of the states leaving it, the six products
//     [dO; dY] [S | M]^T   -> P1 = dO S^T, P2 = dO M^T, P5 = dY S^T, P6 = dY M^T
//     [Vt; K]  [dS | dM]^T -> P3 = Vt dS^T, P4 = Vt dM^T  (product rows 64..127 unused)
// are two groups of eight tcgen05.mma (M 128, N 256, K 128; bf16 operands,
// fp32 accumulators in 512 TMEM columns).  The epilogue forms the parts of dq
// and dk they carry,
//     dq = Diag(alphabar) P1 - Diag(b) P2
//     dk = Diag(Gamma_C) P3 - Diag(w) P4 - Diag(alphabar) P5 + Diag(D2) P6 - d dq
// (the last term from Qhat = Q - d K, for this kernel's part of dq) and the
// row sums that feed the gate gradients, as the CUDA-core kernel does.  Every
// operand arrives by the copy engines, K-major with the 128-byte swizzle: the
// states and adjoints as bf16 images of the B operands (written by the state
// scan and the reverse chain) and dY as the reverse chain's bf16 image, by
// bulk copies; the dO, Vt, K and Q rows by TMA.  12 warps, three per TMEM lane
// quadrant, each a third of the columns; dq and dk leave as 512-byte row
// stores from staging tiles over the state images.
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
constexpr uint32_t SA2 = 32768;      // [Vt; K]: the product rows of K are not read; the
                                     // epilogue reads K from there
constexpr uint32_t SB1 = 65536;      // [S | M] as 256 rows: 2 K-panels x 256 rows x 128 B
constexpr uint32_t SB2 = 131072;     // [dS | dM]
constexpr uint32_t SQ = 196608;      // Q rows for the epilogue: 2 K-panels x 64 rows x 128 B
constexpr int kThrS = 384;           // threads of the state-product kernel (3 warps per TMEM quadrant)
constexpr int kSumSlots = 18;        // row-sum partial slots (see the kernel)
constexpr uint32_t SSUM = SQ + 16384;  // fp32 row-sum partials [18][64], then scalars [12][3]
constexpr uint32_t SBAR = SSUM + kSumSlots * 64 * 4 + (kThrS / 32) * 3 * 4;
constexpr uint32_t SMISC = SBAR + 16;  // after two mbarriers (MMAs done, state images landed)
constexpr uint32_t SMEM_BYTES = SMISC + 16 + 1024;  // + alignment slack
constexpr int XS = 129;              // row stride (floats) of the dk exchange tile over SA1
constexpr int kRowS = 132;           // row stride (floats) of the dq / dk staging tiles: rows
                                     // 16-byte aligned, float4 accesses of 8 rows conflict-free
static_assert(2 * 64 * kRowS * 4 <= SQ - SB1, "dq / dk staging tiles over the state images");

__device__ __forceinline__ size_t tokrow(const BwdArgs& a, int b, int t, int h) {
    return ((size_t)b * a.T + t) * a.H + h;
}

// Per-phase cycle counts of the per-chunk kernels, as seen by thread 0 of
// every CTA and summed over CTAs (slot kBwdClkCtas of each kernel's block
// counts them).  Diagnostic builds only (MDN_PHASE_CLOCKS, with the buffer set
// by mdn_diag_bwd_clock); otherwise every call is empty.
#ifdef MDN_PHASE_CLOCKS
constexpr int kBwdClkSlots = 32, kBwdClkCtas = 31;
__device__ float* g_bwd_clk = nullptr;
struct BwdClock {
    long long t;
    float acc[kBwdClkSlots];
    bool on;
    __device__ __forceinline__ void start(bool o) {
        on = o;
#pragma unroll
        for (int k = 0; k < kBwdClkSlots; ++k) acc[k] = 0.f;
        t = clock_now();
    }
    __device__ __forceinline__ void lap(int k) {
        if (on) {
            const long long now = clock_now();
            acc[k] += (float)(now - t);
            t = now;
        }
    }
    __device__ __forceinline__ void flush(int block) {
        float* out = g_bwd_clk;
        if (!on || !out) return;
        out += block * kBwdClkSlots;
        for (int k = 0; k < kBwdClkCtas; ++k) atomicAdd(out + k, acc[k]);
        atomicAdd(out + kBwdClkCtas, 1.f);
    }
};
#else
struct BwdClock {
    __device__ __forceinline__ void start(bool) {}
    __device__ __forceinline__ void lap(int) {}
    __device__ __forceinline__ void flush(int) {}
};
#endif

__global__ void __launch_bounds__(kThrS, 1)
bwd_state_grads_tc_kernel(const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_vt,
                          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                          BwdArgs a)
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
    // fixed order: sa from (row kind, column group) in slots 0..5, then sb,
    // sd2, sgl, sw from the three column groups in slots 6..17
    float* part = reinterpret_cast<float*>(sm + SSUM);
    float* wsum = part + kSumSlots * C;                      // [12 warps][3]
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SBAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SMISC);
    BwdClock clk;
    clk.start(tid == 0);

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_fence_init();
        // every operand by the copy engines: [S | M] entering the chunk and
        // [dS | dM] leaving it (bf16 images of the B operands), dY (the reverse
        // chain's bf16 image), and the dO, Vt, K, Q rows by TMA (rows past the
        // end of the sequence read as zero)
        mbar_arrive_expect_tx(&bar[1], 2 * kStateImgBytes + kDyImgBytes + 4 * 16384);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            bulk_load(sm + SB1 + p * 16384, a.ss_img + chunk * kStateImgBytes + p * 16384, 16384, &bar[1]);
            bulk_load(sm + SB2 + p * 16384, a.dss_img + chunk * kStateImgBytes + p * 16384, 16384, &bar[1]);
        }
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_4d(sm + SA1 + p * 16384, &tm_do, p * 64, h, n * C, b, &bar[1]);
            bulk_load(sm + SA1 + p * 16384 + 8192, a.dy_img + chunk * kDyImgBytes + p * 8192, 8192, &bar[1]);
            tma_load_4d(sm + SA2 + p * 16384, &tm_vt, p * 64, h, n * C, b, &bar[1]);
            tma_load_4d(sm + SA2 + p * 16384 + 8192, &tm_k, p * 64, h, n * C, b, &bar[1]);
            tma_load_4d(sm + SQ + p * 8192, &tm_q, p * 64, h, n * C, b, &bar[1]);
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    for (int i = tid; i < kSumSlots * C; i += kThrS) part[i] = 0.f;
    fence_proxy_async_smem();
    __syncthreads();
    clk.lap(0);
    // the chunk-end scalars' adjoints: <S, dS>, <M, dS>, <M, dM> over the
    // bf16 states the products use (a warp reads 32 consecutive rows of one
    // 8-column group: conflict-free under the swizzle)
    bool ok = mbar_wait(&bar[1], 0);
    float s1 = 0.f, s2 = 0.f, s3 = 0.f;
    if (ok) {
#pragma unroll 2
        for (int i = tid; i < D * 16; i += kThrS) {
            const int row = i & (D - 1), g = i >> 7;
            float sv[8], mv[8], dsv[8], dmv[8];
            unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + SB1 + state_img_off(row, g)), sv);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + SB1 + state_img_off(row + D, g)), mv);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + SB2 + state_img_off(row, g)), dsv);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + SB2 + state_img_off(row + D, g)), dmv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                s1 = fmaf(sv[e], dsv[e], s1);
                s2 = fmaf(mv[e], dsv[e], s2);
                s3 = fmaf(mv[e], dmv[e], s3);
            }
        }
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
    tc_fence_before_sync();
    ok = __syncthreads_and(ok);
    tc_fence_after_sync();
    clk.lap(1);
    const uint32_t tmem = *tmem_slot;

    if (tid == 0 && ok) {
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
        mma_commit(&bar[0]);
    }
    // Epilogue.  Warp w reads TMEM lanes 32 (w % 4) ..; warps w, w + 4, w + 8
    // take columns [0, 48), [48, 96), [96, 128) of each product.  Its
    // coefficients are loaded while the products run; K and Q come from
    // shared memory.
    const int quad = warp & 3, grp = warp >> 2;
    const int c_lo = 48 * grp, c_hi = grp == 2 ? 128 : c_lo + 48;
    const int R = quad * 32 + lane;               // TMEM lane: dO rows 0..63, dY rows 64..127
    const uint32_t tq = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    float* X = reinterpret_cast<float*>(sm + SA1);  // dk of the dY rows, [64][XS], over the operands
    // rows of dq and dk staged for bulk stores (row stride kRowS floats), over
    // the state images
    float* QT = reinterpret_cast<float*>(sm + SB1);
    float* KT = QT + C * kRowS;
    const int r = R & 63, t = n * C + r;
    const bool in = t < a.T;
    const size_t grow = in ? tokrow(a, b, t, h) * D : 0;
    const float abar = expf(a.la[crow + r]), bco = a.bco[crow + r];
    const float al = in ? expf(a.alpha_log[tokrow(a, b, t, h)]) : 1.f;
    const float d2 = r > 0 ? a.bco[crow + r - 1] * al : 0.f;
    const float gl = a.gamma[chunk * C * C + (C - 1) * C + r];
    const float et = in ? a.eta[tokrow(a, b, t, h)] : 0.f;
    const float w = et * expf(a.lm[crow + C - 1] - a.lm[crow + r]);
    // row r of K (rows 64.. of the [Vt; K] tile) and of Q, 16 columns at k0
    auto ld_row16 = [&](uint32_t tile, uint32_t panel, int row, int k0, float* x) {
        const uint32_t o = tile + (k0 >> 6) * panel + sw128_off(row, (k0 & 63) >> 3);
        unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + o), x);
        unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + (o ^ 16)), x + 8);
    };
    ok = __syncthreads_and(ok && mbar_wait(&bar[0], 0));
    tc_fence_after_sync();
    clk.lap(2);
    float sa = 0.f, sb = 0.f, sd2 = 0.f, sgl = 0.f, sw = 0.f;
    if (ok && R >= 64) {
        // dY rows: dk part -Diag(alphabar) P5 + Diag(D2) P6, into the exchange tile
#pragma unroll 1
        for (int k0 = c_lo; k0 < c_hi; k0 += 16) {
            float p5[16], p6[16], kv[16];
            tmem_ld16(tq + k0, p5);
            tmem_ld16(tq + 128 + k0, p6);
            ld_row16(SA2, 16384, 64 + r, k0, kv);
            tmem_wait_ld();
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
    clk.lap(3);
    if (ok && R < 64) {
#pragma unroll 1
        for (int k0 = c_lo; k0 < c_hi; k0 += 16) {
            float p1[16], p2[16], p3[16], p4[16], kv[16], qh[16];
            tmem_ld16(tq + k0, p1);
            tmem_ld16(tq + 128 + k0, p2);
            tmem_ld16(tq + 256 + k0, p3);
            tmem_ld16(tq + 384 + k0, p4);
            ld_row16(SA2, 16384, 64 + r, k0, kv);
            ld_row16(SQ, 8192, r, k0, qh);
            tmem_wait_ld();
            if (in) {  // the TMEM loads above stay warp-uniform
                float dq[16], dk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    qh[e] -= a.dcorr * kv[e];
                    sa = fmaf(qh[e], p1[e], sa);
                    sb = fmaf(-qh[e], p2[e], sb);
                    sgl = fmaf(kv[e], p3[e], sgl);
                    sw = fmaf(-kv[e], p4[e], sw);
                    dq[e] = fmaf(abar, p1[e], -bco * p2[e]);
                    // dk carries -d dq (Qhat = Q - d K) for this part of dq; the
                    // chunk-local kernel adds its parts of both
                    dk[e] = fmaf(-a.dcorr, dq[e], fmaf(gl, p3[e], -w * p4[e]) + X[r * XS + k0 + e]);
                }
#pragma unroll
                for (int e4 = 0; e4 < 4; ++e4) {
                    *reinterpret_cast<float4*>(QT + r * kRowS + k0 + 4 * e4) =
                        make_float4(dq[4 * e4], dq[4 * e4 + 1], dq[4 * e4 + 2], dq[4 * e4 + 3]);
                    *reinterpret_cast<float4*>(KT + r * kRowS + k0 + 4 * e4) =
                        make_float4(dk[4 * e4], dk[4 * e4 + 1], dk[4 * e4 + 2], dk[4 * e4 + 3]);
                }
            }
        }
    }
    // row sums of the three column groups (and, for sa, of both row kinds)
    if (ok && in) {
        const int kind = R < 64 ? 0 : 1;
        part[(3 * kind + grp) * C + r] = sa;
        if (R < 64) {
            part[(6 + grp) * C + r] = sb;
            part[(12 + grp) * C + r] = sgl;
            part[(15 + grp) * C + r] = sw;
        } else {
            part[(9 + grp) * C + r] = sd2;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    // one 512-byte bulk store per row of dq and of dk
    if (ok && tid < 2 * C && n * C + (tid & (C - 1)) < a.T) {
        const int row = tid & (C - 1);
        const size_t g = tokrow(a, b, n * C + row, h) * D;
        bulk_store((tid < C ? a.dq : a.dk) + g, (tid < C ? QT : KT) + row * kRowS, D * 4);
        bulk_commit_group();
    }
    float* rec = a.crec_bw + chunk * kBwdRec;
    clk.lap(4);
    if (tid < C) {
        const float* p0 = part + tid;
        auto sum3 = [&](int s0) { return (p0[s0 * C] + p0[(s0 + 1) * C]) + p0[(s0 + 2) * C]; };
        rec[tid] = sum3(0) + sum3(3);
        rec[C + tid] = sum3(6);
        rec[2 * C + tid] = sum3(9);
        rec[3 * C + tid] = sum3(12);
        rec[4 * C + tid] = sum3(15);
    }
    if (tid < 3) {
        float acc = 0.f;
        for (int w = 0; w < kThrS / 32; ++w) acc += wsum[w * 3 + tid];
        rec[5 * C + tid] = acc;
    }
    if (!ok && tid == 0) {
        atomicOr(a.status + 1, 1u);
        (void)mbar_wait(&bar[1], 0);  // the state copies land before shared memory is released
    }
    bulk_wait_group_read<0>();  // the row stores have read their staging tiles
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
    clk.lap(5);
    clk.flush(0);
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
// Two CTAs share an SM, so that one chunk's serial phases overlap another's:
// stage 2 accumulates over stage 1's TMEM columns (256 in all), its operands
// are written over stage 1's once those have been read, the exchange tile of
// the last epilogue over stage 2's, and Gamma's factor Gp and the adjoint dG
// are kept as packed lower triangles (about 102 KB of shared memory).
constexpr uint32_t LA_QK = 0;        // [Qhat; K]  K-major, 2 K-panels x 128 rows x 128 B (its K rows double as B of K K^T)
constexpr uint32_t LA_DY = 32768;    // [dO; dY]   K-major (stage 1)
constexpr uint32_t LB_V = 65536;     // Vt         K-major, 2 K-panels x 64 rows x 128 B (stage 1)
constexpr uint32_t LA_3 = 32768;     // [dOVG; dPK]          K = 64: 1 panel x 128 rows x 128 B (stage 2)
constexpr uint32_t LA_4 = 49152;     // [dOVG^T | dPKa^T; .] K = 128: 2 panels x 128 rows x 128 B (stage 2;
                                     // rows 64..127 unused)
constexpr uint32_t L_Q = 0;          // fp32 dq part [64][LXS] (once stage 2 has completed)
constexpr uint32_t L_X = 33792;      // fp32 alpha_r dP [64][LXS], then the dk part in place
constexpr int LXS = 132;             // their row stride (floats): rows 16-byte aligned for the
                                     // bulk reductions, float4 accesses of 8 rows conflict-free
constexpr uint32_t L_GP = 81920;     // fp32 Gp, packed lower triangle
constexpr uint32_t L_DG = L_GP + PackedLower::kFloats * 4;   // fp32 dG, packed lower triangle
constexpr uint32_t L_VEC = L_DG + PackedLower::kFloats * 4;  // 12 x 64 floats
constexpr uint32_t L_REC = L_VEC + 3072;  // the chunk record (kBwdRec floats)
constexpr uint32_t L_BAR = L_REC + kBwdRec * 4;  // MMA stage 1, stage 2, operand copies
constexpr uint32_t L_MISC = L_BAR + 32;
constexpr uint32_t L_SMEM = L_MISC + 16 + 1024;
constexpr uint32_t kLocalTmemCols = 256;
static_assert(L_Q + 64 * LXS * 4 <= L_X && L_X + 64 * LXS * 4 <= L_GP, "staging tiles");
static_assert(LA_4 + 32768 <= L_GP && LB_V + 16384 <= L_GP, "operand map");
static_assert(2 * (L_SMEM + 1024) <= 233472, "two CTAs per SM");

__device__ __forceinline__ void st_bf16(uint8_t* p, float x) {
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(x);
}
// byte offset of element (row, k) in a K-major 128-byte-swizzled tile whose
// K-panels (64 elements) are panel_bytes apart
__device__ __forceinline__ uint32_t kmaj_off(int row, int k, uint32_t panel_bytes) {
    return (k >> 6) * panel_bytes + sw128_off(row, (k & 63) >> 3) + (k & 7) * 2;
}

__global__ void __launch_bounds__(kThr, 2)
bwd_local_grads_tc_kernel(const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_qh,
                          const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_vt,
                          BwdArgs a)
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
    const PackedLower at;
    float* Gp = reinterpret_cast<float*>(sm + L_GP);
    float* dG = reinterpret_cast<float*>(sm + L_DG);
    float* recs = reinterpret_cast<float*>(sm + L_REC);
    const BwdVec v = bwd_vec(reinterpret_cast<float*>(sm + L_VEC));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L_MISC);
    BwdClock clk;
    clk.start(tid == 0);

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        mbar_fence_init();
        // operands by the copy engines, K-major with the 128-byte swizzle: dO,
        // K and Vt rows by TMA (zero past the end of the sequence), Qhat rows
        // (bf16, from the chain's operand kernel) by TMA, dY as the reverse
        // chain's bf16 image
        mbar_arrive_expect_tx(&bars[2], 4 * 16384 + kDyImgBytes);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_4d(sm + LA_DY + p * 16384, &tm_do, p * 64, h, n * C, b, &bars[2]);
            bulk_load(sm + LA_DY + p * 16384 + 8192, a.dy_img + chunk * kDyImgBytes + p * 8192, 8192, &bars[2]);
            tma_load_3d(sm + LA_QK + p * 16384, &tm_qh, p * 64, 0, (int)chunk, &bars[2]);
            tma_load_4d(sm + LA_QK + p * 16384 + 8192, &tm_k, p * 64, h, n * C, b, &bars[2]);
            tma_load_4d(sm + LB_V + p * 8192, &tm_vt, p * 64, h, n * C, b, &bars[2]);
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kLocalTmemCols);
        tmem_relinquish();
    }
    // the chunk's coefficient-adjoint record and gate vectors (every global
    // load of a thread before its shared-memory stores)
    {
        static_assert(kBwdRec <= 2 * kThr, "record copy");
        const float* rec_g = a.crec_bw + chunk * kBwdRec;
        const float rc0 = rec_g[tid], rc1 = tid + kThr < kBwdRec ? rec_g[tid + kThr] : 0.f;
        float gal = 0.f, gbe = 0.f, get = 0.f, gla = 0.f, glm = 0.f, gb = 0.f, gmu = 0.f;
        const int tg = n * C + tid;
        const bool gin = tid < C && tg < a.T;
        if (tid < C) {
            const size_t gi = gin ? tokrow(a, b, tg, h) : 0;
            if (gin) {
                gal = a.alpha_log[gi];
                gbe = a.beta[gi];
                get = a.eta[gi];
                gmu = a.mu_log[gi];
            }
            gla = a.la[crow + tid];
            glm = a.lm[crow + tid];
            gb = a.bco[crow + tid];
        }
        recs[tid] = rc0;
        if (tid + kThr < kBwdRec) recs[tid + kThr] = rc1;
        if (tid < C) {
            const int r = tid;
            v.al[r] = gin ? expf(gal) : 1.f;
            v.be[r] = gbe;
            v.et[r] = get;
            v.la[r] = gla;
            v.lm[r] = glm;
            v.b[r] = gb;
            v.da[r] = 0.f;
            v.de[r] = gin ? expf(gmu) : 1.f;  // mu_r, until the coefficient phase
        }
    }
    tc_fence_before_sync();
    __syncthreads();  // the barriers' initialisation and the TMEM address are visible from here
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    clk.lap(0);
    bool ok = __syncthreads_and(mbar_wait(&bars[2], 0));
    clk.lap(1);
    if (tid == 0 && ok) {
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
    // Gamma without eta, by its column recurrence (overlaps the products):
    // Gp_{r,i} = alpha_r Gp_{r-1,i} + beta_r f_r with f_r = mubar_r / mubar_i a
    // running product of mu (held in v.de until the coefficient phase), by
    // blocks of 16 rows on four threads per column (part p owns rows 16p ..).
    // The block's rows map a carry (g, f) entering it to (A g + f G, f F);
    // the maps of the blocks below give each block its carry, and a second
    // pass over the block writes Gp.
    {
        const int i = tid >> 2, part = tid & 3, lo = 16 * part;
        float ar[16], br[16], mr[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            ar[e] = v.al[lo + e];
            br[e] = v.be[lo + e];
            mr[e] = v.de[lo + e];
        }
        float A = 1.f, G = 0.f, F = 1.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int r = lo + e;
            if (r == i) {
                A = 0.f;
                G = br[e];
                F = 1.f;
            } else if (r > i) {
                G = fmaf(ar[e], G, br[e] * mr[e] * F);
                A *= ar[e];
                F *= mr[e];
            }
        }
        const unsigned full = 0xffffffffu;
        const int base = lane & ~3;
        float g = 0.f, f = 1.f;  // the carry entering this block
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            const float aq = __shfl_sync(full, A, base + q);
            const float gq = __shfl_sync(full, G, base + q);
            const float fq = __shfl_sync(full, F, base + q);
            if (q < part) {
                g = fmaf(aq, g, f * gq);
                f *= fq;
            }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int r = lo + e;
            if (r == i) {
                f = 1.f;
                g = br[e];
            } else if (r > i) {
                f *= mr[e];
                g = fmaf(ar[e], g, br[e] * f);
            }
            if (r >= i) Gp[at(r, i)] = g;
        }
    }
    ok = __syncthreads_and(ok && mbar_wait(&bars[0], 0));
    tc_fence_after_sync();
    clk.lap(2);

    // stage-1 epilogue: warp w reads lanes 32 (w % 4) ..; warps w, w + 4 take
    // columns i in [32 half, 32 half + 32), 16 at a time
    const int quad = warp & 3, half = warp >> 2;
    const int R = quad * 32 + lane, r = R & 63;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    float dgm[32];  // dY rows: dA o (P K^T), owed to dG[r - 1][i]
    if (ok) {
        // (rows 64..127 of the second stage-2 operand are left as they are: the
        // product rows they give, lanes 64..127 of the dK part, are not read)
        const float al_r = v.al[r];
        // Gamma's row (r, resp. r - 1 on the dY rows) over this thread's
        // columns, read before any store of the epilogue
        const int gr = R < 64 ? r : r - 1;
        float gam[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int i = 32 * half + e;
            gam[e] = i <= gr ? v.et[i] * Gp[at(gr, i)] : 0.f;
        }
#pragma unroll
        for (int p2 = 0; p2 < 2; ++p2) {
            float x1[16], x2[16];
            tmem_ld16(tq + 32 * half + 16 * p2, x1);        // dO Vt^T  (dY Vt^T on lanes 64..127)
            tmem_ld16(tq + 64 + 32 * half + 16 * p2, x2);   // Qhat K^T (K K^T)
            tmem_wait_ld();
            float row3[16];  // this row's 16 entries of [dOVG; dPK], two 16-byte stores
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int i = 32 * half + 16 * p2 + e;
                const float g = gam[16 * p2 + e];
                if (R < 64) {
                    float ovg = 0.f;
                    if (i <= r) {
                        ovg = x1[e] * g;
                        dG[at(r, i)] = x1[e] * x2[e];
                    }
                    row3[e] = ovg;                                               // row r of [dOVG; .]
                    st_bf16(sm + LA_4 + kmaj_off(i, r, 16384), ovg);             // (dOVG^T)[i][r]
                } else {
                    float pk = 0.f, dm = 0.f;
                    if (i < r) {
                        pk = -x1[e] * g;
                        dm = -x1[e] * al_r * x2[e];
                    }
                    dgm[16 * p2 + e] = dm;
                    row3[e] = pk;                                                // row 64 + r: dPK
                    st_bf16(sm + LA_4 + kmaj_off(i, 64 + r, 16384), pk * al_r); // (Diag(alpha) dPK)^T
                }
            }
            {
                const int k0 = 32 * half + 16 * p2;  // a multiple of 16: two whole 16-byte chunks
                const uint32_t o = kmaj_off(R < 64 ? r : 64 + r, k0, 16384);
                st_bf16x8(sm + LA_3 + o, row3);
                st_bf16x8(sm + LA_3 + (o ^ 16), row3 + 8);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    clk.lap(3);
    if (ok && R >= 64) {  // one writer per entry; every read before the first write
        float cur[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int i = 32 * half + e;
            cur[e] = i < r ? dG[at(r - 1, i)] : 0.f;
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int i = 32 * half + e;
            if (i < r) dG[at(r - 1, i)] = cur[e] + dgm[e];
        }
    }
    if (tid == 0 && ok) {
        constexpr uint32_t id2 = idesc_bf16(128, 128, false, true);
        // [dOVG; dPK] K: B = K (K-dim i = rows 64..127 of the [Qhat; K] tile, N = features)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            mma_bf16(tmem, smem_desc(sbase + LA_3 + ks * 32, 16, 1024, kSw128),
                     smem_desc(sbase + LA_QK + 8192 + ks * 2048, 16384, 1024, kSw128), id2, ks > 0);
        // [dOVG^T | dPKa^T] [Qhat; K]: B = the whole [Qhat; K] tile, K-dim 128 rows
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_bf16(tmem + 128,
                     smem_desc(sbase + LA_4 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128),
                     smem_desc(sbase + LA_QK + ks * 2048, 16384, 1024, kSw128), id2, ks > 0);
        mma_commit(&bars[1]);
    }
    __syncthreads();
    if (tid < C) dG[at(C - 1, tid)] += recs[3 * C + tid];  // Gamma_{C,i} in the state update
    ok = __syncthreads_and(ok && mbar_wait(&bars[1], 0));
    tc_fence_after_sync();
    clk.lap(4);

    // stage-2 epilogue: lanes 64..127 hold dP = dPK K; lanes 0..63 the dQhat
    // and dK parts; warps w, w + 4 take feature columns [64 half, 64 half + 64)
    float* X = reinterpret_cast<float*>(sm + L_X);  // alpha_r dP[r][c], over stage 2's operands
    const int t = n * C + r;
    const bool in = t < a.T;
    const size_t grow = in ? tokrow(a, b, t, h) * D : 0;
    if (ok && R >= 64) {
        float dar = 0.f;
        const float al_r = v.al[r];
#pragma unroll 1
        for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
            float dp[16], kv[16];
            tmem_ld16(tq + c0, dp);
            // row r of K from the [Qhat; K] tile (zero past the end of the sequence)
            unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + LA_QK + kmaj_off(64 + r, c0, 16384)), kv);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(sm + LA_QK + kmaj_off(64 + r, c0 + 8, 16384)), kv + 8);
            tmem_wait_ld();
            if (in) {
#pragma unroll
                for (int e = 0; e < 16; ++e) dar = fmaf(dp[e], kv[e], dar);
            }
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4)
                *reinterpret_cast<float4*>(X + r * LXS + c0 + 4 * e4) =
                    make_float4(al_r * dp[4 * e4], al_r * dp[4 * e4 + 1], al_r * dp[4 * e4 + 2],
                                al_r * dp[4 * e4 + 3]);
        }
        atomicAdd(v.da + r, dar);  // two addends onto 0: the same sum in either order
    }
    __syncthreads();
    clk.lap(5);
    if (ok && R < 64) {
        // this kernel's parts of dq and dk, staged by rows (dk over the row of
        // X it has read) and added to the state products' by bulk reductions
        float* QL = reinterpret_cast<float*>(sm + L_Q);
#pragma unroll 1
        for (int c0 = 64 * half; c0 < 64 * half + 64; c0 += 16) {
            float dqb[16], dkb[16];
            tmem_ld16(tq + c0, dqb);
            tmem_ld16(tq + 128 + c0, dkb);
            float4 xr[4];
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) xr[e4] = *reinterpret_cast<const float4*>(X + r * LXS + c0 + 4 * e4);
            tmem_wait_ld();
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
                const float* q4 = dqb + 4 * e4;
                const float* k4 = dkb + 4 * e4;
                *reinterpret_cast<float4*>(QL + r * LXS + c0 + 4 * e4) = make_float4(q4[0], q4[1], q4[2], q4[3]);
                *reinterpret_cast<float4*>(X + r * LXS + c0 + 4 * e4) =
                    make_float4(k4[0] + xr[e4].x - a.dcorr * q4[0], k4[1] + xr[e4].y - a.dcorr * q4[1],
                                k4[2] + xr[e4].z - a.dcorr * q4[2], k4[3] + xr[e4].w - a.dcorr * q4[3]);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kLocalTmemCols);
    }
    // one 512-byte bulk reduction per row of dq and of dk (one addition per element)
    if (ok && tid < 2 * C && n * C + (tid & (C - 1)) < a.T) {
        const int row = tid & (C - 1);
        const size_t g = tokrow(a, b, n * C + row, h) * D;
        bulk_reduce_add_f32((tid < C ? a.dq : a.dk) + g, sm + (tid < C ? L_Q : L_X) + row * LXS * 4, D * 4);
        bulk_commit_group();
    }
    clk.lap(6);
    if (!ok) {
        if (tid == 0) {
            atomicOr(a.status + 1, 1u);
            (void)mbar_wait(&bars[2], 0);  // the operand copies land before shared memory is released
        }
        return;
    }
    struct Sub {  // the coefficient phase's laps in slots 7 ..
        BwdClock* c;
        __device__ __forceinline__ void lap(int k) { c->lap(7 + k); }
    } sub{&clk};
    bwd_coeff_phase<PackedLower>(a, recs, v, dG, Gp, recs, tid, n, b, h, true, kThr, &sub);
    bulk_wait_group_read<0>();  // the row reductions have read their staging tiles
    clk.flush(1);
}

// ---------------------------------------------------------------------------
// T = (I + A)^{-1} with A = (P K^T) o Gamma-, and Att = (Qhat K^T) o Gamma, per
// chunk (bf16, d = 128): the forward pass's intra-chunk product on tcgen05,
//   G = [K; Qhat] [K; Qhat]^T   (M 128, N 128, K 128; lane i < 64: k_i.k_r in
//                                columns r, k_i.qhat_r in columns 64 + r)
// then thread i forms column i of A and Att from lane i, and T follows by
// 16 x 16 blocks (inverse_blocked).  Qhat is rounded to bf16 as in the
// forward pass.
constexpr uint32_t Q_KQ = 0;                 // [K; Qhat] K-major: 2 panels x 128 rows x 128 B
constexpr uint32_t Q_A = 32768;              // fp32 A [64][LDF], then B_ik in place
constexpr uint32_t Q_T = Q_A + 64 * LDF * 4; // fp32 Gamma [64][LDF], then T
constexpr uint32_t Q_AL = Q_T + 64 * LDF * 4; // alpha_r
constexpr uint32_t Q_BAR = Q_AL + 256;
constexpr uint32_t Q_MISC = Q_BAR + 16;
constexpr uint32_t Q_SMEM = Q_MISC + 16 + 1024;

// acc0, acc1 += rows r0, r0 + 1 of the 16 x 16 block at X times columns
// c0 .. c0 + 3 of the block at Y (row stride LDF).
__device__ __forceinline__ void blk_2x4(const float* X, const float* Y, int r0, int c0, float4& acc0,
                                        float4& acc1) {
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
        const float4 a0 = lds4(X + r0 * LDF + 4 * k4), a1 = lds4(X + (r0 + 1) * LDF + 4 * k4);
        const float x0[4] = {a0.x, a0.y, a0.z, a0.w}, x1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float4 y = lds4(Y + (4 * k4 + e) * LDF + c0);
            acc0.x = fmaf(x0[e], y.x, acc0.x); acc0.y = fmaf(x0[e], y.y, acc0.y);
            acc0.z = fmaf(x0[e], y.z, acc0.z); acc0.w = fmaf(x0[e], y.w, acc0.w);
            acc1.x = fmaf(x1[e], y.x, acc1.x); acc1.y = fmaf(x1[e], y.y, acc1.y);
            acc1.z = fmaf(x1[e], y.z, acc1.z); acc1.w = fmaf(x1[e], y.w, acc1.w);
        }
    }
}

// T = (I + A)^{-1} for a strictly lower 64 x 64 A (row stride LDF) into T (same
// stride, row-major), by 16 x 16 blocks: the diagonal blocks by forward
// substitution (one column per thread), B_ik = -T_ii A_ik in place of A_ik,
// then T_ij = sum_{k=j}^{i-1} B_ik T_kj level by level (i - j = 1, 2, 3).
// Every thread of the 256-thread CTA calls it; it synchronises.
__device__ void inverse_blocked(float* A, float* T, int tid)
{
    if (tid < C) {
        const int o = 16 * (tid >> 4), cl = tid & 15;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) t[r] = (r == cl) ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
            float av[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float4 v4 = lds4(A + (o + r) * LDF + o + 4 * q4);
                av[4 * q4] = v4.x; av[4 * q4 + 1] = v4.y; av[4 * q4 + 2] = v4.z; av[4 * q4 + 3] = v4.w;
            }
            float acc0 = 0.f, acc1 = 0.f;  // two partial sums: a shorter dependency chain
#pragma unroll
            for (int kk = 0; kk < r; kk += 2) {
                acc0 = fmaf(av[kk], t[kk], acc0);
                if (kk + 1 < r) acc1 = fmaf(av[kk + 1], t[kk + 1], acc1);
            }
            if (r > cl) t[r] = -(acc0 + acc1);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) T[(o + r) * LDF + o + cl] = t[r];
    } else {
        // the six blocks above the diagonal are zero
        for (int idx = tid - C; idx < 6 * 256; idx += kThr - C) {
            const int bidx = idx >> 8, w = idx & 255;
            const int bi = bidx < 3 ? 0 : (bidx < 5 ? 1 : 2);
            const int bj = bidx < 3 ? bidx + 1 : (bidx < 5 ? bidx - 1 : 3);
            T[(16 * bi + (w >> 4)) * LDF + 16 * bj + (w & 15)] = 0.f;
        }
    }
    __syncthreads();
    // B_ik = -T_ii A_ik, blocks (i, k) = (1,0) (2,0) (2,1) (3,0) (3,1) (3,2): 32 tiles of 2 x 4 each
    float4 r0v = make_float4(0.f, 0.f, 0.f, 0.f), r1v = r0v;
    int where = -1;
    if (tid < 192) {
        const int bidx = tid >> 5;
        const int bi = bidx < 1 ? 1 : (bidx < 3 ? 2 : 3);
        const int bk = bidx < 1 ? 0 : (bidx < 3 ? bidx - 1 : bidx - 3);
        const int r0 = 2 * ((tid >> 2) & 7), c0 = 4 * (tid & 3);
        blk_2x4(T + 16 * bi * LDF + 16 * bi, A + 16 * bi * LDF + 16 * bk, r0, c0, r0v, r1v);
        where = (16 * bi + r0) * LDF + 16 * bk + c0;
    }
    __syncthreads();  // every read of A_ik precedes its overwrite
    if (where >= 0) {
        *reinterpret_cast<float4*>(A + where) = make_float4(-r0v.x, -r0v.y, -r0v.z, -r0v.w);
        *reinterpret_cast<float4*>(A + where + LDF) = make_float4(-r1v.x, -r1v.y, -r1v.z, -r1v.w);
    }
    __syncthreads();
    for (int L = 1; L < 4; ++L) {
        if (tid < (4 - L) * 32) {
            const int i = L + (tid >> 5), j = i - L;
            const int r0 = 2 * ((tid >> 2) & 7), c0 = 4 * (tid & 3);
            float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
            for (int kb = j; kb < i; ++kb)
                blk_2x4(A + 16 * i * LDF + 16 * kb, T + 16 * kb * LDF + 16 * j, r0, c0, acc0, acc1);
            float* t = T + (16 * i + r0) * LDF + 16 * j + c0;
            *reinterpret_cast<float4*>(t) = acc0;
            *reinterpret_cast<float4*>(t + LDF) = acc1;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThr)
bwd_prep_tc_kernel(BwdArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int n = blockIdx.x % a.NT;
    const long long bh = blockIdx.x / a.NT;
    const int b = (int)(bh / a.H), h = (int)(bh % a.H);
    const size_t chunk = blockIdx.x;
    float* As = reinterpret_cast<float*>(sm + Q_A);
    float* Ts = reinterpret_cast<float*>(sm + Q_T);
    float* alpha_s = reinterpret_cast<float*>(sm + Q_AL);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Q_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Q_MISC);
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    // K, Q rows and Gamma: every global load of a thread before its stores
    {
        constexpr int PER = C * 16 / kThr;   // 16-byte pieces of K (and of Q) per thread
        constexpr int PG = C * C / 4 / kThr;  // float4 of Gamma per thread
        uint4 rk[PER], rq[PER];
        float4 rg[PG];
        const float* G = a.gamma + chunk * C * C;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int i = tid + kThr * u, r = i >> 4, c16 = i & 15, t = n * C + r;
            rk[u] = rq[u] = make_uint4(0, 0, 0, 0);
            if (t < a.T) {
                const size_t g = tokrow(a, b, t, h) * D + c16 * 8;
                rk[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.k) + g);
                rq[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + g);
            }
        }
#pragma unroll
        for (int u = 0; u < PG; ++u) rg[u] = __ldg(reinterpret_cast<const float4*>(G) + tid + kThr * u);
        float al = 1.f;
        if (tid < C && n * C + tid < a.T) al = expf(a.alpha_log[tokrow(a, b, n * C + tid, h)]);
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int i = tid + kThr * u, r = i >> 4, c16 = i & 15;
            const uint32_t off = (c16 >> 3) * 16384 + sw128_off(r, c16 & 7);
            float k[8], q[8];
            unpack_bf16x8(rk[u], k);
            unpack_bf16x8(rq[u], q);
#pragma unroll
            for (int e = 0; e < 8; ++e) q[e] -= a.dcorr * k[e];
            *reinterpret_cast<uint4*>(sm + Q_KQ + off) = rk[u];
            *reinterpret_cast<uint4*>(sm + Q_KQ + off + 8192) = bf16x8(q);  // rows 64..127
        }
#pragma unroll
        for (int u = 0; u < PG; ++u) {
            const int idx = (tid + kThr * u) * 4, r = idx / C, c = idx % C;
            *reinterpret_cast<float4*>(Ts + r * LDF + c) = rg[u];
        }
        if (tid < C) alpha_s[tid] = al;
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        constexpr uint32_t id = idesc_bf16(128, 128, false, false);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint64_t ad = smem_desc(sbase + Q_KQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128);
            mma_bf16(tmem, ad, ad, id, ks > 0);
        }
        mma_commit(bar);
    }
    const bool ok = __syncthreads_and(mbar_wait(bar, 0));
    tc_fence_after_sync();
    __nv_bfloat16* att = reinterpret_cast<__nv_bfloat16*>(a.att) + chunk * C * C;  // bf16 on this path
    if (ok && tid < C) {
        // column i of A and of Att from TMEM lane i (warps 0, 1: lanes 0..63)
        const int i = tid;
        const uint32_t lane_sel = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll 1
        for (int r16 = 0; r16 < C; r16 += 16) {
            float kk[16], kh[16];
            tmem_ld16(tmem + lane_sel + r16, kk);      // k_i . k_r
            tmem_ld16(tmem + lane_sel + C + r16, kh);  // k_i . qhat_r
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int r = r16 + e;
                const float av = i < r ? alpha_s[r] * kk[e] * Ts[(r - 1) * LDF + i] : 0.f;
                const float tv = i <= r ? kh[e] * Ts[r * LDF + i] : 0.f;
                As[r * LDF + i] = av;
                att[r * C + i] = __float2bfloat16_rn(tv);
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();  // A complete; Gamma read
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 128);
    }
    if (!ok) {
        if (tid == 0) atomicOr(a.status + 1, 1u);
        return;
    }
    inverse_blocked(As, Ts, tid);
    // T in bf16, row-major: the chain-operand kernel's input and the reverse
    // chain's MN-major A of T^T dVtilde
    uint2* Tm = reinterpret_cast<uint2*>(a.bc_tt + chunk * C * C);
    for (int idx = tid; idx < C * C / 4; idx += kThr) {
        const float4 t4 = lds4(Ts + (idx >> 4) * LDF + 4 * (idx & 15));
        const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
        Tm[idx] = bf16x4(tv);
    }
}

// ---------------------------------------------------------------------------
// The chunk-only operands of the tensor-core reverse chain (bf16, d = 128):
//   U  = [-K^T Diag(alphabar) T^T ; K^T Diag(D2) T^T]   bf16 [256][64]  (A of U dVtilde)
//   T  row-major                                        bf16 [64][64]   (T^T as the MN-major A
//                                                                        of T^T dVtilde = dv)
//   P  = Att^T dO     fp32, slice-major [D/32][64][32]  (dVtilde's chain-free part)
//   Qhat rows (bf16 [64][128]) and Diag(alphabar) dO, -Diag(b) dO by 32-column
//   slice (bf16, the reverse chain's shared-memory image of its B operands)
//   record: Gamma_{C,r} (64), w_r (64), then alphabar_C, b_C, mubar_C at 192..194
// plus the increments of the state rebuild, D_S = K^T Diag(Gamma_C) Vtilde and
// D_M = K^T Diag(w) Vtilde, which turn the rebuild into an elementwise scan
// over the chunks.  Products (K^T and Att^T are the MN-major forms of K's and
// Att's rows, so nothing is transposed on the way into shared memory):
//   U = K^T [Diag(-alphabar) T^T | Diag(D2) T^T]                M 128, N 64 + 64
//   P = Att^T dO                                                 M 64 (of 128), N 128
//   D = K^T [Diag(Gamma_C) Vtilde | Diag(w) Vtilde]             M 128, N 128 + 128 (second round,
//                                                                over the first round's columns)
// E = Qhat^T Diag(alphabar) dO and F = Qhat^T Diag(b) dO are formed in the
// reverse chain itself (by the MMA lane while it waits for each chunk's
// dVtilde), from Qhat and the scaled dO slices written here.  Two CTAs share
// an SM (256 TMEM columns, about 100 KB of shared memory each).
constexpr uint32_t PA_KT = 0;        // K^T as an MN-major A: K's rows [64 r][128 i], 2 M-panels
                                     // of 64 rows x 128 B, 16 KB
constexpr uint32_t PA_AT = 16384;    // Att^T as an MN-major A: Att's rows [64 r][64 i] (M-panel 0;
                                     // the product rows of panel 1 are not read)
constexpr uint32_t PB_O = 32768;     // dO      [64 r][128 j]  MN-major: 2 N-panels x 64 rows
constexpr uint32_t PB_VG = 49152;    // Diag(Gamma_C) Vtilde
constexpr uint32_t PB_VW = 65536;    // Diag(w) Vtilde
constexpr uint32_t PB_TS = 81920;    // -alphabar_{r2} T[r][r2]  [64 r][64 r2]  K-major, 8 KB
constexpr uint32_t PB_TM = 90112;    //  D2_{r2} T[r][r2]
constexpr uint32_t P_VEC = 98304;    // alphabar, b, D2, Gamma_C, w
constexpr uint32_t P_BAR = P_VEC + 1280;
constexpr uint32_t P_MISC = P_BAR + 16;
constexpr uint32_t P_SMEM = P_MISC + 16 + 1024;
static_assert(2 * (P_SMEM + 1024) <= 233472, "two CTAs per SM");

// byte offset of element (row, col) of an MN-major tile with 64-element
// column panels of `rows` rows (128-byte swizzle)
__device__ __forceinline__ uint32_t mn_off(int row, int col, int rows) {
    return (col >> 6) * rows * 128 + sw128_off(row, (col & 63) >> 3) + (col & 7) * 2;
}

__global__ void __launch_bounds__(kThr, 2)
bwd_chain_prep_tc_kernel(BwdArgs a)
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
    float* v_ab = reinterpret_cast<float*>(sm + P_VEC);
    float* v_b = v_ab + C;
    float* v_d2 = v_b + C;
    float* v_g = v_d2 + C;
    float* v_w = v_g + C;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P_MISC);
    float* rec = a.bc_rec + chunk * 256;
    BwdClock clk;
    clk.start(tid == 0);

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    // one round of global loads: this position's gate values (threads < C)
    // and the token tiles (64 rows x 16 groups of 8, kept as packed bf16)
    constexpr int U8 = C * 16 / kThr;  // 4
    uint4 kx[U8], qx[U8], ox[U8], vx[U8];
    float g_la = 0.f, g_al = 0.f, g_gl = 0.f, g_et = 0.f, g_lm = 0.f, g_b = 0.f, g_bp = 0.f;
    float g_laC = 0.f, g_lmC = 0.f;
    const bool gin = tid < C && n * C + tid < a.T;
    if (tid < C) {
        const int r = tid;
        g_la = a.la[crow + r];
        if (gin) {
            g_al = a.alpha_log[tokrow(a, b, n * C + r, h)];
            g_et = a.eta[tokrow(a, b, n * C + r, h)];
        }
        g_gl = a.gamma[chunk * C * C + (C - 1) * C + r];
        g_lm = a.lm[crow + r];
        g_lmC = a.lm[crow + C - 1];
        g_laC = a.la[crow + C - 1];
        g_b = a.bco[crow + r];
        g_bp = r > 0 ? a.bco[crow + r - 1] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < U8; ++u) {
        const int i = tid + kThr * u, r = i >> 4, c8 = (i & 15) * 8, t = n * C + r;
        kx[u] = qx[u] = ox[u] = vx[u] = make_uint4(0, 0, 0, 0);
        if (t < a.T) {
            const size_t g = tokrow(a, b, t, h) * D + c8;
            kx[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.k) + g);
            qx[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + g);
            ox[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.dout) + g);
            vx[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.vt) + g);
        }
    }
    if (tid < C) {
        const int r = tid;
        const float al = gin ? expf(g_al) : 1.f;
        const float w = g_et * expf(g_lmC - g_lm);
        v_ab[r] = expf(g_la);
        v_b[r] = g_b;
        v_d2[r] = r > 0 ? g_bp * al : 0.f;
        v_g[r] = g_gl;
        v_w[r] = w;
        rec[r] = g_gl;
        rec[C + r] = w;
        if (r == 0) {
            rec[3 * C] = expf(g_laC);
            rec[3 * C + 1] = a.bco[crow + C - 1];
            rec[3 * C + 2] = expf(g_lmC);
        }
    }
    __syncthreads();
    clk.lap(0);
    // the token tiles into shared memory (nothing transposed) and the chain's
    // per-chunk copies to global memory
    {
#pragma unroll
        for (int u = 0; u < U8; ++u) {
            const int i = tid + kThr * u, r = i >> 4, c8 = (i & 15) * 8;
            const float ab = v_ab[r], bb = v_b[r], gl = v_g[r], w = v_w[r];
            float kf[8], qf[8], of[8], vf[8];
            unpack_bf16x8(kx[u], kf);
            unpack_bf16x8(qx[u], qf);
            unpack_bf16x8(ox[u], of);
            unpack_bf16x8(vx[u], vf);
            float qh[8], oa[8], ob[8], vg[8], vw[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                qh[e] = qf[e] - a.dcorr * kf[e];
                oa[e] = ab * of[e];
                ob[e] = -bb * of[e];
                vg[e] = gl * vf[e];
                vw[e] = w * vf[e];
            }
            const uint32_t o = mn_off(r, c8, 64);
            *reinterpret_cast<uint4*>(sm + PA_KT + o) = kx[u];
            *reinterpret_cast<uint4*>(sm + PB_O + o) = ox[u];
            st_bf16x8(sm + PB_VG + o, vg);
            st_bf16x8(sm + PB_VW + o, vw);
            // Qhat rows, and the reverse chain's E / F operands Diag(alphabar) dO and
            // -Diag(b) dO by 32-column slice, each in the chain's shared-memory image
            *reinterpret_cast<uint4*>(a.bc_qh + (chunk * C + r) * D + c8) = bf16x8(qh);
            uint8_t* eo = a.bc_eo + (chunk * (D / 32) + (c8 >> 5)) * 8192 + sw64_off(r, (c8 & 31) >> 3);
            *reinterpret_cast<uint4*>(eo) = bf16x8(oa);
            *reinterpret_cast<uint4*>(eo + 4096) = bf16x8(ob);
        }
    }
    // T and Att (bf16, row-major, from the prep kernel): the scaled T tiles
    // (K-major) and Att's rows (the MN-major form of Att^T)
    {
        constexpr int U4 = C * C / 4 / kThr;  // 4
        uint2 tx[U4], ax[U4];
        const __nv_bfloat16* Tg = a.bc_tt + chunk * C * C;
        const __nv_bfloat16* Ag = reinterpret_cast<const __nv_bfloat16*>(a.att) + chunk * C * C;
#pragma unroll
        for (int u = 0; u < U4; ++u) {
            const int idx = (tid + kThr * u) * 4;
            tx[u] = *reinterpret_cast<const uint2*>(Tg + idx);
            ax[u] = *reinterpret_cast<const uint2*>(Ag + idx);
        }
#pragma unroll
        for (int u = 0; u < U4; ++u) {
            const int idx = (tid + kThr * u) * 4, r = idx / C, r2 = idx % C;
            float tv[4], av[4];
            unpack_bf16x4(tx[u], tv);
            unpack_bf16x4(ax[u], av);
            float ts[4], tm[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ts[e] = -v_ab[r2 + e] * tv[e];
                tm[e] = v_d2[r2 + e] * tv[e];
            }
            // four consecutive elements of row r: 8 bytes in each tile
            *reinterpret_cast<uint2*>(sm + PB_TS + kmaj_off(r, r2, 8192)) = bf16x4(ts);
            *reinterpret_cast<uint2*>(sm + PB_TM + kmaj_off(r, r2, 8192)) = bf16x4(tm);
            *reinterpret_cast<uint2*>(sm + PA_AT + kmaj_off(r, r2, 8192)) = ax[u];
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    clk.lap(1);
    if (tid == 0) {
        constexpr uint32_t idmn = idesc_bf16(128, 128, true, true);   // A, B MN-major
        constexpr uint32_t idk = idesc_bf16(128, 64, true, false);    // A MN-major, B K-major
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ak = smem_desc(sbase + PA_KT + ks * 2048, 8192, 1024, kSw128);
            const uint64_t aa = smem_desc(sbase + PA_AT + ks * 2048, 8192, 1024, kSw128);
            mma_bf16(tmem, ak, smem_desc(sbase + PB_TS + ks * 32, 16, 1024, kSw128), idk, ks > 0);
            mma_bf16(tmem + 64, ak, smem_desc(sbase + PB_TM + ks * 32, 16, 1024, kSw128), idk, ks > 0);
            mma_bf16(tmem + 128, aa, smem_desc(sbase + PB_O + ks * 2048, 8192, 1024, kSw128), idmn, ks > 0);
        }
        mma_commit(&bars[0]);
    }
    bool ok = __syncthreads_and(mbar_wait(&bars[0], 0));
    tc_fence_after_sync();
    clk.lap(2);
    const int quad = warp & 3, half = warp >> 2;
    const int R = quad * 32 + lane;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    if (ok) {
        // U: row i = R of the S half (half 0) or of the M half (half 1)
        {
            uint4* Uo = reinterpret_cast<uint4*>(a.bc_u + chunk * 256 * 64 + (size_t)(128 * half + R) * 64);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float u16[16];
                tmem_ld16(tq + 64 * half + 16 * g, u16);
                tmem_wait_ld();
                Uo[2 * g] = bf16x8(u16);
                Uo[2 * g + 1] = bf16x8(u16 + 8);
            }
        }
        // P = Att^T dO: rows r = R < 64, columns [64 half, 64 half + 64), by 32-column slice
        if (R < 64) {
            __nv_bfloat16* Po = a.bc_p + chunk * C * D;
#pragma unroll 1
            for (int k0 = 64 * half; k0 < 64 * half + 64; k0 += 16) {
                float p16[16];
                tmem_ld16(tq + 128 + k0, p16);
                tmem_wait_ld();
                const int sl = k0 >> 5, jj = k0 & 31;
                uint4* dst = reinterpret_cast<uint4*>(Po + (sl * C + R) * 32 + jj);
                dst[0] = bf16x8(p16);
                dst[1] = bf16x8(p16 + 8);
            }
        }  // (R < 64 is warp-uniform: quadrants 0, 1)
    }
    // second round: the rebuild increments, over the first round's columns
    // (every TMEM read above has completed: tmem_wait_ld, then the barrier)
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (tid == 0 && ok) {
        constexpr uint32_t idmn = idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint64_t ak = smem_desc(sbase + PA_KT + ks * 2048, 8192, 1024, kSw128);
            mma_bf16(tmem, ak, smem_desc(sbase + PB_VG + ks * 2048, 8192, 1024, kSw128), idmn, ks > 0);
            mma_bf16(tmem + 128, ak, smem_desc(sbase + PB_VW + ks * 2048, 8192, 1024, kSw128), idmn, ks > 0);
        }
        mma_commit(&bars[1]);
    }
    ok = __syncthreads_and(ok && mbar_wait(&bars[1], 0));
    tc_fence_after_sync();
    clk.lap(3);
    if (ok) {
        __nv_bfloat16* Do = a.bc_d + (chunk * 2) * D * D;  // chain order
#pragma unroll 1
        for (int k0 = 64 * half; k0 < 64 * half + 64; k0 += 16) {
            float s16[16], m16[16];
            tmem_ld16(tq + k0, s16);
            tmem_ld16(tq + 128 + k0, m16);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int o = chain_off(R, k0 + 4 * q);
                *reinterpret_cast<uint2*>(Do + o) = bf16x4(s16 + 4 * q);
                *reinterpret_cast<uint2*>(Do + D * D + o) = bf16x4(m16 + 4 * q);
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 256);
    }
    clk.lap(4);
    clk.flush(2);
    if (!ok && tid == 0) atomicOr(a.status + 1, 1u);
}

// The states entering every chunk by the elementwise recurrence
// S <- alphabar_C S - b_C M + D_S, M <- mubar_C M - D_M, in fp32 registers;
// each chunk's entering pair is stored as the bf16 image the state products
// copy in (state_img_off).  A thread owns 8 columns of one row of a head's S
// and M; eight consecutive lanes take the eight 16-byte pieces of one row of
// a 64-column panel, so a warp's stores fill four whole 128-byte lines (its
// loads of the increments, in chain order, are eight runs of 64 bytes).  Each
// thread keeps the next two chunks' increments in flight.
__global__ void __launch_bounds__(256)
bwd_state_scan_kernel(const float* __restrict__ S0, const float* __restrict__ M0,
                      const __nv_bfloat16* __restrict__ dinc, const float* __restrict__ rec,
                      uint8_t* __restrict__ img, int NT, long long heads)
{
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    constexpr int per = D * (D / 8);
    if (gid >= heads * per) return;
    const long long bh = gid / per;
    const int rem = (int)(gid % per), i = (rem & 1023) >> 3, g = (rem >> 10) * 8 + (rem & 7);
    float s[8], m[8];
    const size_t r0 = (size_t)bh * D * D + (size_t)i * D + 8 * g;  // S0, M0 are row-major
#pragma unroll
    for (int h4 = 0; h4 < 2; ++h4) {
        const float4 x = S0 ? *reinterpret_cast<const float4*>(S0 + r0 + 4 * h4) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 y = M0 ? *reinterpret_cast<const float4*>(M0 + r0 + 4 * h4) : make_float4(0.f, 0.f, 0.f, 0.f);
        s[4 * h4] = x.x; s[4 * h4 + 1] = x.y; s[4 * h4 + 2] = x.z; s[4 * h4 + 3] = x.w;
        m[4 * h4] = y.x; m[4 * h4 + 1] = y.y; m[4 * h4 + 2] = y.z; m[4 * h4 + 3] = y.w;
    }
    const int o0 = chain_off(i, 8 * g), o1 = chain_off(i, 8 * g + 4);
    const uint32_t ps = state_img_off(i, g), pm = state_img_off(i + D, g);
    struct Step { uint2 ds0, ds1, dm0, dm1; float aC, bC, mC; };
    auto load = [&](int nn) {
        Step st;
        if (nn < NT) {
            const size_t chunk = (size_t)bh * NT + nn;
            const __nv_bfloat16* dn = dinc + chunk * 2 * D * D;
            st.ds0 = __ldg(reinterpret_cast<const uint2*>(dn + o0));
            st.ds1 = __ldg(reinterpret_cast<const uint2*>(dn + o1));
            st.dm0 = __ldg(reinterpret_cast<const uint2*>(dn + D * D + o0));
            st.dm1 = __ldg(reinterpret_cast<const uint2*>(dn + D * D + o1));
            st.aC = __ldg(rec + chunk * 256 + 3 * C);
            st.bC = __ldg(rec + chunk * 256 + 3 * C + 1);
            st.mC = __ldg(rec + chunk * 256 + 3 * C + 2);
        }
        return st;
    };
    Step n1 = load(0), n2 = load(1);
    for (int nn = 0; nn < NT; ++nn) {
        const Step cu = n1;
        n1 = n2;
        n2 = load(nn + 2);
        uint8_t* im = img + ((size_t)bh * NT + nn) * kStateImgBytes;
        *reinterpret_cast<uint4*>(im + ps) = bf16x8(s);
        *reinterpret_cast<uint4*>(im + pm) = bf16x8(m);
        float dsv[8], dmv[8];
        unpack_bf16x4(cu.ds0, dsv);
        unpack_bf16x4(cu.ds1, dsv + 4);
        unpack_bf16x4(cu.dm0, dmv);
        unpack_bf16x4(cu.dm1, dmv + 4);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float sn = fmaf(cu.aC, s[e], fmaf(-cu.bC, m[e], dsv[e]));
            m[e] = fmaf(cu.mC, m[e], -dmv[e]);
            s[e] = sn;
        }
    }
}

}  // namespace


#ifdef MDN_PHASE_CLOCKS
// Diagnostic builds: where the per-phase cycle sums go (3 x kBwdClkSlots
// floats: state products, local products, chain operands), or null.
extern "C" int mdn_diag_bwd_clock(float* p)
{
    return cudaMemcpyToSymbol(g_bwd_clk, &p, sizeof(p)) == cudaSuccess ? 0 : 1;
}
#endif

cudaError_t launch_bwd_state_grads_tc(const BwdArgs& a, cudaStream_t s)
{
    if (a.D != D) return cudaErrorNotSupported;
    const long long chunks = (long long)a.B * a.H * a.NT;
    cudaError_t e = cudaFuncSetAttribute(bwd_state_grads_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    CUtensorMap mdo, mvt, mk, mq;
    if (!make_token_map(&mdo, a.dout, a.B, a.T, a.H, 64, true) ||
        !make_token_map(&mvt, a.vt, a.B, a.T, a.H, 64, true) ||
        !make_token_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_token_map(&mq, a.q, a.B, a.T, a.H, 64, true))
        return cudaErrorInvalidValue;
    ProfScope ps(kBwdStateGrads, s);
    bwd_state_grads_tc_kernel<<<(unsigned)chunks, kThrS, SMEM_BYTES, s>>>(mdo, mvt, mk, mq, a);
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
    if (e == cudaSuccess)  // two CTAs per SM need the larger carve-out
        e = cudaFuncSetAttribute(bwd_local_grads_tc_kernel,
                                 cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    CUtensorMap mdo, mqh, mk, mvt;
    if (!make_token_map(&mdo, a.dout, a.B, a.T, a.H, 64, true) ||
        !make_chunk_map(&mqh, a.bc_qh, chunks, C, D, C) ||
        !make_token_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_token_map(&mvt, a.vt, a.B, a.T, a.H, 64, true))
        return cudaErrorInvalidValue;
    ProfScope ps(kBwdLocal, s);
    bwd_local_grads_tc_kernel<<<(unsigned)chunks, kThr, L_SMEM, s>>>(mdo, mqh, mk, mvt, a);
    return cudaGetLastError();
}

}  // namespace mdn

namespace mdn {

cudaError_t launch_bwd_prep_tc(const BwdArgs& a, cudaStream_t s)
{
    if (a.D != D) return cudaErrorNotSupported;
    const long long chunks = (long long)a.B * a.H * a.NT;
    cudaError_t e = cudaFuncSetAttribute(bwd_prep_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Q_SMEM);
    if (e != cudaSuccess) return e;
    ProfScope ps(kBwdPrep, s);
    bwd_prep_tc_kernel<<<(unsigned)chunks, kThr, Q_SMEM, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_bwd_chain_prep_tc(const BwdArgs& a, cudaStream_t s)
{
    if (a.D != D) return cudaErrorNotSupported;
    const long long chunks = (long long)a.B * a.H * a.NT;
    cudaError_t e = cudaFuncSetAttribute(bwd_chain_prep_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)P_SMEM);
    if (e == cudaSuccess)  // two CTAs per SM need the larger carve-out
        e = cudaFuncSetAttribute(bwd_chain_prep_tc_kernel,
                                 cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    {
        ProfScope ps(kBwdChainPrep, s);
        bwd_chain_prep_tc_kernel<<<(unsigned)chunks, kThr, P_SMEM, s>>>(a);
    }
    if ((e = cudaGetLastError())) return e;
    const long long heads = (long long)a.B * a.H;
    const long long threads = heads * D * (D / 8);
    ProfScope ps(kBwdStates, s);
    bwd_state_scan_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
        a.S0, a.M0, a.bc_d, a.bc_rec, a.ss_img, a.NT, heads);
    return cudaGetLastError();
}

}  // namespace mdn
