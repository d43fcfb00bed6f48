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
// Vtilde are independent) and walks the chunks in order.  The intra-chunk
// kernel has prepared Qhat, [T; Att T] and A2T = [K^T Diag(Gamma_C) T;
// -K^T Diag(w) T] for every chunk.  Per chunk n:
//     A1 = [K; Qhat] [S | M]                      (M=128, N=64, K=128)
//     Y  = V - (D1 KS - D2 KM);   Oi = Diag(alphabar) QhatS - Diag(b) QhatM
//     A2 = [A2T_S; A2T_M] Y   (two M=128, N=32, K=64)
//     S, M <- (alphabar_C S - b_C M, mubar_C M) + A2
//     A3 = [T; Att T] Y  (M=128, N=32, K=64):  Vtilde = A3[0:64],  o = Oi + A3[64:128]
// The critical path of a chunk is A1 -> Y -> A2 -> state; the stores of chunk
// n-1 run while A1 of chunk n executes.  Eight warps: warp w owns TMEM lanes
// 32(w%4).. and columns 16(w/4).. of the CTA's 32, so a thread holds 16
// columns of one row of S and M in fp32 registers; their bf16 copy in shared
// memory is the B operand of A1.  Loads are double-buffered in two groups by
// lifetime (K, Qhat, V, coefficients: free after A1; [T; Att T], A2T: free
// after A2, A3).  Every mbarrier wait is bounded; a wait that runs out sets
// status[1] and the CTA stops.
#include "mdn_internal.cuh"
#include "tc_common.cuh"

namespace mdn {
namespace {

using namespace sm100;
using namespace tc;

constexpr int NS = 32;         // d_v columns per CTA
constexpr int NH = 16;         // columns per thread
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 256;

// Shared memory map (byte offsets from a 1024-byte aligned base).
constexpr uint32_t KQ0 = 0;                  // [K; Qhat], 2 buffers x 2 panels x (128 x 128 B)
constexpr uint32_t TAT0 = 2 * 32768;         // [T; Att T] 128 x 64 bf16 (K-major SW128), 2 buffers
constexpr uint32_t A2T0 = TAT0 + 2 * 16384;  // [A2T_S | A2T_M] 2 panels of 128 x 64, 2 buffers
constexpr uint32_t ST = A2T0 + 2 * 32768;    // [S | M] bf16, 128 rows x (32 + 32), MN-major SW128
constexpr uint32_t YB = ST + 16384;          // Y 64 x 32 bf16, MN-major SW64
constexpr uint32_t V0 = YB + 4096;           // V slice 64 x 32 bf16 (plain rows), 2 buffers
constexpr uint32_t CR0 = V0 + 8192;          // chunk coefficients (256 floats), 2 buffers
constexpr uint32_t OST0 = CR0 + 2 * 1024;    // output staging: [Vtilde | o] 64 x 32 bf16 each, 2 buffers
constexpr uint32_t BARS = OST0 + 2 * 8192;
constexpr uint32_t MISC = BARS + 128;
constexpr uint32_t SMEM_BYTES = MISC + 16 + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory map too large");

// TMEM columns
constexpr uint32_t TM_A1 = 0, TM_A2 = 64, TM_A3 = 128;

constexpr uint32_t kTxA = 32768 + 4096 + 1024;   // K, Qhat, V, coefficients
constexpr uint32_t kTxB = 16384 + 32768;         // [T; Att T], A2T

// mbarriers
constexpr int B_FA0 = 0, B_FB0 = 2, B_M1 = 4, B_M2 = 5, B_M3 = 6;

struct InterArgs {
    const float* crec;
    const float* S0;
    const float* M0;
    float* S_T;
    float* M_T;
    __nv_bfloat16* o;
    __nv_bfloat16* vt;
    unsigned* status;
    float* dbg;  // diagnostics: CTA 0 dumps its first chunk's intermediates and phase clocks
    int T, H, NT;
};

// Offsets (floats) of the diagnostic dump.
constexpr int DBG_A1 = 49152, DBG_Y = 57344, DBG_A2 = 59392, DBG_A3 = 67584, DBG_S = 71680,
              DBG_M = 75776, DBG_CLK = 80400;

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_inter_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_qh,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_tat,
                   const __grid_constant__ CUtensorMap tm_a2t, const __grid_constant__ CUtensorMap tm_vt,
                   const __grid_constant__ CUtensorMap tm_o, const InterArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int lane = ((warp & 3) << 5) | (tid & 31);  // TMEM lane = operand row
    const int hc = warp >> 2;                          // column half: columns 16*hc .. 16*hc+15
    const int r = lane & 63;
    const bool producer = tid == 128;  // issues every TMA load and store of the CTA
    const int slice = blockIdx.x % (D / NS);
    const int bh = blockIdx.x / (D / NS);
    const int b = bh / a.H, h = bh % a.H;
    const int j0 = slice * NS;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);

    if (tid == 0) {
        for (int k = 0; k < 7; ++k) mbar_init(&bars[k], 1);
        mbar_fence_init();
        *reinterpret_cast<volatile int*>(sm + MISC + 4) = 0;
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // entering state: row `lane` of S and M, columns j0 + 16 hc ..
    float s[NH], m[NH];
    {
        const size_t row = ((size_t)bh * D + lane) * D + j0 + NH * hc;
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            s[j] = a.S0 ? a.S0[row + j] : 0.f;
            m[j] = a.M0 ? a.M0[row + j] : 0.f;
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            st_bf16x8(sm + ST + sw128_off(lane, 2 * hc + c), s + 8 * c);
            st_bf16x8(sm + ST + sw128_off(lane, 4 + 2 * hc + c), m + 8 * c);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + NH * hc;

    auto load_a = [&](int n) {  // K, Qhat, V, coefficients of chunk n
        const int buf = n & 1;
        uint64_t* fb = &bars[B_FA0 + buf];
        const long long chunk = (long long)bh * a.NT + n;
        mbar_arrive_expect_tx(fb, kTxA);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_4d(sm + KQ0 + buf * 32768 + p * 16384, &tm_k, p * 64, h, n * C, b, fb);
            tma_load_3d(sm + KQ0 + buf * 32768 + p * 16384 + 8192, &tm_qh, p * 64, 0, (int)chunk, fb);
        }
        tma_load_4d(sm + V0 + buf * 4096, &tm_v, j0, h, n * C, b, fb);
        bulk_load(sm + CR0 + buf * 1024, a.crec + chunk * 256, 1024, fb);
    };
    auto load_b = [&](int n) {  // [T; Att T] and A2T of chunk n
        const int buf = n & 1;
        uint64_t* fb = &bars[B_FB0 + buf];
        const long long chunk = (long long)bh * a.NT + n;
        mbar_arrive_expect_tx(fb, kTxB);
        tma_load_3d(sm + TAT0 + buf * 16384, &tm_tat, 0, 0, (int)chunk, fb);
        tma_load_3d(sm + A2T0 + buf * 32768, &tm_a2t, 0, 0, (int)chunk, fb);
        tma_load_3d(sm + A2T0 + buf * 32768 + 16384, &tm_a2t, 0, 128, (int)chunk, fb);
    };
    if (producer) {
        for (int n = 0; n < 2 && n < a.NT; ++n) {
            load_a(n);
            load_b(n);
        }
    }
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + MISC + 4);

    bool ok = true;
    PhaseClock clk;
    clk.start((a.dbg && blockIdx.x == 0 && tid == 0) ? a.dbg + DBG_CLK + 16 : nullptr);
    float oi[NH];
    // Vtilde and o of chunk n once its A3 product has completed; then the
    // [T; Att T] / A2T buffer of chunk n is free for chunk n + 2.
    auto store_outputs = [&](int n) -> bool {
        if (!mbar_wait(&bars[B_M3], n & 1)) return false;
        tc_fence_after_sync();
        if (producer && n + 2 < a.NT) load_b(n + 2);
        float o3[NH];
        tmem_ld16(tl + TM_A3, o3);
        tmem_wait_ld();
        if (a.dbg != nullptr && blockIdx.x == 0 && n == 0)
            for (int j = 0; j < NH; ++j) a.dbg[DBG_A3 + lane * 32 + NH * hc + j] = o3[j];
        // rows of Vtilde (lanes 0..63) and o (lanes 64..127) into the staging tile;
        // a TMA store (rows past T are clipped) writes them out
        uint8_t* stg = sm + OST0 + (n & 1) * 8192 + (lane < C ? 0 : 4096) + r * 64 + 32 * hc;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            float w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                w[e] = (lane < C) ? o3[8 * c + e] : o3[8 * c + e] + oi[8 * c + e];
            *reinterpret_cast<uint4*>(stg + 16 * c) = bf16x8(w);
        }
        fence_proxy_async_smem();
        return true;
    };

    auto issue_stores = [&](int n) {  // thread 0, after a barrier that follows store_outputs(n)
        const uint8_t* stg = sm + OST0 + (n & 1) * 8192;
        tma_store_4d(&tm_vt, j0, h, n * C, b, stg);
        tma_store_4d(&tm_o, j0, h, n * C, b, stg + 4096);
        bulk_commit_group();
    };
    // MMA descriptors: base descriptors plus start-address offsets (16-byte units)
    const uint64_t d_kq0 = smem_desc(sbase + KQ0, 16, 1024, kSw128);
    const uint64_t d_st = smem_desc(sbase + ST, 8192, 1024, kSw128);
    const uint64_t d_a20 = smem_desc(sbase + A2T0, 16, 1024, kSw128);
    const uint64_t d_tat0 = smem_desc(sbase + TAT0, 16, 1024, kSw128);
    const uint64_t d_y = smem_desc(sbase + YB, 4096, 512, kSw64);
    const uint32_t id1 = idesc_bf16(128, 64, false, true);
    const uint32_t id2 = idesc_bf16(128, 32, false, true);

    // A wait that runs out sets the abort flag before the next barrier; every
    // thread reads it after that barrier, so all leave the loop together.
    auto fail = [&](bool w) {
        if (!w) *abort_flag = 1;
    };
    for (int n = 0; n < a.NT; ++n) {
        const int buf = n & 1;
        const float* cr = reinterpret_cast<const float*>(sm + CR0 + buf * 1024);
        const bool dump = a.dbg != nullptr && blockIdx.x == 0 && n == 0;
        // the staging tile about to be written (chunk n-1) was last stored for chunk n-3
        if (producer) bulk_wait_group_read<1>();
        fail(mbar_wait(&bars[B_FA0 + buf], (n >> 1) & 1));
        __syncthreads();
        if (*abort_flag) break;
        clk.lap(0);
        const float c_ab = cr[r], c_d2 = cr[C + r], c_b = cr[2 * C + r];
        const float abC = cr[3 * C], bC = cr[3 * C + 1], mbC = cr[3 * C + 2];

        // A1 = [K; Qhat] [S | M]   (warp 0, one elected lane issues)
        if (warp == 0) {
            tc_fence_after_sync();
            const uint64_t dkq = d_kq0 + buf * (32768 >> 4);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = dkq + (((ks >> 2) * 16384 + (ks & 3) * 32) >> 4);
                const uint64_t bd = d_st + ks * (2048 >> 4);
                if (elect_one()) mma_bf16(tmem + TM_A1, ad, bd, id1, ks > 0);
            }
            if (elect_one()) mma_commit(&bars[B_M1]);
            __syncwarp();
        }
        if (n > 0) fail(store_outputs(n - 1));
        fail(mbar_wait(&bars[B_M1], n & 1));
        tc_fence_after_sync();
        __syncthreads();
        if (*abort_flag) break;
        if (producer && n > 0) issue_stores(n - 1);
        clk.lap(1);

        // Y = V - X (rows 0..63); Oi kept in registers (rows 64..127)
        {
            float x[NH], y[NH];
            tmem_ld16(tl + TM_A1, x);
            tmem_ld16(tl + TM_A1 + 32, y);
            tmem_wait_ld();
            if (dump)
                for (int j = 0; j < NH; ++j) {
                    a.dbg[DBG_A1 + lane * 64 + NH * hc + j] = x[j];
                    a.dbg[DBG_A1 + lane * 64 + 32 + NH * hc + j] = y[j];
                }
            if (lane < C) {
                const uint4* vrow = reinterpret_cast<const uint4*>(sm + V0 + buf * 4096 + r * 64) + 2 * hc;
                float yy[NH];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float vv[8];
                    unpack_bf16x8(vrow[c], vv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = 8 * c + e;
                        yy[j] = vv[e] - (c_ab * x[j] - c_d2 * y[j]);
                    }
                }
                if (dump)
                    for (int j = 0; j < NH; ++j) a.dbg[DBG_Y + r * NS + NH * hc + j] = yy[j];
#pragma unroll
                for (int c = 0; c < 2; ++c) st_bf16x8(sm + YB + sw64_off(r, 2 * hc + c), yy + 8 * c);
                fence_proxy_async_smem();
            } else {
#pragma unroll
                for (int j = 0; j < NH; ++j) oi[j] = c_ab * x[j] - c_b * y[j];
            }
        }
        tc_fence_before_sync();
        fail(mbar_wait(&bars[B_FB0 + buf], (n >> 1) & 1));
        __syncthreads();
        if (*abort_flag) break;
        clk.lap(2);

        // A2 = [A2T_S; A2T_M] Y, then A3 = [T; Att T] Y   (warp 0)
        if (warp == 0) {
            tc_fence_after_sync();
            const uint64_t da2 = d_a20 + buf * (32768 >> 4), dtat = d_tat0 + buf * (16384 >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t yd = d_y + ks * (1024 >> 4);
                if (elect_one()) mma_bf16(tmem + TM_A2, da2 + ks * 2, yd, id2, ks > 0);
                if (elect_one()) mma_bf16(tmem + TM_A2 + 32, da2 + (16384 >> 4) + ks * 2, yd, id2, ks > 0);
            }
            if (elect_one()) mma_commit(&bars[B_M2]);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t yd = d_y + ks * (1024 >> 4);
                if (elect_one()) mma_bf16(tmem + TM_A3, dtat + ks * 2, yd, id2, ks > 0);
            }
            if (elect_one()) mma_commit(&bars[B_M3]);
            __syncwarp();
        }
        // K, Qhat, V and the coefficients of this buffer are no longer needed
        if (producer && n + 2 < a.NT) load_a(n + 2);
        fail(mbar_wait(&bars[B_M2], n & 1));
        tc_fence_after_sync();
        clk.lap(3);

        // state update
        {
            float dS[NH], dM[NH];
            tmem_ld16(tl + TM_A2, dS);
            tmem_ld16(tl + TM_A2 + 32, dM);
            tmem_wait_ld();
            if (dump)
                for (int j = 0; j < NH; ++j) {
                    a.dbg[DBG_A2 + lane * 64 + NH * hc + j] = dS[j];
                    a.dbg[DBG_A2 + lane * 64 + 32 + NH * hc + j] = dM[j];
                }
#pragma unroll
            for (int j = 0; j < NH; ++j) {
                const float sn = fmaf(abC, s[j], fmaf(-bC, m[j], dS[j]));
                m[j] = fmaf(mbC, m[j], dM[j]);
                s[j] = sn;
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                st_bf16x8(sm + ST + sw128_off(lane, 2 * hc + c), s + 8 * c);
                st_bf16x8(sm + ST + sw128_off(lane, 4 + 2 * hc + c), m + 8 * c);
            }
            if (dump)
                for (int j = 0; j < NH; ++j) {
                    a.dbg[DBG_S + lane * NS + NH * hc + j] = s[j];
                    a.dbg[DBG_M + lane * NS + NH * hc + j] = m[j];
                }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        clk.lap(4);
    }
    ok = *abort_flag == 0;
    clk.flush();
    __syncthreads();
    ok = *abort_flag == 0;
    if (ok && a.NT > 0) fail(store_outputs(a.NT - 1));
    __syncthreads();
    ok = *abort_flag == 0;
    if (ok && producer && a.NT > 0) issue_stores(a.NT - 1);
    if (producer) bulk_wait_group_all();  // every output tile has been written out
    if (ok) {
        const size_t row = ((size_t)bh * D + lane) * D + j0 + NH * hc;
#pragma unroll
        for (int j = 0; j < NH; ++j) {
            a.S_T[row + j] = s[j];
            a.M_T[row + j] = m[j];
        }
    } else if (producer) {
        atomicOr(a.status + 1, 1u);
        // Loads that were issued must land before the CTA's shared memory is
        // released; only the last two chunks' buffers can still be in flight.
        for (int n = a.NT - 2; n < a.NT; ++n)
            if (n >= 0) {
                (void)mbar_wait(&bars[B_FA0 + (n & 1)], (n >> 1) & 1);
                (void)mbar_wait(&bars[B_FB0 + (n & 1)], (n >> 1) & 1);
            }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_chunk_inter_tc(const ChunkArgs& a, cudaStream_t s)
{
    CUtensorMap mk, mqh, mv, mtat, ma2t, mvt, mo;
    const long long chunks = (long long)a.B * a.H * a.NT;
    if (!make_token_map(&mk, a.k, a.B, a.T, a.H, 64, true) ||
        !make_chunk_map(&mqh, a.qhat, chunks, C, D, C) ||
        !make_token_map(&mv, a.v, a.B, a.T, a.H, NS, false) ||
        !make_chunk_map(&mtat, a.tat, chunks, 2 * C, C, 2 * C) ||
        !make_chunk_map(&ma2t, a.a2t, chunks, 2 * D, C, 128) ||
        !make_token_map(&mvt, a.vt, a.B, a.T, a.H, NS, false) ||
        !make_token_map(&mo, a.o, a.B, a.T, a.H, NS, false))
        return cudaErrorInvalidValue;
    InterArgs t;
    t.crec = a.crec;
    t.S0 = a.S0;
    t.M0 = a.M0;
    t.S_T = a.S_T;
    t.M_T = a.M_T;
    t.o = static_cast<__nv_bfloat16*>(a.o);
    t.vt = static_cast<__nv_bfloat16*>(a.vt);
    t.status = a.status;
    t.dbg = a.dbg;
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
    chunk_inter_kernel<<<(unsigned)blocks, kThreads, SMEM_BYTES, s>>>(mk, mqh, mv, mtat, ma2t, mvt,
                                                                       mo, t);
    return cudaGetLastError();
}

// The tensor-core path: the intra-chunk kernel, then the sequential
// inter-chunk kernel, both on stream s.
cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t s)
{
    if (a.D != D) return cudaErrorNotSupported;
    cudaError_t e = launch_chunk_intra_tc(a, s);
    if (e != cudaSuccess) return e;
    return launch_chunk_inter_tc(a, s);
}

}  // namespace mdn
