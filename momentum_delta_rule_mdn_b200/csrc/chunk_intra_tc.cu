// K-2 on sm_100a: the intra-chunk part of the chunkwise MDN forward pass.
//
// "MDN: Parallelizing Stepwise Momentum for Delta Linear Attention",
// paper.rainbus.top summary, steps 3-5.  Per chunk (positions r, i inside it):
//   Qhat   = Q - d K
//   G      = [K; Qhat] [K; Qhat]^T     tcgen05.mma, M=128, N=128, K=128, bf16 in, fp32 in TMEM
//            lane i < 64: k_i.k_r (columns r), k_i.qhat_r (columns 64 + r)
//   Gamma  down each column i by Gamma_{r,i} = alpha_r Gamma_{r-1,i} + eta_i beta_r mubar_r/mubar_i
//          (mubar_r/mubar_i as a running product of mu: non-negative terms only)
//   A      = (P K^T) o Gamma-:  A_{r,i} = alpha_r k_r.k_i Gamma_{r-1,i}  (i < r)
//   Att    = (Qhat K^T) o Gamma:  Att_{r,i} = qhat_r.k_i Gamma_{r,i}  (i <= r)
//   T      = (I + A)^{-1} in fp32 over 16 x 16 blocks: diagonal blocks by forward
//            substitution, B_ik = -T_ii A_ik, then the blocks off the diagonal in
//            two dependent steps (T_10, T_21, T_32 with C_3k = B_3k + B_32 B_2k, then
//            T_20, T_31 and T_30 = C_30 T_00 + C_31 T_10)
//   P      = [I; Att] T = [T; Att T]                    (M=128, N=64,  K=64)
//   R      = K^T [Diag(Gamma_C) T | -Diag(w) T]          (M=128, N=128, K=64)
//            with w_r = eta_r mubar_C / mubar_r
// and writes, per chunk, the operands of the sequential inter-chunk kernel in
// bf16: Qhat [64 x 128], [T; Att T] [128 x 64], A2T = [R_S; R_M] [256 x 64],
// plus the per-position coefficients alphabar_r, alpha_r b_{r-1}, b_r and the
// chunk scalars alphabar_C, b_C, mubar_C (fp32).
//
// The CTAs are persistent (two per SM) and take chunks from a global counter
// in chunk-major order (chunk 0 of every head first), publishing a ready flag
// per chunk; the inter-chunk kernel, launched as their programmatic
// dependent, starts on the SMs whose CTAs leave first (the CTAs on a reserved
// set of SMs take at most a given number of chunks) and follows the flags.  K and Q of a CTA's
// next chunk are loaded by TMA into a second buffer while the current chunk
// computes, and the gate scan of the next chunk runs on a warp that the
// column pass leaves idle.  The loop's code is kept compact (the loops over
// 16-row groups and output halves are not unrolled): two CTAs at different
// phases share each SM's instruction cache.  Column i of Gamma never leaves the registers of
// the thread that owns it: that thread writes column i of A and K-row i of
// the MN-major [I; Att] operand directly.  T is solved in place over A: the
// diagonal blocks replace A_ii, B_ik replaces A_ik (C_30 replaces B_30, C_31
// goes to a scratch block), and T_ij (i > j) goes to the unused block (j, i).
#include "mdn_internal.cuh"
#include "tc_common.cuh"

namespace mdn {
namespace {

using namespace sm100;
using namespace tc;

constexpr int kThreads = 128;
constexpr int kTmaTid = 64;  // issues every TMA load and store (its warp idles in the column pass)
// Shared memory (byte offsets from a 1024-byte aligned base).
constexpr uint32_t KQ0 = 0;                   // [K; Q] of a chunk, 2 buffers; a buffer holds 2
                                              // feature panels of (64 rows of K, 64 rows of Q) x 128 B
constexpr uint32_t KQ_BYTES = 32768;
constexpr uint32_t AM = 2 * KQ_BYTES;         // fp32 [64][LDF]: A, then T and B in place
constexpr uint32_t IATT = AM + 17408;         // [I; Att] MN-major: 2 M-panels x 64 K-rows x 128 B
constexpr uint32_t DT1 = IATT + 16384;        // N-panel 1 of [D_G T | -D_w T] (8 KB)
constexpr uint32_t REC = DT1 + 8192;          // gate record, 2 buffers x 6 x 64 floats
constexpr uint32_t VEC = REC + 2 * 1536;      // mu_r, w_r, Gamma_{C,r}
constexpr uint32_t BARS = VEC + 768;
constexpr uint32_t MISC = BARS + 32;          // TMEM address; chunk indices of the next two iterations
constexpr uint32_t SMEM_BYTES = MISC + 32 + 1024;  // + alignment slack
static_assert(AM % 1024 == 0 && IATT % 1024 == 0 && DT1 % 1024 == 0, "operand alignment");
static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
// Aliases, each written only once its previous contents are dead.
constexpr uint32_t TB_OFF = 8192;    // T bf16 (B of P): the Q half of panel 0 of the current buffer
constexpr uint32_t DT0_OFF = 24576;  // N-panel 0 of [D_G T | -D_w T] (B of R): the Q half of panel 1
constexpr uint32_t STG_TAT = AM;     // [T; Att T] staging: over T once the bf16 copies are made
constexpr uint32_t C31 = DT1;        // C_31 (fp32, row stride LDF) during the T solve
// TMEM columns
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t TM_G = 0, TM_P = 0, TM_R = 128;  // P reuses G's columns once G is read
// mbarriers: two K/Q buffers, one for the MMA commits
constexpr int B_LD = 0, B_MMA = 2;

struct IntraArgs {
    GateSrc gates;           // [B, T, H] gates, or their pre-activations
    float* crec;             // [chunks][256]
    unsigned* ready;         // [chunks] set to 1 once a chunk's operands are in global memory
    unsigned* queue;         // next chunk (in chunk-major order) to hand out; zero on entry
    unsigned* status;
    float* dbg;              // diagnostics: phase clocks of CTA 0 (null in normal use)
    float dcorr;
    int T, H, NT, BH;
    int reserve;             // CTAs on SMs 0 .. reserve-1 take at most `limit` chunks,
    int limit;               // freeing those SMs early for the inter-chunk kernel
    const int* chunk_order;  // variable-length mode: the order of the padded chunks; else null
};

// Chunk-major order: the c-th chunk is chunk n of head bh (n taken through
// chunk_order in variable-length mode: the longest sequence's chunks first);
// returns its index in the head-major layout of the workspace.
__device__ __forceinline__ long long chunk_of(long long c, const IntraArgs& a, int& n, int& bh) {
    const unsigned cu = (unsigned)c, q = cu / (unsigned)a.BH;  // chunk counts fit 32 bits
    n = a.chunk_order ? a.chunk_order[q] : (int)q;
    bh = (int)(cu - q * (unsigned)a.BH);
    return (long long)bh * a.NT + n;
}

// Marks a chunk's operands as written: its bulk stores have completed (the
// caller waited for them) and the chunk record was stored before a CTA barrier.
__device__ __forceinline__ void publish_chunk(unsigned* ready, long long chunk) {
    fence_proxy_async_global();
    __threadfence();
    st_release_gpu(ready + chunk, 1u);
}

// Gate record of one chunk (one warp): la, lm, b, alpha, beta, eta per
// position, from the gates or from their pre-activations (the fused
// parameterisation); positions past T are steps that leave the state unchanged.  Not
// inlined: the kernel's loop is kept small for the instruction cache.
__device__ __noinline__ void gate_record(const IntraArgs& a, int n, int bh, float* rec, int lane) {
    const int b = bh / a.H, h = bh % a.H;
    const int t0 = n * C + 2 * lane;
    float ga[2] = {0.f, 0.f}, gm[2] = {0.f, 0.f}, gb[2] = {0.f, 0.f}, ge[2] = {0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        if (t0 + e < a.T) {
            gates_at(a.gates, ((size_t)b * a.T + t0 + e) * a.H + h, ga[e], gm[e], gb[e], ge[e]);
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

// acc += rows r0, r0 + 1 of X times columns c0 .. c0 + 3 of Y, for 16 x 16
// blocks X (at x) and Y (at y), both with row stride LDF.
__device__ __forceinline__ void tile_2x4(const float* x, const float* y, int r0, int c0,
                                         float4& acc0, float4& acc1) {
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
        const float4 a0 = lds4(x + r0 * LDF + 4 * k4);
        const float4 a1 = lds4(x + (r0 + 1) * LDF + 4 * k4);
        const float x0[4] = {a0.x, a0.y, a0.z, a0.w};
        const float x1[4] = {a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float4 t4 = lds4(y + (4 * k4 + e) * LDF + c0);
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

__global__ void __launch_bounds__(kThreads)
chunk_intra_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_qh, const __grid_constant__ CUtensorMap tm_tat,
                   const __grid_constant__ CUtensorMap tm_a2t, const IntraArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long chunks = (long long)a.BH * a.NT;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + MISC);
    float* Am = reinterpret_cast<float*>(sm + AM);
    float* mu = reinterpret_cast<float*>(sm + VEC);
    float* wv = mu + C;    // w_r = eta_r mubar_C / mubar_r
    float* wg = wv + C;    // Gamma_{C,r}
    // The inter-chunk kernel may be scheduled as soon as every CTA of this grid
    // has started; it waits for each chunk's ready flag before reading it.
    pdl_launch_dependents();
    PhaseClock clk;
    clk.start((a.dbg && blockIdx.x == 0 && tid == 0) ? a.dbg : nullptr);
#ifdef MDN_PHASE_CLOCKS
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    const uint64_t t_begin = global_timer_ns();
#endif

    // K and Q of the c-th chunk into buffer buf (thread 0); the pending load
    // is remembered so that an abort can drain it.
    int pend_buf = -1;
    uint32_t pend_par = 0;
    auto load_kq = [&](long long c, int iter) {
        int n, bh;
        (void)chunk_of(c, a, n, bh);
        const int b = bh / a.H, h = bh % a.H, buf = iter & 1;
        uint64_t* bar = &bars[B_LD + buf];
        mbar_arrive_expect_tx(bar, KQ_BYTES);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            uint8_t* dst = sm + KQ0 + buf * KQ_BYTES + p * 16384;
            tma_load_4d(dst, &tm_k, p * 64, h, n * C, b, bar);
            tma_load_4d(dst + 8192, &tm_q, p * 64, h, n * C, b, bar);
        }
        pend_buf = buf;
        pend_par = (iter >> 1) & 1;
    };

    // chunk indices of the next two iterations (slot = iteration & 1)
    long long* cslot = reinterpret_cast<long long*>(sm + MISC + 16);
    int fetched = 0, limit = 1 << 30;  // TMA thread: chunks taken from the counter
    auto fetch = [&]() -> long long {
        if (fetched >= limit) return chunks;
        ++fetched;
        const unsigned c = atomicAdd(a.queue, 1u);
        return c < chunks ? (long long)c : chunks;
    };
    if (tid == kTmaTid) {
        uint32_t smid_;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid_));
        if ((int)smid_ < a.reserve) limit = a.limit;
        mbar_init(&bars[B_LD], 1);
        mbar_init(&bars[B_LD + 1], 1);
        mbar_init(&bars[B_MMA], 1);
        mbar_fence_init();
        const long long c0 = fetch();
        cslot[0] = c0;
        cslot[1] = c0 < chunks ? fetch() : chunks;
        if (c0 < chunks) load_kq(c0, 0);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (tid < C) {  // K-row tid of the identity M-panel of [I; Att]; never overwritten
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = (8 * cc + e == tid) ? 1.f : 0.f;
            st_bf16x8(sm + IATT + sw128_off(tid, cc), x);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_sel = static_cast<uint32_t>(warp * 32) << 16;
    if (warp == 3 && cslot[0] < chunks) {  // ordered before use by the loop's first barrier
        int n, bh;
        (void)chunk_of(cslot[0], a, n, bh);
        gate_record(a, n, bh, reinterpret_cast<float*>(sm + REC), lane);
    }

    bool ok = true;
    uint32_t mma_phase = 0;
    int k = 0;
    long long prev_chunk = -1;  // thread 0: the chunk whose stores were issued last
    for (long long c = cslot[0]; c < chunks; ++k) {
        const int buf = k & 1;
        uint8_t* kq = sm + KQ0 + buf * KQ_BYTES;
        const uint32_t kq_s = sbase + KQ0 + buf * KQ_BYTES;
        const float* rec = reinterpret_cast<const float*>(sm + REC + buf * 1536);
        int n, bh;
        const long long chunk = chunk_of(c, a, n, bh);
        const long long c_next = cslot[buf ^ 1];  // written an iteration ago (or before the loop)
        // A is about to be overwritten: the store of [T; Att T] from its staging
        // tile (all store groups but the newest) must have read it
        if (tid == kTmaTid) bulk_wait_group_read<1>();
        ok = __syncthreads_and(mbar_wait(&bars[B_LD + buf], (k >> 1) & 1));
        if (!ok) break;
        if (tid == kTmaTid && pend_buf == buf) pend_buf = -1;
        clk.lap(0);

        // ---- Qhat = Q - d K in place (the Q rows of both panels); chunk record
#pragma unroll 2
        for (int u = 0; u < 8; ++u) {
            const int idx = tid + 128 * u;
            const int pn = idx >> 9, w = idx & 511, r = w >> 3, cc = w & 7;
            const uint4 kw = *reinterpret_cast<const uint4*>(kq + pn * 16384 + sw128_off(r, cc));
            uint8_t* qp = kq + pn * 16384 + sw128_off(r + 64, cc);
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
        if (tid == kTmaTid) {
            tma_store_3d(&tm_qh, 0, 0, (int)chunk, kq + 8192);
            tma_store_3d(&tm_qh, 64, 0, (int)chunk, kq + 16384 + 8192);
            bulk_commit_group();
        }
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t id = idesc_bf16(128, 128, false, false);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad =
                    smem_desc(kq_s + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSw128);
                mma_bf16(tmem + TM_G, ad, ad, id, ks > 0);
            }
            mma_commit(&bars[B_MMA]);
        }
        ok = mbar_wait(&bars[B_MMA], mma_phase);
        mma_phase ^= 1;
        tc_fence_after_sync();
        ok = __syncthreads_and(ok);
        if (!ok) break;
        clk.lap(2);

        // ---- column pass: thread i < 64 owns column i of Gamma, A and Att
        if (tid < C) {
            const int i = tid;
            const float* al = rec + 3 * C;
            const float* be = rec + 4 * C;
            const float eta_i = rec[5 * C + i];
            float gam = 0.f, f = 1.f;
#pragma unroll 1
            for (int r16 = 0; r16 < C; r16 += 16) {
                float kk[16], kh[16];
                tmem_ld16(tmem + lane_sel + TM_G + r16, kk);      // k_i.k_r
                tmem_ld16(tmem + lane_sel + TM_G + C + r16, kh);  // k_i.qhat_r
                tmem_wait_ld();
                float att[16];
#pragma unroll
                for (int r4 = 0; r4 < 16; r4 += 4) {
                    const float4 a4 = lds4(al + r16 + r4), b4 = lds4(be + r16 + r4),
                                 m4 = lds4(mu + r16 + r4);
                    const float ar_[4] = {a4.x, a4.y, a4.z, a4.w};
                    const float br_[4] = {b4.x, b4.y, b4.z, b4.w};
                    const float mr_[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = r16 + r4 + e;
                        Am[r * LDF + i] = (r > i) ? ar_[e] * kk[r4 + e] * gam : 0.f;
                        f = (r > i) ? f * mr_[e] : 1.f;
                        gam = (r >= i) ? fmaf(ar_[e], gam, eta_i * br_[e] * f) : 0.f;
                        att[r4 + e] = kh[r4 + e] * gam;  // gam = 0 above the diagonal
                    }
                }
                // column i of Att, rows r16 .. r16 + 15: M-panel 1, K-row i
                st_bf16x8(sm + IATT + 8192 + sw128_off(i, r16 / 8), att);
                st_bf16x8(sm + IATT + 8192 + sw128_off(i, r16 / 8 + 1), att + 8);
            }
            wg[i] = gam;  // Gamma_{C,i}
        } else if (tid == kTmaTid) {
            // every store group but the newest (Qhat) has completed: the previous
            // chunk is in global memory, and its A2T staging buffer is free for
            // K, Q of the next chunk
            bulk_wait_group<1>();
            if (prev_chunk >= 0) publish_chunk(a.ready, prev_chunk);
            if (c_next < chunks) load_kq(c_next, k + 1);
            // the chunk after next; every thread has read this slot's old value
            cslot[buf] = c_next < chunks ? fetch() : chunks;
        } else if (warp == 3 && c_next < chunks) {
            int n2, bh2;
            (void)chunk_of(c_next, a, n2, bh2);
            gate_record(a, n2, bh2, reinterpret_cast<float*>(sm + REC + (buf ^ 1) * 1536), lane);
        }
        __syncthreads();
        clk.lap(3);

        // ---- diagonal blocks of T by forward substitution, one column per thread
        {
            const int blk = tid >> 4, cl = tid & 15, o = 16 * blk;
            float t[16];
            if (tid < C) {
#pragma unroll
                for (int r = 0; r < 16; ++r) t[r] = (r == cl) ? 1.f : 0.f;
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
                    for (int kk = 0; kk < r; ++kk) acc = fmaf(av[kk], t[kk], acc);
                    if (r > cl) t[r] = -acc;
                }
            }
            __syncthreads();  // A_ii has been read
            if (tid < C) {
#pragma unroll
                for (int r = 0; r < 16; ++r) Am[(o + r) * LDF + o + cl] = t[r];
            }
        }
        __syncthreads();
        clk.lap(4);

        // ---- B_ik = -T_ii A_ik for the six blocks below the diagonal, in place
        {
            // blocks (i, k): (1,0) (2,0) (2,1) (3,0) (3,1) (3,2), 32 tiles of 2 x 4 each
            float4 res[2][2];
            int where[2];
#pragma unroll
            for (int rep = 0; rep < 2; ++rep) {
                const int tile = tid + 128 * rep;
                where[rep] = -1;
                if (tile < 192) {
                    const int bidx = tile >> 5;
                    const int bi = bidx < 1 ? 1 : (bidx < 3 ? 2 : 3);
                    const int bk = bidx < 1 ? 0 : (bidx < 3 ? bidx - 1 : bidx - 3);
                    const int r0 = 2 * ((tile >> 2) & 7), c0 = 4 * (tile & 3);
                    float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
                    tile_2x4(Am + 16 * bi * LDF + 16 * bi, Am + 16 * bi * LDF + 16 * bk, r0, c0,
                             acc0, acc1);
                    res[rep][0] = make_float4(-acc0.x, -acc0.y, -acc0.z, -acc0.w);
                    res[rep][1] = make_float4(-acc1.x, -acc1.y, -acc1.z, -acc1.w);
                    where[rep] = (16 * bi + r0) * LDF + 16 * bk + c0;
                }
            }
            __syncthreads();  // every read of A_ik precedes its overwrite
#pragma unroll
            for (int rep = 0; rep < 2; ++rep)
                if (where[rep] >= 0) {
                    *reinterpret_cast<float4*>(Am + where[rep]) = res[rep][0];
                    *reinterpret_cast<float4*>(Am + where[rep] + LDF) = res[rep][1];
                }
        }
        __syncthreads();
        clk.lap(5);

        // ---- T off the diagonal in two dependent steps instead of three levels:
        //      step 1: T_10 = B_10 T_00, T_21 = B_21 T_11, T_32 = B_32 T_22 into blocks
        //      (0,1), (1,2), (2,3), and C_30 = B_30 + B_32 B_20 over B_30, C_31 = B_31 +
        //      B_32 B_21 into a scratch block over DT1 (free until the bf16 copies);
        //      step 2: T_20 = B_20 T_00 + B_21 T_10, T_31 = B_31 T_11 + B_32 T_21,
        //      T_30 = C_30 T_00 + C_31 T_10 (= B_30 T_00 + B_31 T_10 + B_32 T_20)
#pragma unroll 1
        for (int rep = 0; rep < 2; ++rep) {
            const int tt = tid + 128 * rep;
            if (tt < 160) {
                const int job = tt >> 5;
                const int r0 = 2 * ((tt >> 2) & 7), c0 = 4 * (tt & 3);
                float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
                float* dst;
                if (job < 3) {  // T_{j+1,j} = B_{j+1,j} T_jj
                    const int j = job;
                    tile_2x4(Am + 16 * (j + 1) * LDF + 16 * j, Am + 16 * j * LDF + 16 * j, r0, c0,
                             acc0, acc1);
                    dst = Am + (16 * j + r0) * LDF + 16 * (j + 1) + c0;
                } else {        // C_3k = B_3k + B_32 B_2k, k = 0, 1
                    const int kb = job - 3;
                    const float* b3k = Am + (48 + r0) * LDF + 16 * kb + c0;
                    acc0 = lds4(b3k);
                    acc1 = lds4(b3k + LDF);
                    tile_2x4(Am + 48 * LDF + 32, Am + 32 * LDF + 16 * kb, r0, c0, acc0, acc1);
                    dst = kb == 0 ? Am + (48 + r0) * LDF + c0
                                  : reinterpret_cast<float*>(sm + C31) + r0 * LDF + c0;
                }
                *reinterpret_cast<float4*>(dst) = acc0;
                *reinterpret_cast<float4*>(dst + LDF) = acc1;
            }
        }
        __syncthreads();
        if (tid < 96) {
            const int job = tid >> 5;
            const int r0 = 2 * ((tid >> 2) & 7), c0 = 4 * (tid & 3);
            float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
            const float* x0;
            const float* y0;
            const float* x1;
            const float* y1;
            float* dst;
            if (job == 0) {
                x0 = Am + 32 * LDF;      y0 = Am;                  // B_20, T_00
                x1 = Am + 32 * LDF + 16; y1 = Am + 16;             // B_21, T_10
                dst = Am + r0 * LDF + 32 + c0;
            } else if (job == 1) {
                x0 = Am + 48 * LDF + 16; y0 = Am + 16 * LDF + 16;  // B_31, T_11
                x1 = Am + 48 * LDF + 32; y1 = Am + 16 * LDF + 32;  // B_32, T_21
                dst = Am + (16 + r0) * LDF + 48 + c0;
            } else {
                x0 = Am + 48 * LDF;      y0 = Am;                  // C_30, T_00
                x1 = reinterpret_cast<const float*>(sm + C31);     // C_31
                y1 = Am + 16;                                      // T_10
                dst = Am + r0 * LDF + 48 + c0;
            }
            tile_2x4(x0, y0, r0, c0, acc0, acc1);
            tile_2x4(x1, y1, r0, c0, acc0, acc1);
            *reinterpret_cast<float4*>(dst) = acc0;
            *reinterpret_cast<float4*>(dst + LDF) = acc1;
        }
        __syncthreads();
        clk.lap(6);

        // ---- bf16 copies of T: T (B of P) into the Q half of panel 0, and
        //      [D_G T | -D_w T] (B of R) into the Q half of panel 1 and DT1.  The
        //      store of Qhat must have read both halves.
        if (tid == kTmaTid) bulk_wait_group_read<0>();
        __syncthreads();
        {
            const int r = tid & 63, hf = tid >> 6;  // row r of T, columns 32 hf .. 32 hf + 31
            const int bi = r >> 4;
            const float g = wg[r], w = -wv[r];
#pragma unroll 1
            for (int q = 0; q < 2; ++q) {
                const int bj = 2 * hf + q;  // 16-column block of T
                float x[16];
                if (bj <= bi) {
                    const float* src = (bj == bi) ? Am + r * LDF + 16 * bi
                                                  : Am + (16 * bj + (r & 15)) * LDF + 16 * bi;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 v4 = lds4(src + 4 * q4);
                        x[4 * q4] = v4.x;
                        x[4 * q4 + 1] = v4.y;
                        x[4 * q4 + 2] = v4.z;
                        x[4 * q4 + 3] = v4.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = 0.f;
                }
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const uint32_t off = sw128_off(r, 2 * bj + h8);
                    float y[8], z[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        y[e] = g * x[8 * h8 + e];
                        z[e] = w * x[8 * h8 + e];
                    }
                    st_bf16x8(kq + TB_OFF + off, x + 8 * h8);
                    st_bf16x8(kq + DT0_OFF + off, y);
                    st_bf16x8(sm + DT1 + off, z);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        clk.lap(7);
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t idp = idesc_bf16(128, 64, true, true);
            const uint32_t idr = idesc_bf16(128, 128, true, true);
            const uint32_t dt_lbo = (sbase + DT1) - (kq_s + DT0_OFF);  // N-panel 0 -> 1
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_P, smem_desc(sbase + IATT + ks * 2048, 8192, 1024, kSw128),
                         smem_desc(kq_s + TB_OFF + ks * 2048, 8192, 1024, kSw128), idp, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + TM_R, smem_desc(kq_s + ks * 2048, 16384, 1024, kSw128),
                         smem_desc(kq_s + DT0_OFF + ks * 2048, dt_lbo, 1024, kSw128), idr, ks > 0);
            mma_commit(&bars[B_MMA]);
        }
        ok = mbar_wait(&bars[B_MMA], mma_phase);
        mma_phase ^= 1;
        tc_fence_after_sync();
        ok = __syncthreads_and(ok);
        if (!ok) break;
        clk.lap(8);

        // ---- [T; Att T] row = lane into its staging tile over A, then its store
        float v[64];
        tmem_ld32(tmem + lane_sel + TM_P, *reinterpret_cast<float(*)[32]>(v));
        tmem_ld32(tmem + lane_sel + TM_P + 32, *reinterpret_cast<float(*)[32]>(v + 32));
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) st_bf16x8(sm + STG_TAT + sw128_off(tid, cc), v + 8 * cc);
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == kTmaTid) {
            tma_store_3d(&tm_tat, 0, 0, (int)chunk, sm + STG_TAT);
            bulk_commit_group();
        }
        clk.lap(9);

        // ---- A2T rows (lane, 128 + lane) into the current K/Q buffer (K has been read)
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
            tmem_ld32(tmem + lane_sel + TM_R + 64 * q2, *reinterpret_cast<float(*)[32]>(v));
            tmem_ld32(tmem + lane_sel + TM_R + 64 * q2 + 32, *reinterpret_cast<float(*)[32]>(v + 32));
            tmem_wait_ld();
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) st_bf16x8(kq + q2 * 16384 + sw128_off(tid, cc), v + 8 * cc);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
        if (tid == kTmaTid) {
            tma_store_3d(&tm_a2t, 0, 0, (int)chunk, kq);
            tma_store_3d(&tm_a2t, 0, 128, (int)chunk, kq + 16384);
            bulk_commit_group();
            prev_chunk = chunk;
        }
        clk.lap(10);
        c = c_next;
    }
    clk.flush();
    if (tid == kTmaTid) {
        if (!ok) {
            atomicOr(a.status + 1, 1u);
            // a load that was issued must land before shared memory goes away
            if (pend_buf >= 0) (void)mbar_wait(&bars[B_LD + pend_buf], pend_par);
        }
        bulk_wait_group_all();  // the stores have completed
        if (ok && prev_chunk >= 0) publish_chunk(a.ready, prev_chunk);
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
#ifdef MDN_PHASE_CLOCKS
    if (a.dbg && tid == 0 && blockIdx.x < 2048) {
        double* tl = reinterpret_cast<double*>(a.dbg + 64);
        tl[3 * blockIdx.x] = (double)t_begin;
        tl[3 * blockIdx.x + 1] = (double)global_timer_ns();
        tl[3 * blockIdx.x + 2] = (double)smid;
    }
#endif
}

}  // namespace

cudaError_t launch_chunk_intra_tc(const ChunkArgs& a, cudaStream_t s, int reserve, int limit)
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
    t.gates = a.gates();
    t.crec = a.crec;
    t.ready = a.ready;
    t.queue = a.ready + chunks;
    t.reserve = reserve;
    t.chunk_order = a.chunk_order;
    t.limit = limit > 0 ? limit : 1;
    t.status = a.status;
    t.dbg = a.dbg ? a.dbg + 80512 : nullptr;
    t.dcorr = a.dcorr;
    t.T = a.T;
    t.H = a.H;
    t.NT = a.NT;
    t.BH = a.B * a.H;
    cudaError_t e = cudaFuncSetAttribute(chunk_intra_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    // persistent: two CTAs per SM
    const long long grid = chunks < 2LL * sms ? chunks : 2LL * sms;
    ProfScope ps(kIntraTc, s);
    chunk_intra_kernel<<<(unsigned)grid, kThreads, SMEM_BYTES, s>>>(mq, mk, mqh, mtat, ma2t, t);
    return cudaGetLastError();
}

}  // namespace mdn
