// Shared by the two versions of the backward pass's chunk-local kernel (CUDA
// cores and tcgen05): the per-chunk coefficient vectors and the last phase,
// which turns the adjoints of the chunk coefficients into the gate gradients.
//
// Coefficients of one chunk (chunk-local prefix sums of the log gates la, lm):
//   alphabar_r = exp(la_r), b_r = sum_{j<=r} exp(la_r - la_j) beta_j mubar_j,
//   Gamma_{r,i} = eta_i Gp_{r,i},  Gp_{r,i} = sum_{j=i}^{r} exp(la_r - la_j) beta_j exp(lm_j - lm_i),
//   w_r = eta_r mubar_C / mubar_r, D2_r = b_{r-1} alpha_r.
// Given the adjoints of alphabar, b, D2, w (row sums of the state products,
// in the chunk's record), of Gamma (dG) and the chunk-end scalars, the
// gradients of the log gates follow by reverse recurrences along the chunk:
// R_{j,i} = dG_{j,i} + alpha_{j+1} R_{j+1,i} folds the sum over r >= j of
// dG_{r,i} exp(la_r - la_j), and the reverse cumulative sums of the la, lm
// adjoints give those of alpha_log and mu_log.
#pragma once

#include <cuda_bf16.h>

#include "mdn_internal.cuh"

namespace mdn {

// Eight consecutive elements of a token tensor from element idx (a multiple
// of 8) as fp32: one 16-byte load for bf16, two for fp32.
template <typename Tin>
__device__ __forceinline__ void ld8(const void* base, size_t idx, float* x);
template <>
__device__ __forceinline__ void ld8<__nv_bfloat16>(const void* base, size_t idx, float* x) {
    const uint4 w = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + idx);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&u[e]);
        x[2 * e] = __low2float(v);
        x[2 * e + 1] = __high2float(v);
    }
}
template <>
__device__ __forceinline__ void ld8<float>(const void* base, size_t idx, float* x) {
    const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Per-chunk vectors (C floats each) in shared memory.
struct BwdVec {
    float *al, *be, *et, *la, *lm, *b, *da, *db, *dla, *dlm, *de, *dbe;
};
constexpr int kBwdVecFloats = 12 * kChunk;

__device__ __forceinline__ BwdVec bwd_vec(float* base) {
    constexpr int C = kChunk;
    BwdVec v;
    v.al = base;           // alpha
    v.be = v.al + C;       // beta
    v.et = v.be + C;       // eta
    v.la = v.et + C;       // la
    v.lm = v.la + C;       // lm
    v.b = v.lm + C;        // b
    v.da = v.b + C;        // adjoint of alpha (its direct uses: P = Diag(alpha) K, D2)
    v.db = v.da + C;       // adjoint of b
    v.dla = v.db + C;      // adjoint of la
    v.dlm = v.dla + C;     // adjoint of lm
    v.de = v.dlm + C;      // adjoint of eta
    v.dbe = v.de + C;      // adjoint of beta
    return v;
}

// T = (I + A)^{-1} for a strictly lower C x C matrix A (shared memory, row
// stride C + 1) into Ts (same layout), by forward substitution: column c on
// the four lanes 4c .. 4c + 3 of a 256-thread CTA, each summing every fourth
// term.  The caller synchronises before and after.
__device__ __forceinline__ void bwd_unit_lower_inverse(const float* As, float* Ts, int tid)
{
    constexpr int C = kChunk, AS = kChunk + 1;
    const int c = tid >> 2, part = tid & 3;
    if (part == 0) Ts[c] = (c == 0) ? 1.f : 0.f;  // row 0
    __syncwarp();
    for (int r = 1; r < C; ++r) {
        float acc = 0.f;
        if (r > c)
            for (int i = c + part; i < r; i += 4) acc = fmaf(As[r * AS + i], Ts[i * AS + c], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (part == 0) Ts[r * AS + c] = (r == c) ? 1.f : (r > c ? -acc : 0.f);
        __syncwarp();
    }
}

// Storage of the lower-triangular C x C matrices Gp and dG in shared memory
// (element (r, i), i <= r): rows of C + 1 floats, or the lower triangle
// packed by rows.  Both are conflict-free for a warp that walks a row (one
// column per lane) and for one that walks a column (one row per lane: the
// triangular numbers are distinct modulo 32 over 32 consecutive rows).
struct PaddedLower {
    __device__ __forceinline__ int operator()(int r, int i) const { return r * (kChunk + 1) + i; }
};
struct PackedLower {
    static constexpr int kFloats = kChunk * (kChunk + 1) / 2;
    __device__ __forceinline__ int operator()(int r, int i) const { return ((r * (r + 1)) >> 1) + i; }
};

// The last phase (every thread of a CTA of at least 256 threads calls it): dG
// (overwritten) and Gp, lower triangles stored as Idx says, the record of the
// state products (rec_g, in global memory; rec: kBwdRec floats of shared
// scratch), v.da holding the direct adjoint of alpha from P.  Writes the four
// gate gradients of the chunk's tokens.
// A phase timer that does nothing (the default of the coefficient phase's
// optional per-phase timer; diagnostic builds pass one that records cycles).
struct NoPhaseTimer {
    __device__ __forceinline__ void lap(int) {}
};

template <class Idx = PaddedLower, class Timer = NoPhaseTimer>
__device__ __forceinline__ void bwd_coeff_phase(const BwdArgs& a, const float* rec_g,
                                                const BwdVec& v, float* dG, const float* Gp,
                                                float* rec, int tid, int n, int b, int h,
                                                bool rec_loaded = false, int nthreads = 256,
                                                Timer* timer = nullptr)
{
    auto lap = [&](int k) {
        if (timer) timer->lap(k);
    };
    constexpr int C = kChunk;
    const Idx at;
    // the chunk's record in shared memory (rec: kBwdRec floats), so that the
    // loops below read no global memory; a caller that copied it earlier
    // (and synchronised since) passes rec_loaded
    if (!rec_loaded) {
        for (int i = tid; i < kBwdRec; i += nthreads) rec[i] = rec_g[i];
        __syncthreads();
    }
    float* v_al = v.al;
    float* v_be = v.be;
    float* v_et = v.et;
    float* v_la = v.la;
    float* v_lm = v.lm;
    float* v_b = v.b;
    float* v_da = v.da;
    float* v_db = v.db;
    float* v_dla = v.dla;
    float* v_dlm = v.dlm;
    float* v_de = v.de;
    float* v_dbe = v.dbe;
    // coefficient adjoints -> la, lm, beta, eta, alpha
    if (tid < C) {
        const int r = tid;
        const float dD2 = rec[2 * C + r];
        const float b_prev = r > 0 ? v_b[r - 1] : 0.f;
        v_da[r] += dD2 * b_prev;                           // D2_r = b_{r-1} alpha_r
        float db = rec[C + r];
        if (r + 1 < C) db += rec[2 * C + r + 1] * v_al[r + 1];
        float dabar = rec[r];
        if (r == C - 1) {
            dabar += rec[5 * C];                           // alphabar_C S
            db -= rec[5 * C + 1];                          // - b_C M
        }
        v_db[r] = db;
        const float abar = expf(v_la[r]);
        v_dla[r] = dabar * abar + db * v_b[r];
        const float wr = v_et[r] * expf(v_lm[C - 1] - v_lm[r]);
        const float dw = rec[4 * C + r];
        v_dlm[r] = -dw * wr;
        v_de[r] = dw * expf(v_lm[C - 1] - v_lm[r]);
        v_dbe[r] = 0.f;
    }
    __syncthreads();
    lap(0);
    if (tid < 32) {
        // warp 0, positions j = 2 lane, 2 lane + 1
        const int j0 = 2 * tid, j1 = j0 + 1;
        // mubar_C M plus sum_r dw_r eta_r exp(lm_C - lm_r): a warp sum
        float s = rec[4 * C + j0] * v_et[j0] * expf(v_lm[C - 1] - v_lm[j0]) +
                  rec[4 * C + j1] * v_et[j1] * expf(v_lm[C - 1] - v_lm[j1]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        // b_r = sum_{j<=r} exp(la_r - la_j) beta_j mubar_j gives the reverse
        // recurrence Rb_j = db_j + alpha_{j+1} Rb_{j+1} (Rb_C = 0): a suffix
        // scan of the affine maps x -> db_j + alpha_{j+1} x, composed as
        // (b1, a1) o (b2, a2) = (b1 + a1 b2, a1 a2)
        const float a0 = v_al[j1], a1 = j1 + 1 < C ? v_al[j1 + 1] : 0.f;
        const float b0 = v_db[j0], b1 = v_db[j1];
        float sb = fmaf(a0, b1, b0), sa = a0 * a1;  // f_j0 o f_j1
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float ob = __shfl_down_sync(0xffffffffu, sb, off);
            const float oa = __shfl_down_sync(0xffffffffu, sa, off);
            if (tid + off < 32) {
                sb = fmaf(sa, ob, sb);
                sa *= oa;
            }
        }
        float next = __shfl_down_sync(0xffffffffu, sb, 1);  // Rb at j1 + 1
        if (tid == 31) next = 0.f;
        const float Rb0 = sb, Rb1 = fmaf(a1, next, b1);
        const float rb[2] = {Rb0, Rb1};
        const int jj[2] = {j0, j1};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int j = jj[e];
            const float mb = expf(v_lm[j]);
            const float tj = v_be[j] * mb * rb[e];
            v_dbe[j] += mb * rb[e];
            v_dla[j] -= tj;
            v_dlm[j] += tj;
        }
        if (tid == 31) v_dlm[C - 1] += s + rec[5 * C + 2] * expf(v_lm[C - 1]);  // mubar_C M
    }
    __syncthreads();
    lap(1);
    // Gamma = eta o Gp: row sums of dG o Gamma (threads 0..127, two per row),
    // column sums and eta's share (threads 128..255, two per column); the two
    // halves of a sum (alternate terms) are joined by a shuffle
    if (tid < 4 * C) {
        const bool rows = tid < 2 * C;
        const int x = (tid & (2 * C - 1)) >> 1, part = tid & 1;
        float s0 = 0.f, s1 = 0.f;
        if (rows) {
            for (int y = part; y <= x; y += 2) s0 = fmaf(dG[at(x, y)], v_et[y] * Gp[at(x, y)], s0);
        } else {
            for (int y = x + part; y < C; y += 2) {
                const float gp = Gp[at(y, x)];
                s0 = fmaf(dG[at(y, x)], v_et[x] * gp, s0);
                s1 = fmaf(dG[at(y, x)], gp, s1);
            }
        }
        s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
        s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
        if (part == 0) {
            if (rows) {
                v_dla[x] += s0;
            } else {
                v_dlm[x] -= s0;
                v_de[x] += s1;
            }
        }
    }
    __syncthreads();
    lap(2);
    // R_{j,i} = sum_{r>=j} dG_{r,i} exp(la_r - la_j), in place: the reverse
    // recurrence R_j = dG_j + alpha_{j+1} R_{j+1} down each column, by blocks
    // of 16 rows on four threads per column (thread part p owns rows
    // 16p .. 16p + 15).  Each thread runs its block from a zero carry, keeping
    // L_j and the decay P_j = alpha_{j+1} .. alpha_{hi+1} to its block's top;
    // the carries R_{16(p+1)} come down the four lanes, and R_j = L_j + P_j R.
    if (tid < 4 * C) {
        const int i = tid >> 2, part = tid & 3, lo = 16 * part;
        float L[16], P[16], al1[16];
        // every read of the block before any write
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int j = lo + e;
            L[e] = j >= i ? dG[at(j, i)] : 0.f;
            al1[e] = j + 1 < C ? v_al[j + 1] : 0.f;  // alpha_{j+1}; none past the chunk
        }
        float l = 0.f, pr = 1.f;
#pragma unroll
        for (int e = 15; e >= 0; --e) {
            pr *= al1[e];
            l = L[e] + al1[e] * l;
            L[e] = l;
            P[e] = pr;
        }
        // (L, P) at the block's lowest row, from the blocks above
        const unsigned full = 0xffffffffu;
        const int base = (threadIdx.x & 31) & ~3;
        float carry = 0.f;
#pragma unroll
        for (int q = 3; q >= 1; --q) {
            const float lq = __shfl_sync(full, L[0], base + q);
            const float pq = __shfl_sync(full, P[0], base + q);
            if (q > part) carry = lq + pq * carry;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int j = lo + e;
            if (j >= i) dG[at(j, i)] = L[e] + P[e] * carry;
        }
    }
    __syncthreads();
    lap(3);
    // U_j = sum_{i<=j} eta_i exp(lm_j - lm_i) R_{j,i}: four threads per row
    // (every fourth term each), joined by shuffles
    if (tid < 4 * C) {
        const int j = tid >> 2, part = tid & 3;
        float U = 0.f;
        for (int i = part; i <= j; i += 4) U = fmaf(v_et[i] * expf(v_lm[j] - v_lm[i]), dG[at(j, i)], U);
        U += __shfl_xor_sync(0xffffffffu, U, 1);
        U += __shfl_xor_sync(0xffffffffu, U, 2);
        if (part == 0) {
            v_dbe[j] += U;
            v_dla[j] -= v_be[j] * U;
            v_dlm[j] += v_be[j] * U;
        }
    }
    __syncthreads();
    lap(4);
    if (tid < 32) {
        // reverse cumulative sums (la, lm are inclusive prefix sums of the log
        // gates): a warp suffix scan, two positions per lane
        const int j0 = 2 * tid, j1 = j0 + 1;
        const float xa1 = v_dla[j1], xm1 = v_dlm[j1];
        float sa = v_dla[j0] + xa1, sm = v_dlm[j0] + xm1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float oa = __shfl_down_sync(0xffffffffu, sa, off);
            const float om = __shfl_down_sync(0xffffffffu, sm, off);
            if (tid + off < 32) {
                sa += oa;
                sm += om;
            }
        }
        float na = __shfl_down_sync(0xffffffffu, sa, 1), nm = __shfl_down_sync(0xffffffffu, sm, 1);
        if (tid == 31) na = nm = 0.f;
        v_dla[j0] = sa;
        v_dlm[j0] = sm;
        v_dla[j1] = xa1 + na;
        v_dlm[j1] = xm1 + nm;
    }
    __syncthreads();
    lap(5);
    if (tid < C) {
        const int j = tid, t = n * C + j;
        if (t < a.T) {
            const size_t gi = ((size_t)b * a.T + t) * a.H + h;
            a.dalpha_log[gi] = v_da[j] * v_al[j] + v_dla[j];
            a.dmu_log[gi] = v_dlm[j];
            a.dbeta[gi] = v_dbe[j];
            a.deta[gi] = v_de[j];
        }
    }
    lap(6);
}

}  // namespace mdn
