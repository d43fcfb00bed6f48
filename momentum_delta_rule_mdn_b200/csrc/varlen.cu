// Variable-length sequences packed along the token axis (cu_seqlens).
//
// The pages treat one sequence per batch row; several sequences of different
// lengths in one call are the plain extension: each sequence is an
// independent recurrence from its own entering state.  The chunkwise kernels
// need every chunk to lie inside one sequence, so the inputs are copied once
// into a chunk-aligned layout: sequence s starts at padded chunk
// cu_c[s] = sum_{s' < s} ceil(len_s' / C), and the rows after its last token
// up to the chunk boundary are steps that change nothing (k = v = q = 0,
// alpha = mu = 1, beta = eta = 0), as for a ragged last chunk.  The chain
// kernels then run one chain per (sequence, head) over that sequence's chunks
// and write o and vt straight back to the packed rows.  The longest chain is
// the pass's critical path, so the setup also ranks the sequences by length:
// the chain kernels start the longest sequences' chains first, and the
// intra-chunk kernel produces their chunks first.
#include "mdn_internal.cuh"

namespace mdn {
namespace {

constexpr int kSetupThreads = 1024;

// Inclusive sum over the block (blockDim.x = kSetupThreads); also returns the total.
__device__ int block_incl_sum(int x, int* warp_tot, int& total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int r = x + (warp > 0 ? warp_tot[warp - 1] : 0);
    total = warp_tot[31];
    __syncthreads();  // warp_tot is reused by the next call
    return r;
}

// Sequences are ranked by chunk count (for the work order) when there are at
// most this many; beyond it they keep their call order.
constexpr int kRankMax = 2048;

__global__ void __launch_bounds__(kSetupThreads)
varlen_setup_kernel(const int* __restrict__ cu, int N, int total_T, int NT, int* __restrict__ cu_s,
                    int* __restrict__ cu_c, int* __restrict__ seq_order,
                    int* __restrict__ chunk_order, unsigned* __restrict__ bad)
{
    __shared__ int warp_tot[32];
    __shared__ int cnt_sh[kRankMax];
    const int tid = threadIdx.x;
    int my_bad = 0;
    for (int i = tid; i <= N; i += kSetupThreads) {
        const int x = cu[i];
        if (i == 0 && x != 0) my_bad = 1;
        if (i == N && x != total_T) my_bad = 1;
        if (i < N && cu[i + 1] < x) my_bad = 1;
    }
    const bool any_bad = __syncthreads_or(my_bad) != 0;
    int carry = 0;
    for (int base = 0; base <= N; base += kSetupThreads) {  // uniform trip count
        const int i = base + tid;
        const int cnt = (!any_bad && i < N) ? (cu[i + 1] - cu[i] + kChunk - 1) / kChunk : 0;
        int total;
        const int incl = block_incl_sum(cnt, warp_tot, total);
        if (i <= N) {
            cu_c[i] = carry + incl - cnt;
            cu_s[i] = any_bad ? 0 : cu[i];
        }
        carry += total;
    }
    if (tid == 0 && any_bad) atomicOr(bad, 1u);
    __syncthreads();  // cu_c is complete

    // seq_order: the sequences by decreasing chunk count (ties in call order)
    if (!any_bad && N <= kRankMax) {
        for (int i = tid; i < N; i += kSetupThreads) cnt_sh[i] = cu_c[i + 1] - cu_c[i];
        __syncthreads();
        for (int i = tid; i < N; i += kSetupThreads) {
            const int ci = cnt_sh[i];
            int rank = 0;
            for (int j = 0; j < N; ++j) {
                const int cj = cnt_sh[j];
                rank += (cj > ci) || (cj == ci && j < i);
            }
            seq_order[rank] = i;
        }
    } else {
        for (int i = tid; i < N; i += kSetupThreads) seq_order[i] = i;
    }
    __syncthreads();
    // chunk_order: the padded chunks of seq_order[0], then of seq_order[1], ...,
    // then the unused padded chunks
    carry = 0;
    for (int base = 0; base < N; base += kSetupThreads) {  // uniform trip count
        const int r = base + tid;
        const int sq = r < N ? seq_order[r] : 0;
        const int cnt = r < N ? cu_c[sq + 1] - cu_c[sq] : 0;
        int total;
        const int incl = block_incl_sum(cnt, warp_tot, total);
        const int start = carry + incl - cnt;
        for (int t = 0; t < cnt; ++t) chunk_order[start + t] = cu_c[sq] + t;
        carry += total;
    }
    for (int j = cu_c[N] + tid; j < NT; j += kSetupThreads) chunk_order[j] = j;
}

// One warp per padded row: the row's H*D values of q, k, v (16-byte units)
// and its H gates.
__global__ void __launch_bounds__(128)
varlen_gather_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                     const uint4* __restrict__ v, int vec_per_row,
                     const float* __restrict__ alpha_log, const float* __restrict__ mu_log,
                     const float* __restrict__ beta, const float* __restrict__ eta,
                     const int* __restrict__ cu_s, const int* __restrict__ cu_c, int N, int H,
                     long long rows, uint4* __restrict__ qp, uint4* __restrict__ kp,
                     uint4* __restrict__ vp, float* __restrict__ alp, float* __restrict__ mlp,
                     float* __restrict__ bep, float* __restrict__ etp)
{
    const int lane = threadIdx.x & 31;
    const long long p = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (p >= rows) return;
    const int n = (int)(p / kChunk), r = (int)(p % kChunk);
    const int seq = varlen_seq_of_chunk(cu_c, N, n);
    long long src = -1;
    if (seq >= 0) {
        const int local = (n - cu_c[seq]) * kChunk + r;
        if (local < cu_s[seq + 1] - cu_s[seq]) src = (long long)cu_s[seq] + local;
    }
    const size_t dst_off = (size_t)p * vec_per_row;
    if (src >= 0) {
        const size_t src_off = (size_t)src * vec_per_row;
        for (int e = lane; e < vec_per_row; e += 32) {
            qp[dst_off + e] = __ldcs(q + src_off + e);
            kp[dst_off + e] = __ldcs(k + src_off + e);
            vp[dst_off + e] = __ldcs(v + src_off + e);
        }
        for (int e = lane; e < H; e += 32) {
            const size_t g = (size_t)src * H + e, d = (size_t)p * H + e;
            alp[d] = alpha_log[g];
            mlp[d] = mu_log[g];
            bep[d] = beta[g];
            etp[d] = eta[g];
        }
    } else {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        for (int e = lane; e < vec_per_row; e += 32) {
            qp[dst_off + e] = z;
            kp[dst_off + e] = z;
            vp[dst_off + e] = z;
        }
        for (int e = lane; e < H; e += 32) {
            const size_t d = (size_t)p * H + e;
            alp[d] = 0.f;  // alpha = 1
            mlp[d] = 0.f;  // mu = 1
            bep[d] = 0.f;
            etp[d] = 0.f;
        }
    }
}

}  // namespace

cudaError_t launch_varlen_setup(const int* cu_seqlens, int N, int total_T, int NT, int* cu_s,
                                int* cu_c, int* seq_order, int* chunk_order, unsigned* bad,
                                cudaStream_t s)
{
    ProfScope ps(kVarlen, s);
    varlen_setup_kernel<<<1, kSetupThreads, 0, s>>>(cu_seqlens, N, total_T, NT, cu_s, cu_c,
                                                     seq_order, chunk_order, bad);
    return cudaGetLastError();
}

cudaError_t launch_varlen_gather(const void* q, const void* k, const void* v, size_t elt,
                                 const float* alpha_log, const float* mu_log, const float* beta,
                                 const float* eta, const int* cu_s, const int* cu_c, int N, int H,
                                 int D, int NT, void* qp, void* kp, void* vp, float* alp,
                                 float* mlp, float* bep, float* etp, cudaStream_t s)
{
    const long long rows = (long long)NT * kChunk;
    if (rows == 0) return cudaSuccess;
    const int vec_per_row = (int)((size_t)H * D * elt / 16);  // D * elt is a multiple of 16
    ProfScope ps(kVarlen, s);
    varlen_gather_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, s>>>(
        static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v),
        vec_per_row, alpha_log, mu_log, beta, eta, cu_s, cu_c, N, H, rows,
        static_cast<uint4*>(qp), static_cast<uint4*>(kp), static_cast<uint4*>(vp), alp, mlp, bep,
        etp);
    return cudaGetLastError();
}

}  // namespace mdn
