// Helpers shared by the tensor-core chunk kernels (intra and inter).
#pragma once

#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

#include "sm100.cuh"

namespace mdn {
namespace tc {

constexpr int C = 64;          // chunk length
constexpr int D = 128;         // d_k = d_v
constexpr int LDF = 68;        // leading dimension of fp32 64x64 matrices (16-byte rows)

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
// Eight fp32 values -> one 16-byte chunk of bf16.
__device__ __forceinline__ uint4 bf16x8(const float* x) {
    return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                      pack_bf16(x[6], x[7]));
}
// Four floats as four bf16 (round to nearest even), packed for an 8-byte store.
__device__ __forceinline__ uint2 bf16x4(const float* x) {
    return make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
}
__device__ __forceinline__ void unpack_bf16x4(const uint2 w, float* x) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&w.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w.y);
    x[0] = __low2float(a);
    x[1] = __high2float(a);
    x[2] = __low2float(b);
    x[3] = __high2float(b);
}
__device__ __forceinline__ void st_bf16x8(uint8_t* p, const float* x) {
    *reinterpret_cast<uint4*>(p) = bf16x8(x);
}
// 16-byte chunk of bf16 -> eight fp32 values.
__device__ __forceinline__ void unpack_bf16x8(const uint4 w, float* x) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&u[e]);
        x[2 * e] = __low2float(v);
        x[2 * e + 1] = __high2float(v);
    }
}
__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Arrive on a named barrier without waiting (the producers' side).
__device__ __forceinline__ void named_bar_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also ANDs a predicate over its threads.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sm100::smem_u32(bar)) : "memory");
}
// True in exactly one (the lowest) active lane of the warp.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "elect.sync _|P, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}\n"
        : "=r"(pred));
    return pred != 0;
}
__device__ __forceinline__ long long clock_now() {
    long long t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
    return t;
}
// Cycle counts of a kernel's phases, summed over chunks in registers and
// written out once.  Diagnostic builds only (MDN_PHASE_CLOCKS); otherwise
// every call is empty and costs nothing.
#ifdef MDN_PHASE_CLOCKS
struct PhaseClock {
    static constexpr int kMax = 20;
    float* out;
    long long t;
    float acc[kMax];
    __device__ __forceinline__ void start(float* o) {
        out = o;
#pragma unroll
        for (int k = 0; k < kMax; ++k) acc[k] = 0.f;
        t = clock_now();
    }
    __device__ __forceinline__ void lap(int k) {
        if (out) {
            const long long now = clock_now();
            acc[k] += (float)(now - t);
            t = now;
        }
    }
    __device__ __forceinline__ void flush() {
        if (out)
            for (int k = 0; k < kMax; ++k) out[k] += acc[k];
    }
};
#else
struct PhaseClock {
    __device__ __forceinline__ void start(float*) {}
    __device__ __forceinline__ void lap(int) {}
    __device__ __forceinline__ void flush() {}
};
#endif

// ------------------------------------------------------------------ host side
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 4-D map over a [B, T, H, D] bf16 tensor; box = {box_d, 1, 64, 1}.
inline bool make_token_map(CUtensorMap* map, const void* base, int B, int T, int H, int box_d,
                           bool swizzle128)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// 3-D map over per-chunk bf16 matrices [chunks, rows, cols]; box = {64, box_rows, 1}, 128B swizzle.
inline bool make_chunk_map(CUtensorMap* map, const void* base, long long chunks, int rows, int cols,
                           int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)chunks};
    cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)rows * cols * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace mdn
