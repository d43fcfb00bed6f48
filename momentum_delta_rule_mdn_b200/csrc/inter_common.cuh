// Pieces shared by the inter-chunk (K-3) kernels: their argument block and the
// bounded waits every role uses.
#pragma once

#include "mdn_internal.cuh"
#include "tc_common.cuh"

namespace mdn {
namespace inter {

using namespace sm100;
using namespace tc;

struct InterArgs {
    const float* crec;
    const unsigned* ready;  // [chunks] set by the intra-chunk kernel once a chunk is written
    const float* S0;
    const float* M0;
    float* S_T;
    float* M_T;
    __nv_bfloat16* o;
    __nv_bfloat16* vt;
    unsigned* status;
    float* dbg;  // diagnostics: phase clocks of the MMA and load lanes of CTA 0 (null in normal use)
    int T, H, NT;
    const int* cu_seqlens;  // variable-length mode (see ChunkArgs); null otherwise
    const int* cu_chunks;
    const int* seq_order;
};

constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s

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
// Wait until the intra-chunk kernel has published a chunk (it may still be
// running: this kernel is launched as its programmatic dependent).  Gives up
// like wait_bar.
__device__ __forceinline__ bool wait_ready(const unsigned* flag, volatile int* abort_flag) {
    if (ld_acquire_gpu(flag) != 0u) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        __nanosleep(64);
        if (ld_acquire_gpu(flag) != 0u) return true;
        if ((i & 15u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitNs || i > (1u << 24)) {
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Warp-uniform form: every lane waits, and the warp agrees on the outcome.
// Warp-uniform form: every lane waits, and the warp agrees on the outcome.
// (Polling from one lane and broadcasting the result was measured slower on
// the 32-column chains: it adds a shuffle and a second probe to every hand-off
// on their critical path.)
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, wait_bar(bar, parity, abort_flag));
}

// Fills the argument block from a chunk pass's arguments.
inline InterArgs inter_args(const ChunkArgs& a)
{
    InterArgs t;
    t.crec = a.crec;
    t.ready = a.ready;
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
    t.cu_seqlens = a.cu_seqlens;
    t.cu_chunks = a.cu_chunks;
    t.seq_order = a.seq_order;
    return t;
}

}  // namespace inter
}  // namespace mdn
