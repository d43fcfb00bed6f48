// Optional per-kernel timing: when enabled, every kernel launch of the
// library is bracketed by a pair of CUDA events recorded on the launch
// stream.  mdn_profile_read synchronises the recorded events and returns, per
// kernel name, the launch count and total device time.  Off by default; the
// events are created on first enable and reused.
#include <mutex>
#include <string.h>

#include "mdn_internal.cuh"

namespace mdn {
namespace {

constexpr int kSlots = 16384;

struct Profiler {
    std::mutex mu;
    bool enabled = false;
    bool created = false;
    cudaEvent_t start[kSlots];
    cudaEvent_t stop[kSlots];
    int kind[kSlots];
    int used = 0;
    double total_ms[kKernelKinds] = {};
    long long launches[kKernelKinds] = {};
};

Profiler& prof() {
    static Profiler p;
    return p;
}

const char* const kNames[kKernelKinds] = {
    "gate_prep", "intra_simt", "inter_simt", "output_simt", "step", "finite_check",
    "chunk_tc", "intra_tc", "inter_tc", "output_tc", "gate_params", "varlen_prep", "bwd_prep", "bwd_states", "bwd_chain",
    "bwd_state_grads", "bwd_local_grads", "bwd_chain_prep",
};

// Fold every recorded pair into the totals (caller holds the lock).
int drain(Profiler& p) {
    for (int i = 0; i < p.used; ++i) {
        if (cudaEventSynchronize(p.stop[i]) != cudaSuccess) return -1;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, p.start[i], p.stop[i]) != cudaSuccess) return -1;
        p.total_ms[p.kind[i]] += ms;
        p.launches[p.kind[i]] += 1;
    }
    p.used = 0;
    return 0;
}

}  // namespace

int prof_begin(KernelKind k, cudaStream_t s) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    if (!p.enabled) return -1;
    if (p.used == kSlots && drain(p) != 0) return -1;
    const int slot = p.used++;
    p.kind[slot] = (int)k;
    cudaEventRecord(p.start[slot], s);
    return slot;
}

void prof_end(int slot, cudaStream_t s) {
    if (slot < 0) return;
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    cudaEventRecord(p.stop[slot], s);
}

}  // namespace mdn

using namespace mdn;

extern "C" {

int mdn_profile_enable(int on) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    if (on && !p.created) {
        for (int i = 0; i < kSlots; ++i) {
            if (cudaEventCreate(&p.start[i]) != cudaSuccess ||
                cudaEventCreate(&p.stop[i]) != cudaSuccess)
                return -1;
        }
        p.created = true;
    }
    const int prev = p.enabled;
    p.enabled = on != 0;
    return prev;
}

int mdn_profile_read(int reset, const char** names, double* total_ms, long long* launches,
                     int capacity) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> g(p.mu);
    if (p.created && drain(p) != 0) return -1;
    int n = 0;
    for (int k = 0; k < kKernelKinds && n < capacity; ++k) {
        if (!p.launches[k]) continue;
        if (names) names[n] = kNames[k];
        if (total_ms) total_ms[n] = p.total_ms[k];
        if (launches) launches[n] = p.launches[k];
        ++n;
    }
    if (reset) {
        memset(p.total_ms, 0, sizeof(p.total_ms));
        memset(p.launches, 0, sizeof(p.launches));
    }
    return n;
}

}  // extern "C"
