// mdn_chunk_fwd_noalloc: the chunkwise forward pass with its scratch space in
// a fixed device array that belongs to the library, for callers that cannot
// allocate device memory themselves.
//
// The array is a file-scope static __device__ object, so every GPU that loads
// this library holds it until the process exits.  In host code its name is
// only a host-side stand-in; the device address is looked up once per device
// with cudaGetSymbolAddress (with that device current) and cached.
#include <mutex>

#include "mdn_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up on the
// first call for that device, then cached).
cudaError_t scratch_on_current_device(void** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> g(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" mdn_status mdn_chunk_fwd_noalloc(
    const void* q, const void* k, const void* v, mdn_dtype in_dtype, const float* alpha_log,
    const float* mu_log, const float* beta, const float* eta, float d_corr, const float* S0,
    const float* M0, int B, int T, int H, int dk, int dv, int C, void* o, void* vtilde,
    float* S_T, float* M_T, int flags, mdn_stream_t stream)
{
    const size_t need =
        mdn_chunk_fwd_workspace_size_flags(B, T, H, dk, dv, C, in_dtype, flags);
    if (need == 0 || B == 0 || H == 0 || T == 0) {
        // Invalid or unsupported sizes (mdn_chunk_fwd's own validation reports
        // them before anything touches a device), or nothing that needs
        // scratch (no heads; T = 0 only copies the states): no array needed.
        return mdn_chunk_fwd(q, k, v, in_dtype, alpha_log, mu_log, beta, eta, d_corr, S0, M0,
                             B, T, H, dk, dv, C, o, vtilde, S_T, M_T, nullptr, 0, flags, stream);
    }
    if (need > kStaticScratchBytes) return MDN_ERR_UNSUPPORTED;
    void* ws = nullptr;
    const cudaError_t e = scratch_on_current_device(&ws);
    if (e != cudaSuccess) return mdn::cuda_fail(e);
    return mdn_chunk_fwd(q, k, v, in_dtype, alpha_log, mu_log, beta, eta, d_corr, S0, M0, B, T,
                         H, dk, dv, C, o, vtilde, S_T, M_T, ws, kStaticScratchBytes, flags,
                         stream);
}
