// sol_attn_fwd_noalloc: the pool + fused forward for callers that must not allocate device memory
// (for example code that runs inside a fixed device-memory budget, a host framework whose
// allocator may not be re-entered from this call, or a plugin that owns no allocator of its own).
// Its scratch, the pooled keys/values and the status words that sol_attn_pool/sol_attn_fwd keep
// in a caller-provided workspace, lives in one file-scope device array instead.
//
// The array is a host-side stand-in for a device symbol: host code must never pass its name to a
// kernel.  Its device address is obtained once per device with cudaGetSymbolAddress, with that
// device current, and cached once the lookup succeeds.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "sol_attn.h"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[SOL_ATTN_NOALLOC_MAX_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
std::atomic<void *> g_addr[kMaxDevices];

sol_status shape_error(int B, int H, int N, int d)
{
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return SOL_ERR_INVALID_ARG;
    if (!sol::head_dim_supported(d) || N > sol::kMaxBlocks * sol::kTile) return SOL_ERR_UNSUPPORTED;
    return SOL_ERR_INVALID_ARG;
}

}  // namespace

namespace sol {
sol_status pool_fwd_unsplit(const void *q, const void *k, const void *v, int B, int H, int N, int d,
                            float beta, void *workspace, void *out, int32_t *density, cudaStream_t stream);

cudaError_t noalloc_scratch(void **addr)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void *a = g_addr[dev].load(std::memory_order_acquire);
    if (!a) {
        // Only a successful lookup is cached: one made during a stream capture, or after a
        // transient error, is retried by the next call.
        std::lock_guard<std::mutex> lock(g_mu);
        a = g_addr[dev].load(std::memory_order_relaxed);
        if (!a) {
            e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
            if (e != cudaSuccess || !a) {
                cudaGetLastError();   // do not leave the error for a later launch check to report
                return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
            }
            g_addr[dev].store(a, std::memory_order_release);
        }
    }
    *addr = a;
    return cudaSuccess;
}
}  // namespace sol

extern "C" sol_status sol_attn_fwd_noalloc(const void *q, const void *k, const void *v, int B,
                                           int H, int N, int d, float beta, void *out,
                                           int32_t *density_out, void *stream)
{
    if (sol_attn_workspace_bytes(B, H, N, d) == 0) return shape_error(B, H, N, d);   // bad shape
    const long long BH = static_cast<long long>(B) * H;
    const long long Nk = (N + sol::kTile - 1) / sol::kTile;
    const size_t need = sol::workspace_layout(BH, Nk, d, false).total;
    if (need > SOL_ATTN_NOALLOC_MAX_BYTES) return SOL_ERR_SCRATCH_LIMIT;

    void *scratch = nullptr;
    if (sol::noalloc_scratch(&scratch) != cudaSuccess) return SOL_ERR_CUDA;

    // The pool clears the status words and overwrites every pooled row the forward reads, so
    // nothing left in the array by an earlier call is used.  The scratch has no split region.
    return sol::pool_fwd_unsplit(q, k, v, B, H, N, d, beta, scratch, out, density_out,
                                 static_cast<cudaStream_t>(stream));
}
