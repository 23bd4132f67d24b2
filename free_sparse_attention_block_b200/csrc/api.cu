// Host side of the C ABI declared in include/sol_attn.h: argument checks, workspace layout,
// TMA tensor-map encoding and kernel launches.  Allocates no memory.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "sol_attn.h"

namespace sol {

WorkspaceLayout workspace_layout(long long BH, long long Nk, int d)
{
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t elems = static_cast<size_t>(BH) * static_cast<size_t>(Nk) * static_cast<size_t>(d);
    WorkspaceLayout w{};
    w.kbar32 = kHeaderBytes;
    w.vbar32 = up(w.kbar32 + elems * 4);
    w.kbar16 = up(w.vbar32 + elems * 4);
    w.vbar16 = up(w.kbar16 + elems * 2);
    w.total = up(w.vbar16 + elems * 2);
    return w;
}

namespace {

constexpr int kMaxN = kMaxBlocks * kTile;   // 524288

struct Shape {
    int BH, N, Nk, Nq, d;
};

sol_status check_shape(int B, int H, int N, int d, Shape *s)
{
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return SOL_ERR_INVALID_ARG;
    if (!head_dim_supported(d)) return SOL_ERR_UNSUPPORTED;
    if (N > kMaxN) return SOL_ERR_UNSUPPORTED;
    const long long BH = static_cast<long long>(B) * H;
    const long long Nk = (N + kTile - 1) / kTile;
    if (BH > 0x7FFFFFFFLL || BH * ((Nk + 1) / 2) > 0x7FFFFFFFLL) return SOL_ERR_INVALID_ARG;
    s->BH = static_cast<int>(BH);
    s->N = N;
    s->Nk = static_cast<int>(Nk);
    s->Nq = static_cast<int>(Nk);
    s->d = d;
    return SOL_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sol_status check_ptrs(std::initializer_list<const void *> ptrs)
{
    for (const void *p : ptrs)
        if (!p) return SOL_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned16(p)) return SOL_ERR_ALIGNMENT;
    return SOL_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 3-D bf16 map over [BH][rows][d] with a {64 channels, box_rows} box, 128-byte swizzle and
// zero fill outside the tensor (rows past the end read as 0).
bool encode_rows(CUtensorMap *map, const void *base, long long rows, int BH, int box_rows, int d)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                             static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Routing rule and its parameter for one call.
struct RouteArg {
    int route = kRouteThreshold;
    int topk = 0;
    float topp = 0.0f;
};

sol_status run_fwd(const void *q, const void *k, const void *v, int B, int H, int N, int d,
                   float beta, const float *beta_head, void *workspace, void *out, int32_t *density,
                   float *dbg_proxy, uint8_t *dbg_mask, float *dbg_stats, int fault_flags,
                   unsigned long long timeout_ns, cudaStream_t stream, RouteArg ra = RouteArg{})
{
    Shape s{};
    sol_status st = check_shape(B, H, N, d, &s);
    if (st != SOL_OK) return st;
    if (std::isnan(beta)) return SOL_ERR_INVALID_ARG;
    st = check_ptrs({q, k, v, workspace, out});
    if (st != SOL_OK) return st;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SOL_ERR_ALIGNMENT;
    if (density && (reinterpret_cast<uintptr_t>(density) & 3u)) return SOL_ERR_ALIGNMENT;
    if (beta_head && (reinterpret_cast<uintptr_t>(beta_head) & 3u)) return SOL_ERR_ALIGNMENT;

    const WorkspaceLayout wl = workspace_layout(s.BH, s.Nk, s.d);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    CUtensorMap tq, tk, tv, tkb, tvb;
    if (!encode_rows(&tq, q, s.N, s.BH, 128, s.d) || !encode_rows(&tk, k, s.N, s.BH, kTile, s.d) ||
        !encode_rows(&tv, v, s.N, s.BH, kTile, s.d) ||
        !encode_rows(&tkb, ws + wl.kbar16, s.Nk, s.BH, kTile, s.d) ||
        !encode_rows(&tvb, ws + wl.vbar16, s.Nk, s.BH, kTile, s.d))
        return SOL_ERR_CUDA;
    FwdLaunch L{};
    L.tm_q = &tq;
    L.tm_k = &tk;
    L.tm_v = &tv;
    L.tm_kb = &tkb;
    L.tm_vb = &tvb;
    L.BH = s.BH;
    L.N = s.N;
    L.Nk = s.Nk;
    L.Nq = s.Nq;
    L.d = s.d;
    L.beta = beta;
    L.beta_head = beta_head;
    L.kbar32 = reinterpret_cast<const float *>(ws + wl.kbar32);
    L.out = out;
    L.density = density;
    L.status = reinterpret_cast<DeviceStatus *>(ws);
    L.dbg_proxy = dbg_proxy;
    L.dbg_mask = dbg_mask;
    L.dbg_stats = dbg_stats;
    L.fault_flags = fault_flags;
    L.timeout_ns = timeout_ns;
    L.route = ra.route;
    L.topk = ra.topk;
    L.topp = ra.topp;
    return launch_sol_fwd(L, stream) == cudaSuccess ? SOL_OK : SOL_ERR_CUDA;
}

constexpr unsigned long long kDefaultTimeoutNs = 2000ull * 1000ull * 1000ull;   // 2 s

// Validates a rule and its parameter: top-k needs k >= 0 (values above Nk keep every block),
// top-p a non-NaN p (<= 0 keeps none, >= 1 keeps every block).
sol_status route_arg(int route, double param, RouteArg *ra)
{
    ra->route = route;
    switch (route) {
    case kRouteThreshold:
        return std::isnan(param) ? SOL_ERR_INVALID_ARG : SOL_OK;
    case kRouteTopK:
        if (std::isnan(param) || param < 0.0 || param != std::floor(param)) return SOL_ERR_INVALID_ARG;
        ra->topk = param > 1e9 ? 1000000000 : static_cast<int>(param);
        return SOL_OK;
    case kRouteTopP:
        if (std::isnan(param)) return SOL_ERR_INVALID_ARG;
        ra->topp = static_cast<float>(param);
        return SOL_OK;
    }
    return SOL_ERR_INVALID_ARG;
}

}  // namespace
}  // namespace sol

using namespace sol;

extern "C" {

size_t sol_attn_workspace_bytes(int B, int H, int N, int d)
{
    Shape s{};
    if (check_shape(B, H, N, d, &s) != SOL_OK) return 0;
    return workspace_layout(s.BH, s.Nk, s.d).total;
}

sol_status sol_attn_pool(const void *k, const void *v, int B, int H, int N, int d,
                         void *workspace, void *stream)
{
    Shape s{};
    sol_status st = check_shape(B, H, N, d, &s);
    if (st != SOL_OK) return st;
    st = check_ptrs({k, v, workspace});
    if (st != SOL_OK) return st;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SOL_ERR_ALIGNMENT;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const WorkspaceLayout wl = workspace_layout(s.BH, s.Nk, s.d);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (cudaMemsetAsync(ws, 0, sizeof(DeviceStatus), cs) != cudaSuccess) return SOL_ERR_CUDA;
    cudaError_t e = launch_pool_kv(k, v, s.BH, s.N, s.Nk, s.d, reinterpret_cast<float *>(ws + wl.kbar32),
                                   reinterpret_cast<float *>(ws + wl.vbar32), ws + wl.kbar16,
                                   ws + wl.vbar16, cs);
    return e == cudaSuccess ? SOL_OK : SOL_ERR_CUDA;
}

sol_status sol_attn_fwd(const void *q, const void *k, const void *v, int B, int H, int N, int d,
                        float beta, void *workspace, void *out, int32_t *density_out, void *stream)
{
    return run_fwd(q, k, v, B, H, N, d, beta, nullptr, workspace, out, density_out, nullptr,
                   nullptr, nullptr, 0, kDefaultTimeoutNs, static_cast<cudaStream_t>(stream));
}

sol_status sol_attn_fwd_betas(const void *q, const void *k, const void *v, int B, int H, int N,
                              int d, const float *beta_per_head, void *workspace, void *out,
                              int32_t *density_out, void *stream)
{
    if (!beta_per_head) return SOL_ERR_INVALID_ARG;
    return run_fwd(q, k, v, B, H, N, d, 0.0f, beta_per_head, workspace, out, density_out, nullptr,
                   nullptr, nullptr, 0, kDefaultTimeoutNs, static_cast<cudaStream_t>(stream));
}

sol_status sol_attn_fwd_topk(const void *q, const void *k, const void *v, int B, int H, int N,
                             int d, int k_blocks, void *workspace, void *out, int32_t *density_out,
                             void *stream)
{
    RouteArg ra;
    const sol_status st = route_arg(kRouteTopK, static_cast<double>(k_blocks), &ra);
    if (st != SOL_OK) return st;
    return run_fwd(q, k, v, B, H, N, d, 0.0f, nullptr, workspace, out, density_out, nullptr,
                   nullptr, nullptr, 0, kDefaultTimeoutNs, static_cast<cudaStream_t>(stream), ra);
}

sol_status sol_attn_fwd_topp(const void *q, const void *k, const void *v, int B, int H, int N,
                             int d, float p, void *workspace, void *out, int32_t *density_out,
                             void *stream)
{
    RouteArg ra;
    const sol_status st = route_arg(kRouteTopP, static_cast<double>(p), &ra);
    if (st != SOL_OK) return st;
    return run_fwd(q, k, v, B, H, N, d, 0.0f, nullptr, workspace, out, density_out, nullptr,
                   nullptr, nullptr, 0, kDefaultTimeoutNs, static_cast<cudaStream_t>(stream), ra);
}

sol_status sol_attn_fwd_debug_route(const void *q, const void *k, const void *v, int B, int H,
                                    int N, int d, int route, float param, void *workspace,
                                    void *out, int32_t *density_out, float *proxy_out,
                                    uint8_t *mask_out, float *stats_out, void *stream)
{
    if ((proxy_out && !aligned16(proxy_out)) || (stats_out && !aligned16(stats_out)))
        return SOL_ERR_ALIGNMENT;
    RouteArg ra;
    sol_status st = route_arg(route, static_cast<double>(param), &ra);
    if (st != SOL_OK) return st;
    const float beta = route == kRouteThreshold ? param : 0.0f;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    st = run_fwd(q, k, v, B, H, N, d, beta, nullptr, workspace, out, density_out, proxy_out,
                 mask_out, stats_out, 0, kDefaultTimeoutNs, cs, ra);
    if (st != SOL_OK) return st;
    return sol_attn_read_status(workspace, nullptr, stream);
}

sol_status sol_attn_read_status(void *workspace, int *where_out, void *stream)
{
    if (!workspace) return SOL_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(cs) != cudaSuccess) return SOL_ERR_CUDA;
    DeviceStatus h{};
    if (cudaMemcpy(&h, workspace, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return SOL_ERR_CUDA;
    if (cudaMemset(workspace, 0, sizeof h) != cudaSuccess) return SOL_ERR_CUDA;
    if (where_out) *where_out = h.where;
    if (h.code == 0) return SOL_OK;
    return h.code == SOL_ERR_TIMEOUT ? SOL_ERR_TIMEOUT : SOL_ERR_CUDA;
}

sol_status sol_attn_fwd_debug(const void *q, const void *k, const void *v, int B, int H, int N,
                              int d, float beta, void *workspace, void *out,
                              int32_t *density_out, float *proxy_out, uint8_t *mask_out,
                              float *stats_out, int fault_flags, int timeout_ms, void *stream)
{
    if ((proxy_out && !aligned16(proxy_out)) || (stats_out && !aligned16(stats_out)))
        return SOL_ERR_ALIGNMENT;
    const unsigned long long tns =
        timeout_ms > 0 ? static_cast<unsigned long long>(timeout_ms) * 1000000ull : kDefaultTimeoutNs;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    sol_status st = run_fwd(q, k, v, B, H, N, d, beta, nullptr, workspace, out, density_out,
                            proxy_out, mask_out, stats_out, fault_flags, tns, cs);
    if (st != SOL_OK) return st;
    return sol_attn_read_status(workspace, nullptr, stream);
}

sol_status sol_attn_fwd_host(const void *h_q, const void *h_k, const void *h_v, int B, int H,
                             int N, int d, float beta, void *d_q, void *d_k, void *d_v,
                             void *workspace, void *d_out, int32_t *d_density, void *h_out,
                             int32_t *h_density, void *stream)
{
    Shape s{};
    sol_status st = check_shape(B, H, N, d, &s);
    if (st != SOL_OK) return st;
    if (!h_q || !h_k || !h_v || !h_out || ((h_density == nullptr) != (d_density == nullptr)))
        return SOL_ERR_INVALID_ARG;
    st = check_ptrs({d_q, d_k, d_v, workspace, d_out});
    if (st != SOL_OK) return st;
    if (std::isnan(beta)) return SOL_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const size_t bytes = static_cast<size_t>(s.BH) * s.N * s.d * 2;
    if (cudaMemcpyAsync(d_q, h_q, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(d_k, h_k, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(d_v, h_v, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return SOL_ERR_CUDA;
    st = sol_attn_pool(d_k, d_v, B, H, N, d, workspace, stream);
    if (st != SOL_OK) return st;
    st = sol_attn_fwd(d_q, d_k, d_v, B, H, N, d, beta, workspace, d_out, d_density, stream);
    if (st != SOL_OK) return st;
    if (cudaMemcpyAsync(h_out, d_out, bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess) return SOL_ERR_CUDA;
    if (h_density &&
        cudaMemcpyAsync(h_density, d_density, static_cast<size_t>(s.BH) * s.Nq * sizeof(int32_t),
                        cudaMemcpyDeviceToHost, cs) != cudaSuccess)
        return SOL_ERR_CUDA;
    return SOL_OK;
}

const char *sol_attn_error_string(sol_status status)
{
    switch (status) {
    case SOL_OK: return "success";
    case SOL_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size or NaN beta)";
    case SOL_ERR_UNSUPPORTED: return "unsupported shape (head dim must be 64 or 128, N <= 524288)";
    case SOL_ERR_ALIGNMENT: return "pointer not aligned (tensors 16 B, workspace 256 B)";
    case SOL_ERR_CUDA: return "CUDA call or kernel launch failed";
    case SOL_ERR_TIMEOUT: return "a device pipeline wait timed out";
    case SOL_ERR_SCRATCH_LIMIT: return "shape needs more than the no-alloc scratch (SOL_ATTN_NOALLOC_MAX_BYTES)";
    }
    return "unknown status";
}

}  // extern "C"
