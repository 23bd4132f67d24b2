// Host side of the C ABI declared in include/sol_attn.h: argument checks, workspace layout,
// TMA tensor-map encoding and kernel launches.  Allocates no memory.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "sol_attn.h"

namespace sol {

WorkspaceLayout workspace_layout(long long BH, long long Nk, int d, bool with_split)
{
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t elems = static_cast<size_t>(BH) * static_cast<size_t>(Nk) * static_cast<size_t>(d);
    WorkspaceLayout w{};
    w.kbar32 = kHeaderBytes;
    w.vbar32 = up(w.kbar32 + elems * 4);
    w.kbar16 = up(w.vbar32 + elems * 4);
    w.vbar16 = up(w.kbar16 + elems * 2);
    w.split_part = up(w.vbar16 + elems * 2);
    const long long pairs = BH * ((Nk + 1) / 2);     // tile pairs of the call (Nq = Nk)
    w.split_cap = with_split ? static_cast<int>(std::min<long long>(pairs, kSplitCap)) : 0;
    w.total = up(w.split_part + static_cast<size_t>(w.split_cap) * 2 * kBM * (static_cast<size_t>(d) + 4) * 4);
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

// Device pointers of the pooled arrays and status words for heads [bh0, bh0 + count) of a call
// whose workspace is laid out for the shape `full`.
struct Pooled {
    float *k32, *v32;
    uint8_t *k16, *v16;
    DeviceStatus *status;
    int split_cap;       // the split region serves every head group of a call (one at a time)
    int *split_cnt;
    float *split_part;
    long long call_units;   // tile pairs of the whole call, and of the heads before bh0
    long long unit0;
};

Pooled pooled_at(void *workspace, const Shape &full, int bh0, bool with_split = true)
{
    const WorkspaceLayout wl = workspace_layout(full.BH, full.Nk, full.d, with_split);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t off = static_cast<size_t>(bh0) * static_cast<size_t>(full.Nk) * static_cast<size_t>(full.d);
    Pooled p{};
    p.k32 = reinterpret_cast<float *>(ws + wl.kbar32) + off;
    p.v32 = reinterpret_cast<float *>(ws + wl.vbar32) + off;
    p.k16 = ws + wl.kbar16 + off * 2;
    p.v16 = ws + wl.vbar16 + off * 2;
    p.status = reinterpret_cast<DeviceStatus *>(ws);
    p.split_cap = wl.split_cap;
    p.split_cnt = reinterpret_cast<int *>(ws + kSplitCntOffset);
    p.split_part = reinterpret_cast<float *>(ws + wl.split_part);
    const long long pairs = (full.Nq + 1) / 2;
    p.call_units = static_cast<long long>(full.BH) * pairs;
    p.unit0 = static_cast<long long>(bh0) * pairs;
    return p;
}

// Bytes at the start of the workspace that every call clears: the status words and the split
// counters (the kernel also returns each counter it uses to zero).
constexpr size_t kClearBytes = kSplitCntOffset + 4 * static_cast<size_t>(kSplitCap);

// Pool K, V of the s.BH heads starting at k, v into `pw` (no argument checks); with clear_header
// the pool kernel also zeroes the workspace header's status words and split counters.
sol_status launch_pool(const void *k, const void *v, const Shape &s, const Pooled &pw, cudaStream_t stream,
                       bool clear_header)
{
    int *clear = clear_header ? reinterpret_cast<int *>(pw.status) : nullptr;
    return launch_pool_kv(k, v, s.BH, s.N, s.Nk, s.d, pw.k32, pw.v32, pw.k16, pw.v16, clear,
                          static_cast<int>(kClearBytes / 4), stream) == cudaSuccess
               ? SOL_OK : SOL_ERR_CUDA;
}

// Fused forward over the s.BH heads starting at q, k, v, out, density (no argument checks).
sol_status launch_fwd(const void *q, const void *k, const void *v, const Shape &s, const Pooled &pw,
                      float beta, const float *beta_head, void *out, int32_t *density,
                      float *dbg_proxy, uint8_t *dbg_mask, float *dbg_stats, int fault_flags,
                      unsigned long long timeout_ns, cudaStream_t stream, const RouteArg &ra)
{
    CUtensorMap tq, tk, tv, tkb, tvb;
    if (!encode_rows(&tq, q, s.N, s.BH, 128, s.d) || !encode_rows(&tk, k, s.N, s.BH, kTile, s.d) ||
        !encode_rows(&tv, v, s.N, s.BH, kTile, s.d) || !encode_rows(&tkb, pw.k16, s.Nk, s.BH, kTile, s.d) ||
        !encode_rows(&tvb, pw.v16, s.Nk, s.BH, kTile, s.d))
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
    L.kbar32 = pw.k32;
    L.out = out;
    L.density = density;
    L.status = pw.status;
    L.dbg_proxy = dbg_proxy;
    L.dbg_mask = dbg_mask;
    L.dbg_stats = dbg_stats;
    L.fault_flags = fault_flags;
    L.timeout_ns = timeout_ns;
    L.route = ra.route;
    L.topk = ra.topk;
    L.topp = ra.topp;
    L.split_cap = pw.split_cap;
    L.split_cnt = pw.split_cnt;
    L.split_part = pw.split_part;
    L.split_all = (fault_flags & 2) != 0;
    L.call_units = pw.call_units;
    L.unit0 = pw.unit0;
    return launch_sol_fwd(L, stream) == cudaSuccess ? SOL_OK : SOL_ERR_CUDA;
}

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
    return launch_fwd(q, k, v, s, pooled_at(workspace, s, 0), beta, beta_head, out, density, dbg_proxy,
                      dbg_mask, dbg_stats, fault_flags, timeout_ns, stream, ra);
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

// Copy streams and events of the pipelined host entry point: one set per device, created on first
// use and kept until the process exits.  A call uses about one head group per kHostGroupBytes of
// upload, at most kHostGroups when a head's tile pairs leave their last wave of CTAs at least 90 %
// full, else at most kHostGroupsRagged: each group's launch ends in that partly empty wave, which a
// compute-bound call pays once per group.  Measured on B200 (host link ~55 GB/s each way, ~71 GB/s
// both ways at once; with 8 / 16 / 32 groups): 32 heads x 262144 tokens (6.4 GB up, 2048 tile
// pairs per head = 6.92 waves of 296 CTAs) 140.5 / 131.5 / 130.0 ms; 40 x 75600 (591 pairs,
// 2.00 waves) 50.1 / 48.2 / 47.7; 24 x 118800 (929 pairs, 3.14 waves) 58.0 / 58.8 / 61.7; 12 x 16384
// (151 MB up) ran best with 5 groups.
constexpr int kHostGroups = 32;
constexpr int kHostGroupsRagged = 8;
constexpr size_t kHostGroupBytes = 32u << 20;

struct HostPipe {
    std::once_flag once;
    std::mutex mu;          // one enqueue at a time per device (the events are reused)
    cudaError_t err = cudaSuccess;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t uploaded[kHostGroups] = {};
    cudaEvent_t computed[kHostGroups] = {};
    int slots = 0;          // CTAs of the fused kernel resident at once (two per SM)
};

HostPipe g_host_pipes[64];

HostPipe *host_pipe()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    HostPipe &hp = g_host_pipes[dev];
    std::call_once(hp.once, [&hp, dev] {
        auto event = [&hp](cudaEvent_t *e) {
            if (hp.err == cudaSuccess) hp.err = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
        };
        hp.err = cudaStreamCreateWithFlags(&hp.up, cudaStreamNonBlocking);
        if (hp.err == cudaSuccess) hp.err = cudaStreamCreateWithFlags(&hp.down, cudaStreamNonBlocking);
        event(&hp.start);
        event(&hp.done);
        for (int g = 0; g < kHostGroups; ++g) {
            event(&hp.uploaded[g]);
            event(&hp.computed[g]);
        }
        int sms = 0;
        if (hp.err == cudaSuccess) hp.err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        hp.slots = 2 * sms;
    });
    return hp.err == cudaSuccess ? &hp : nullptr;
}

}  // namespace

// Pool + forward in a workspace laid out without the split region (the no-alloc entry point's
// fixed scratch): the same kernels, no tile pair split over two CTAs.
sol_status pool_fwd_unsplit(const void *q, const void *k, const void *v, int B, int H, int N, int d,
                            float beta, void *workspace, void *out, int32_t *density, cudaStream_t stream)
{
    Shape s{};
    sol_status st = check_shape(B, H, N, d, &s);
    if (st != SOL_OK) return st;
    if (std::isnan(beta)) return SOL_ERR_INVALID_ARG;
    st = check_ptrs({q, k, v, workspace, out});
    if (st != SOL_OK) return st;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SOL_ERR_ALIGNMENT;
    if (density && (reinterpret_cast<uintptr_t>(density) & 3u)) return SOL_ERR_ALIGNMENT;
    const Pooled pw = pooled_at(workspace, s, 0, false);
    st = launch_pool(k, v, s, pw, stream, true);
    if (st != SOL_OK) return st;
    return launch_fwd(q, k, v, s, pw, beta, nullptr, out, density, nullptr, nullptr, nullptr, 0,
                      kDefaultTimeoutNs, stream, RouteArg{});
}

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
    return launch_pool(k, v, s, pooled_at(workspace, s, 0), cs, true);
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
    // NULL: the status words of sol_attn_fwd_noalloc's built-in scratch on the current device
    if (!workspace && noalloc_scratch(&workspace) != cudaSuccess) return SOL_ERR_CUDA;
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
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SOL_ERR_ALIGNMENT;
    if (d_density && (reinterpret_cast<uintptr_t>(d_density) & 3u)) return SOL_ERR_ALIGNMENT;
    if (std::isnan(beta)) return SOL_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    HostPipe *hp = host_pipe();
    if (!hp) return SOL_ERR_CUDA;
    std::lock_guard<std::mutex> lock(hp->mu);

    // Heads are split into up to kHostGroups contiguous groups.  Group g's inputs are uploaded on
    // the `up` stream; `stream` pools and runs the forward for g once they have landed (while the
    // next groups upload); its output is downloaded on the `down` stream while later groups
    // compute.  The last download is joined back into `stream`.
    const size_t head_bytes = static_cast<size_t>(s.N) * static_cast<size_t>(s.d) * 2;
    const size_t upload = 3 * head_bytes * static_cast<size_t>(s.BH);
    const long long slots = std::max(1, hp->slots);
    const long long last_wave = ((s.Nq + 1) / 2) % slots;   // a head's tile pairs in its last wave
    const bool full_waves = last_wave == 0 || 10 * last_wave >= 9 * slots;
    const int G = static_cast<int>(std::min<size_t>(
        std::min<size_t>(full_waves ? kHostGroups : kHostGroupsRagged, static_cast<size_t>(s.BH)),
        std::max<size_t>(1, (upload + kHostGroupBytes - 1) / kHostGroupBytes)));
    const size_t head_dens = static_cast<size_t>(s.Nq) * sizeof(int32_t);
    auto fail = [](cudaError_t e) { return e != cudaSuccess; };
    if (fail(cudaMemsetAsync(workspace, 0, kClearBytes, cs)) ||
        fail(cudaEventRecord(hp->start, cs)) || fail(cudaStreamWaitEvent(hp->up, hp->start, 0)) ||
        fail(cudaStreamWaitEvent(hp->down, hp->start, 0)))
        return SOL_ERR_CUDA;
    // An error return after this point still orders the copies already queued on the internal
    // streams before later work on `stream` (best effort: the joins themselves may fail too), so
    // that the caller's buffers are not read or written behind its back.
    auto join_and = [&](sol_status status) {
        if (cudaEventRecord(hp->done, hp->down) == cudaSuccess) cudaStreamWaitEvent(cs, hp->done, 0);
        if (cudaEventRecord(hp->start, hp->up) == cudaSuccess) cudaStreamWaitEvent(cs, hp->start, 0);
        return status;
    };
    // group g covers heads [edge(g), edge(g+1)); the first and the last group get half the weight
    // of the others: the first one's upload delays the compute of a compute-bound call, the last
    // one's compute and download follow the last upload of a link-bound one
    auto edge = [&](int g) -> int {
        if (G < 3) return static_cast<int>(static_cast<long long>(s.BH) * g / G);
        const long long wsum = 2LL * (G - 1);                               // weights 1, 2, .., 2, 1
        const long long wbefore = g == 0 ? 0 : (g == G ? wsum : 2LL * g - 1);
        return static_cast<int>((static_cast<long long>(s.BH) * wbefore + wsum / 2) / wsum);
    };
    for (int g = 0; g < G; ++g) {
        const int h0 = edge(g);
        const int h1 = edge(g + 1);
        if (h1 <= h0) continue;
        const size_t off = static_cast<size_t>(h0) * head_bytes;
        const size_t bytes = static_cast<size_t>(h1 - h0) * head_bytes;
        uint8_t *gq = static_cast<uint8_t *>(d_q) + off;
        uint8_t *gk = static_cast<uint8_t *>(d_k) + off;
        uint8_t *gv = static_cast<uint8_t *>(d_v) + off;
        uint8_t *go = static_cast<uint8_t *>(d_out) + off;
        if (fail(cudaMemcpyAsync(gq, static_cast<const uint8_t *>(h_q) + off, bytes, cudaMemcpyHostToDevice, hp->up)) ||
            fail(cudaMemcpyAsync(gk, static_cast<const uint8_t *>(h_k) + off, bytes, cudaMemcpyHostToDevice, hp->up)) ||
            fail(cudaMemcpyAsync(gv, static_cast<const uint8_t *>(h_v) + off, bytes, cudaMemcpyHostToDevice, hp->up)) ||
            fail(cudaEventRecord(hp->uploaded[g], hp->up)) || fail(cudaStreamWaitEvent(cs, hp->uploaded[g], 0)))
            return join_and(SOL_ERR_CUDA);
        Shape gs = s;
        gs.BH = h1 - h0;
        const Pooled pw = pooled_at(workspace, s, h0);
        int32_t *gd = d_density ? d_density + static_cast<size_t>(h0) * s.Nq : nullptr;
        st = launch_pool(gk, gv, gs, pw, cs, false);   // the header was cleared once for the call
        if (st == SOL_OK)
            st = launch_fwd(gq, gk, gv, gs, pw, beta, nullptr, go, gd, nullptr, nullptr, nullptr, 0,
                            kDefaultTimeoutNs, cs, RouteArg{});
        if (st != SOL_OK) return join_and(st);
        if (fail(cudaEventRecord(hp->computed[g], cs)) || fail(cudaStreamWaitEvent(hp->down, hp->computed[g], 0)) ||
            fail(cudaMemcpyAsync(static_cast<uint8_t *>(h_out) + off, go, bytes, cudaMemcpyDeviceToHost, hp->down)))
            return join_and(SOL_ERR_CUDA);
        if (h_density &&
            fail(cudaMemcpyAsync(h_density + static_cast<size_t>(h0) * s.Nq, gd,
                                 static_cast<size_t>(h1 - h0) * head_dens, cudaMemcpyDeviceToHost, hp->down)))
            return join_and(SOL_ERR_CUDA);
    }
    if (fail(cudaEventRecord(hp->done, hp->down)) || fail(cudaStreamWaitEvent(cs, hp->done, 0)))
        return join_and(SOL_ERR_CUDA);
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
