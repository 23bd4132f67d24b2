// Internal launch interface between the C-ABI host code and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace sol {

constexpr int kMaxHeadDim = 128;     // head dimensions d = 64 and d = 128 are compiled
inline bool head_dim_supported(int d) { return d == 64 || d == 128; }
constexpr int kTile = 64;            // query tile / key block length T
constexpr int kMaxBlocks = 8192;     // Nk limit: two float proxy rows (64 KB) in shared memory
constexpr size_t kHeaderBytes = 1024;  // workspace header: status words, then split counters
constexpr size_t kSplitCntOffset = 256; // first split counter (int) in the header
constexpr int kSplitCap = 128;          // most tile pairs one call splits over two CTAs
static_assert(kSplitCntOffset + 4 * kSplitCap <= kHeaderBytes, "split counters fit the header");
constexpr int kBM = 128;                // rows of one tile pair (two 64-row query tiles)

// Device status words (first bytes of the workspace header).
struct DeviceStatus {
    int code;   // 0 = ok, otherwise a sol_status value
    int where;  // which wait gave up (see WaitSite in sol_fwd.cu)
};

// Workspace carve-up, all offsets in bytes from the workspace base.  split_part holds, for up to
// split_cap tile pairs processed by two CTAs each, both halves' unnormalised output rows with
// their running max and sum: [split_cap][2][128 rows][d + 4] float32 (O[d], max, sum, 2 unused,
// so every row starts 16-byte aligned).
struct WorkspaceLayout {
    size_t kbar32, vbar32, kbar16, vbar16, split_part, total;
    int split_cap;
};
// with_split = false leaves out the split region (split_cap = 0: no tile pair is split).
WorkspaceLayout workspace_layout(long long BH, long long Nk, int d, bool with_split = true);

// clear (or null): block 0 of the pool also zeroes clear[0, clear_words), the workspace header's
// status words and split counters, which the forward that follows in stream order reads.
cudaError_t launch_pool_kv(const void *k, const void *v, int BH, int N, int Nk, int d, float *kbar32,
                           float *vbar32, void *kbar16, void *vbar16, int *clear, int clear_words,
                           cudaStream_t stream);

// Block-selection rule of the routing step.  The page's own rule is the threshold
// mu + beta*sigma; top-k and top-p are the prior-art rules it compares against, run on the same
// proxy row in the same kernel.
enum Route : int { kRouteThreshold = 0, kRouteTopK = 1, kRouteTopP = 2 };

struct FwdLaunch {
    const CUtensorMap *tm_q, *tm_k, *tm_v, *tm_kb, *tm_vb;
    int BH, N, Nk, Nq, d;
    float beta;
    const float *beta_head;   // device [BH] or null
    const float *kbar32;
    void *out;
    int32_t *density;
    DeviceStatus *status;
    float *dbg_proxy;
    uint8_t *dbg_mask;
    float *dbg_stats;
    int fault_flags;
    unsigned long long timeout_ns;
    int route;      // Route
    int topk;       // kRouteTopK: blocks kept per query tile
    float topp;     // kRouteTopP: probability mass covered per query tile
    int split_cap;  // tile pairs the workspace can split (0: none)
    int *split_cnt;       // [split_cap] arrival counters (launch tag << 2 | count); a merging CTA
                          // returns its counter to 0, and a stale tag counts as 0
    float *split_part;    // [split_cap][2][128][d + 4] partial rows
    bool split_all;       // split every tile pair up to split_cap (test entry point)
    long long call_units; // tile pairs of the whole call this launch is part of (its head groups)
    long long unit0;      // the call's index of this launch's first tile pair
};
cudaError_t launch_sol_fwd(const FwdLaunch &L, cudaStream_t stream);

// Device address of sol_attn_fwd_noalloc's built-in scratch on the current device (looked up once
// per device and cached; a failed lookup is not cached, so the next call retries).
cudaError_t noalloc_scratch(void **addr);

}  // namespace sol
