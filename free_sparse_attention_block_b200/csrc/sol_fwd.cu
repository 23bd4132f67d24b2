// Fused Sol-Attn forward for sm_100a: routing, exact block-sparse attention and the pooled
// correction of skipped blocks in one online-softmax pass.
//
// Source: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
// Sparsification" (Li et al., 2026): the routing paragraphs (per-query proxy scores against key
// blocks, their mean mu and standard deviation sigma, keep a block iff its score >= mu +
// beta*sigma) and the paragraph on the fused operator (routing is not a separate pass before the
// sparse attention, and skipped blocks are approximated rather than dropped).
//
// One CTA owns one 128-row MMA tile = two adjacent 64-row routing tiles (A: rows 0-63, B: rows
// 64-127) of one head.  Two CTAs fit on an SM (about 110 KB of shared memory at d = 128, 94 KB at
// d = 64, and 256 TMEM columns each), so one CTA's routing and softmax overlap the other's
// tensor-core work.  The kernel is compiled for head dimensions d = 128 and d = 64 (template
// parameter D), and for the threshold rule or the top-k / top-p rules (template parameter kRank).
//
//  1. Routing (all 6 warps).  TMA brings the Q tile into shared memory; q_bar of each routing
//     tile is summed from it in float32; every warp computes proxy scores
//     S_j = (q_bar . k_bar_j) / sqrt(d) for its key blocks (float32 k_bar_j read from the pooled
//     workspace) into two shared-memory rows that alias the K/V ring; mu and sigma are reduced in
//     double with warp shuffles; blocks with S_j >= tau become bit masks (tile A, tile B, union).
//     The proxy rows never reach global memory (except through the debug outputs).
//  2. Pipeline.  Work items are first the 64-wide chunks of pooled blocks that still hold a
//     skipped block (the correction), then every block kept by tile A or tile B (the exact part).
//     Warp 4 (one lane) streams the item's 64 x d K and V tiles by TMA into a 2-stage ring.
//     Warp 5 (one lane) issues S = Q K^T (M=128, N=64, K=d) into TMEM, and once the softmax has
//     written P, O += P V (M=128, N=d, K=64) with P read straight from TMEM.
//     Warps 0-3 (one thread per row) load S from TMEM, apply the per-row routing decision
//     (a row of tile A ignores blocks only tile B kept, and vice versa; a correction column is
//     -inf if the row's tile kept that block, else its logit gets + log2(n_j)), keep a running
//     max (rescaling O in TMEM only when the max grows by more than 2^8), and store P as bf16
//     over the first 32 columns of the same TMEM buffer.
//  3. Epilogue: O / l rounded to bf16 and written to global memory.
//
// Every mbarrier wait is bounded (globaltimer): on expiry the CTA records SOL_ERR_TIMEOUT and the
// wait site in the workspace status words, sets a shared abort flag, lets in-flight TMA copies
// and MMAs land, frees its TMEM and exits.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstddef>
#include <mutex>

#include <type_traits>

#include "internal.h"
#include "sm100.cuh"

namespace sol {
namespace {

constexpr int kThreads = 192;
constexpr int kNumWarps = 6;
constexpr int kSoftmaxThreads = 128;   // warps 0-3: one thread per row (TMEM lane)
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;

constexpr uint32_t kQHalfBytes = kBM * 64 * 2;         // 128 rows x 64 channels, bf16
constexpr uint32_t kKVHalfBytes = kTile * 64 * 2;      // 64 rows x 64 channels, bf16
constexpr int kStages = 2;

constexpr uint32_t kTmemCols = 256;
constexpr int kMaxSBufs = 3;
__device__ __forceinline__ uint32_t tmem_s_col(int b) { return 64u * static_cast<uint32_t>(b); }

constexpr float kRescaleLog2 = 8.0f;                   // rescale O only if the max grows > 2^8

// Of the 32 column pairs of a row, this many take exp2 on the FMA pipe (exp2_poly2) and the rest
// on the MUFU unit.  Measured on the mid workload (beta 0.5): 0 pairs 0.592 ms, 6: 0.601,
// 12: 0.619, 20: 0.643 -- the MUFU unit is not the limit at this pipeline depth, so the default
// keeps every exp2 on MUFU; the polynomial stays available for a deeper pipeline.
#ifndef SOL_EXP2_POLY_PAIRS
#define SOL_EXP2_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = SOL_EXP2_POLY_PAIRS;

constexpr int kMaskWords = kMaxBlocks / 32;
constexpr int kChunkWords = (kMaxBlocks / 64 + 31) / 32;

// Shared-memory and MMA geometry for head dimension D.  A row of D bf16 channels is split into
// D/64 swizzle atoms ("halves") of 64 channels = 128 bytes, each its own TMA box and buffer.
template <int D>
struct Geo {
    static_assert(D == 64 || D == 128, "head dimension 64 or 128");
    static constexpr int kHalves = D / 64;
    static constexpr uint32_t kQBytes = kHalves * kQHalfBytes;
    static constexpr uint32_t kKVTileBytes = kHalves * kKVHalfBytes;
    static constexpr uint32_t kOffQ = 0;
    static constexpr uint32_t kOffK = kOffQ + kQBytes;
    static constexpr uint32_t kOffV = kOffK + kStages * kKVTileBytes;
    static constexpr uint32_t kRingEnd = kOffV + kStages * kKVTileBytes;
    static constexpr uint32_t kOffRowA = kOffK;          // proxy rows alias the K/V ring
    static constexpr uint32_t kOffRowB = kOffK + kMaxBlocks * 4;
    static constexpr uint32_t kRowsEnd = kOffRowB + kMaxBlocks * 4;
    static constexpr uint32_t kOffMisc = ((kRingEnd > kRowsEnd ? kRingEnd : kRowsEnd) + 1023u) & ~1023u;
    static constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, 64, false);
    static constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, true);
    static constexpr int kOChunks = D / 32;              // 32-column TMEM loads of a row of O
    // S buffers of 64 columns in TMEM, then O (D columns): three buffers fit next to a 64-column O
    // (the MMA warp then issues QK two items ahead), two next to a 128-column one
    static constexpr int kSBufs = D == 64 ? 3 : 2;
    static constexpr uint32_t kTmemO = 64u * kSBufs;
    static constexpr int kLaneCh = D / 32;               // channels per lane in the proxy dot products
    static_assert(kOffMisc % 1024 == 0, "shared-memory tiles need 1024-byte alignment");
    static_assert(kTmemO + D <= kTmemCols, "S buffers and O must fit in the TMEM allocation");
    static_assert(kSBufs <= kMaxSBufs, "barrier arrays");
};

enum SelState : int { kSelRun = 0, kSelNone = 1, kSelAll = 2 };

enum WaitSite : int {
    kSiteQ = 1, kSiteProdK = 2, kSiteProdV = 3, kSiteMmaK = 4, kSiteMmaP = 5, kSiteMmaV = 6,
    kSiteSoftS = 7, kSiteSoftO = 8, kSiteEpilogue = 9, kSiteFault = 10, kSiteDrain = 11,
    kSiteProdDrain = 12, kSiteMerge = 13
};

struct Misc {
    double red[2][kNumWarps];
    double mu[2], sigma[2], tau[2];
    uint64_t q_full, k_full[kStages], v_full[kStages], v_empty[kStages];
    uint64_t s_full[kMaxSBufs], p_full[kMaxSBufs], o_final, drain, never;
    uint64_t merge_full;      // the other half's partial rows have landed (split units)
    uint32_t mask_a[kMaskWords];
    uint32_t mask_b[kMaskWords];
    uint32_t mask_u[kMaskWords];
    uint32_t need[kChunkWords];
    alignas(16) float qbar[2][kMaxHeadDim];   // read as float4 / float2
    // routing shared with the other CTA of the cluster: its q_bar of tiles A, B (written by it),
    // and its partial sums of this CTA's proxy scores over the key blocks it scored
    alignas(16) float qbar_x[2][kMaxHeadDim];
    double red_x[2][kNumWarps];
    int bh_x;                 // its head (b*H + h), or -1 for a CTA that only completes a cluster
    // radix selection of the top-k / top-p routing rules; index 0 = tile A, 1 = tile B
    double hist_mass[2][256];
    uint32_t hist_cnt[2][256];
    double sel_target[2];     // blocks (top-k) or probability mass (top-p) still to be covered
    float row_max[2];
    uint32_t sel_key[2];      // score key of the last kept block
    uint32_t sel_min[2];      // smallest kept key (the threshold statistic of the debug output)
    int sel_state[2];         // kSelRun, kSelNone or kSelAll
    int sel_ceq[2];           // blocks whose key equals sel_key
    int sel_neq[2];           // how many of those (lowest indices first) are kept
    uint32_t tmem_base;
    int abort_flag;
    int count_a, count_b;
    int split_n, split_half, split_slot, split_old;   // split units (two CTAs)
};

template <int D>
constexpr uint32_t smem_bytes() { return Geo<D>::kOffMisc + sizeof(Misc) + 1024; }   // + alignment slack
// 228 KB of shared memory per SM, of which the driver reserves 1 KB per CTA
static_assert(2 * (smem_bytes<128>() + 1024) <= 228 * 1024, "two CTAs must fit on an SM");
static_assert(offsetof(Misc, qbar) % 16 == 0, "q_bar is read with 16-byte vector loads");
static_assert(offsetof(Misc, q_full) % 8 == 0, "mbarriers need 8-byte alignment");

struct Params {
    int BH, N, Nk, Nq, npairs, nchunks;
    float beta;
    const float *beta_head;  // per-head beta [BH] (device) or null: then beta for every head
    float scale;           // (float)(1/sqrt(d)) for the proxy
    float scale_log2;      // log2(e)/sqrt(d) for the softmax
    float last_bias_log2;  // log2(n_last) for the last (possibly partial) block
    const float *kbar32;
    __nv_bfloat16 *out;
    int32_t *density;
    DeviceStatus *status;
    float *dbg_proxy;
    uint8_t *dbg_mask;
    float *dbg_stats;
    int fault_flags;
    unsigned long long timeout_ns;
    int route;               // kRouteThreshold, kRouteTopK or kRouteTopP
    int topk;                // blocks kept per query tile (top-k)
    float topp;              // probability mass to cover per query tile (top-p)
    int pair;                // 1: CTAs run in clusters of two that share the proxy scoring
    int grid_real;           // CTAs with a work unit; a last CTA past them only fills a cluster
    int split_first;         // units from this one on run as two CTAs each (the unit count: none)
    int split_slot0;         // the call's split slot of unit split_first (head groups of one call)
    int *split_cnt;          // arrival counter per split unit: launch tag << 2 | count
    int split_gen;           // this launch's tag (nonzero); another tag in a counter reads as 0
    float *split_part;       // [split unit][half][128 rows][D + 4] partial rows
};

__device__ __forceinline__ int volatile_load(const int *p) { return *reinterpret_cast<const volatile int *>(p); }

// Slow path of wait_bar, out of line so that every wait site in the pipeline loops stays small.
__device__ __noinline__ bool wait_bar_slow(uint64_t *bar, uint32_t parity, int *abort_flag,
                                           DeviceStatus *status, unsigned long long timeout_ns,
                                           int site, bool honor_abort)
{
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0) {
            if (honor_abort && volatile_load(abort_flag)) return false;
            if (globaltimer_ns() - t0 > timeout_ns) {
                *reinterpret_cast<volatile int *>(abort_flag) = 1;
                if (atomicCAS(&status->code, 0, 5) == 0) atomicExch(&status->where, site);
                return false;
            }
        }
    }
}

// Bounded wait on an mbarrier phase.  honor_abort=false is used while draining in-flight copies.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Misc &m, const Params &p,
                                         int site, bool honor_abort = true)
{
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, &m.abort_flag, p.status, p.timeout_ns, site, honor_abort);
}

// The work-item sequence every role walks identically: the correction chunks whose bit is set in
// `need`, then the key blocks whose bit is set in `mask_u`, each in ascending order.  The current
// 32-bit mask word is kept in a register and its visited bits cleared, so a step is usually one
// find-first-set (a step that re-scans shared memory cost about 450 cycles per item).
struct Walker {
    int phase = 0;      // 0: correction chunks, 1: kept blocks, 2: done
    int idx = -1;       // the current item's chunk or block index
    int wi = -1;        // index of the cached mask word
    uint32_t cur = 0;   // its bits not yet visited
    int nchunks, nblocks;   // bit counts of the two phases, held in registers
    __device__ __forceinline__ explicit Walker(const Params &p) : nchunks(p.nchunks), nblocks(p.Nk) {}
    __device__ __forceinline__ bool next(const Misc &m)
    {
        while (phase < 2) {
            const uint32_t *bits = phase == 0 ? m.need : m.mask_u;
            const int limit = phase == 0 ? nchunks : nblocks;
            const int nw = (limit + 31) >> 5;
            while (cur == 0u && wi + 1 < nw) cur = bits[++wi];
            if (cur != 0u) {
                const int r = (wi << 5) + __ffs(cur) - 1;
                cur &= cur - 1u;
                if (r < limit) {   // bits past the limit are never set; the test is a safeguard
                    idx = r;
                    return true;
                }
            }
            ++phase;
            idx = -1;
            wi = -1;
            cur = 0u;
        }
        return false;
    }
};

__device__ __forceinline__ float bf16_at(const uint8_t *p)
{
    return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t *>(p)) << 16);
}

// ----------------------------------------------------------------------------- roles

template <int D>
__device__ __forceinline__ void load_tile(uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int row, int bh)
{
    mbar_arrive_expect_tx(bar, Geo<D>::kKVTileBytes);
#pragma unroll
    for (int h = 0; h < Geo<D>::kHalves; ++h) tma_load_3d(dst + h * kKVHalfBytes, map, bar, 64 * h, row, bh);
}

// One thread feeds both rings.  The tensor core retires work in the order
// QK(it-2), PV(it-3), QK(it-1), PV(it-2), ... (the MMA issuer emits QK(j) then PV(j-1)), so the
// producer loads K(it) once QK(it-2) has freed its stage and then V(it-1) once PV(it-3) has freed
// its stage: its blocking waits follow the completion order, and a K load never queues behind a V
// stage that frees later.  K stage s is free when the QK of item it-2 has completed, which is the
// phase of s_full[s] for that item (the S buffer and the K stage share the index); that phase
// cannot be overtaken because QK(it) needs the tile loaded here.
template <int D>
__device__ __forceinline__ void producer_role(const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                              const CUtensorMap *tm_kb, const CUtensorMap *tm_vb, uint8_t *smem,
                              Misc &m, const Params &p, int bh)
{
    using G = Geo<D>;
    int issued_k[kStages], issued_v[kStages];
    for (int s = 0; s < kStages; ++s) issued_k[s] = issued_v[s] = -1;
    Walker wk(p), wv(p);
    bool more_k = wk.next(m), more_v = wv.next(m);
    bool ok = true;
    for (int it = 0; ok && (more_k || more_v); ++it) {
        if (more_k) {
            const int s = it & 1;
            constexpr int B = Geo<D>::kSBufs;
            if (it >= 2 && !wait_bar(&m.s_full[(it - 2) % B], ((it - 2) / B) & 1, m, p, kSiteProdK)) { ok = false; break; }
            load_tile<D>(smem + G::kOffK + s * G::kKVTileBytes, wk.phase == 0 ? tm_kb : tm_k, &m.k_full[s], wk.idx * kTile, bh);
            issued_k[s] = it;
            more_k = wk.next(m);
        }
        const int iv = it - 1;
        if (iv >= 0 && more_v) {
            const int s = iv & 1;
            if (iv >= 2 && !wait_bar(&m.v_empty[s], ((iv - 2) >> 1) & 1, m, p, kSiteProdV)) { ok = false; break; }
            load_tile<D>(smem + G::kOffV + s * G::kKVTileBytes, wv.phase == 0 ? tm_vb : tm_v, &m.v_full[s], wv.idx * kTile, bh);
            issued_v[s] = iv;
            more_v = wv.next(m);
        }
    }
    // No TMA write may still be in flight when the CTA exits.
    for (int s = 0; s < kStages; ++s) {
        if (issued_k[s] >= 0) wait_bar(&m.k_full[s], (issued_k[s] >> 1) & 1, m, p, kSiteProdDrain, false);
        if (issued_v[s] >= 0) wait_bar(&m.v_full[s], (issued_v[s] >> 1) & 1, m, p, kSiteProdDrain, false);
    }
}

template <int D>
__device__ __forceinline__ bool issue_pv(int t, uint32_t tmem, uint64_t dv0, Misc &m, const Params &p)
{
    using G = Geo<D>;
    const int b = t % G::kSBufs, s = t & 1;
    if (!wait_bar(&m.p_full[b], (t / G::kSBufs) & 1, m, p, kSiteMmaP)) return false;
    if (!wait_bar(&m.v_full[s], (t >> 1) & 1, m, p, kSiteMmaV)) return false;
    tc_fence_after();
    // B = V tile of stage s, MN-major: 64 channels contiguous per key row (128 B, swizzled), next
    // 8 keys at +1024 B (SBO), channels 64..127 (d = 128) at +8192 B (LBO); 16 keys per MMA ->
    // +2048 B, i.e. +128 in the descriptor's 16-byte address units.
    const uint64_t dv = dv0 + static_cast<uint64_t>(s) * (G::kKVTileBytes >> 4);
    const uint32_t a0 = tmem + tmem_s_col(b);
    const uint32_t o = tmem + G::kTmemO;
    if (t > 0) mma_ts_acc(o, a0, dv, G::kIdescPV);
    else mma_ts(o, a0, dv, G::kIdescPV, 0u);
    mma_ts_acc(o, a0 + 8, dv + 128, G::kIdescPV);
    mma_ts_acc(o, a0 + 16, dv + 256, G::kIdescPV);
    mma_ts_acc(o, a0 + 24, dv + 384, G::kIdescPV);
    mma_commit(&m.v_empty[s]);
    return true;
}

template <int D>
__device__ __forceinline__ void mma_role(uint32_t tmem, uint8_t *smem, Misc &m, const Params &p)
{
    using G = Geo<D>;
    bool ok = true;
    if (p.fault_flags & 1) ok = wait_bar(&m.never, 0, m, p, kSiteFault);
    if (ok) ok = wait_bar(&m.q_full, 0, m, p, kSiteQ);
    if (ok) {
        tc_fence_after();
        // Descriptors are built once; a k-step or stage only adds a compile-time offset to the
        // 14-bit start-address field (16-byte units; every address stays below 256 KB).
        // A = Q (128 x d), B = K tile (64 x d), both K-major 128B-swizzled with 8-row groups
        // 1024 B apart; channels 64..127 (d = 128) live in the second half buffer and a
        // 16-channel step advances the start address by 32 B inside the swizzle atom.
        const uint64_t dq = desc_sw128(smem_u32(smem + G::kOffQ), 16, 1024);
        const uint64_t dk0 = desc_sw128(smem_u32(smem + G::kOffK), 16, 1024);
        const uint64_t dv0 = desc_sw128(smem_u32(smem + G::kOffV), kKVHalfBytes, 1024);
        constexpr uint64_t kQh = kQHalfBytes >> 4, kKh = kKVHalfBytes >> 4;
        // QK(it) is issued before PV(it - L), L = kSBufs - 1: S buffer it % kSBufs held P(it - kSBufs),
        // whose PV was issued in an earlier iteration.
        constexpr int L = G::kSBufs - 1;
        Walker w(p);
        int it = 0;
        while (ok && w.next(m)) {
            const int s = it & 1, b = it % G::kSBufs;
            if (!wait_bar(&m.k_full[s], (it >> 1) & 1, m, p, kSiteMmaK)) { ok = false; break; }
            tc_fence_after();
            const uint64_t dk = dk0 + static_cast<uint64_t>(s) * (G::kKVTileBytes >> 4);
            const uint32_t d = tmem + tmem_s_col(b);
            mma_ss(d, dq, dk, G::kIdescQK, 0u);
            mma_ss_acc(d, dq + 2, dk + 2, G::kIdescQK);
            mma_ss_acc(d, dq + 4, dk + 4, G::kIdescQK);
            mma_ss_acc(d, dq + 6, dk + 6, G::kIdescQK);
            if constexpr (G::kHalves == 2) {
                mma_ss_acc(d, dq + kQh, dk + kKh, G::kIdescQK);
                mma_ss_acc(d, dq + kQh + 2, dk + kKh + 2, G::kIdescQK);
                mma_ss_acc(d, dq + kQh + 4, dk + kKh + 4, G::kIdescQK);
                mma_ss_acc(d, dq + kQh + 6, dk + kKh + 6, G::kIdescQK);
            }
            mma_commit(&m.s_full[b]);
            if (it >= L && !issue_pv<D>(it - L, tmem, dv0, m, p)) { ok = false; break; }
            ++it;
        }
        for (int t = it - L < 0 ? 0 : it - L; ok && t < it; ++t) ok = issue_pv<D>(t, tmem, dv0, m, p);
        if (ok && it > 0) mma_commit(&m.o_final);
    }
    // Every MMA issued so far must finish before TMEM is freed.
    mma_commit(&m.drain);
    wait_bar(&m.drain, 0, m, p, kSiteDrain, false);
}

// Kinds of softmax work item: a correction chunk of 64 pooled blocks, a full kept key block, and
// the last key block when it is partial.  They run in separate loops (correction chunks first,
// the partial block last), so the loop over full kept blocks, where the time goes, carries neither
// the correction nor the tail-masking code (the smaller loop measured about 10 % faster per item).
enum ItemKind : int { kItemCorr = 0, kItemFull = 1, kItemPartial = 2 };

// One softmax work item for the thread that owns TMEM lane `row`: wait for S, mask, update the
// running max (rescaling O in TMEM when it grows by more than 2^8), exponentiate, publish P.
// Returns false if a wait gave up.
template <int D, int kKind>
__device__ __forceinline__ bool softmax_item(uint32_t tmem, Misc &m, const Params &p,
                                             const uint32_t *mymask, uint32_t lane_base, int it,
                                             int idx, float &m_used, float &l)
{
    const int b = it % Geo<D>::kSBufs;
    bool ok = wait_bar(&m.s_full[b], (it / Geo<D>::kSBufs) & 1, m, p, kSiteSoftS);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (!ok) return false;
    tc_fence_after();
    const uint32_t s_addr = tmem + lane_base + tmem_s_col(b);
    uint32_t pk[32];
    bool rescale = false;
    float factor = 1.0f;
    const bool participate =
        kKind == kItemCorr || ((mymask[idx >> 5] >> (idx & 31)) & 1u);   // warp-uniform
    if (participate) {
        uint32_t r[64];
        tmem_ld64(s_addr, r);
        tmem_wait_ld();
        float mx;          // row max of the log2-domain logits of this item
        uint64_t mul2;     // exp2 argument = r * mul2 - m_ref, two columns at a time
        if constexpr (kKind == kItemCorr) {
            // Correction chunk: column i is pooled block j0 + i with logit
            // S*log2(e)/sqrt(d) + log2(n_j), or -inf if this row's tile kept block j (it is
            // computed exactly) or j is past the last block.
            const int c = idx;
            const int j0 = c * 64;
            uint64_t use = ~(static_cast<uint64_t>(mymask[2 * c]) |
                             (static_cast<uint64_t>(mymask[2 * c + 1]) << 32));
            const int nvalid = p.Nk - j0;
            if (nvalid < 64) use &= (1ull << nvalid) - 1ull;
            const int last = p.Nk - 1 - j0;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float bias = (i == last) ? p.last_bias_log2 : 6.0f;
                const float x = fmaf(__uint_as_float(r[i]), p.scale_log2, bias);
                r[i] = ((use >> i) & 1ull) ? __float_as_uint(x) : __float_as_uint(-INFINITY);
            }
            mul2 = f2(1.0f, 1.0f);
        } else {
            // Kept block: exact logits; columns past the sequence end (only in the last, partial
            // block) are -inf.
            if constexpr (kKind == kItemPartial) {
                const int nvalid = p.N - idx * kTile;
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if (i >= nvalid) r[i] = __float_as_uint(-INFINITY);
            }
            mul2 = f2(p.scale_log2, p.scale_log2);
        }
        uint64_t sum2;
        // Exponentials against mref: P into pk, the row sum into sum2; with kTrack the pass also
        // forms the item's row max (of r) in mx.
        auto exp_pass = [&](float mref, auto track) {
            constexpr bool kTrack = decltype(track)::value;
            const uint64_t add2 = f2(-mref, -mref);
            sum2 = f2(0.0f, 0.0f);
            if constexpr (kTrack) mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float r0 = __uint_as_float(r[2 * i]), r1 = __uint_as_float(r[2 * i + 1]);
                if constexpr (kTrack) mx = max3f(mx, r0, r1);
                const uint64_t a2 = ffma2(f2(r0, r1), mul2, add2);
                float e0, e1;
                if (i < kPolyPairs) {
                    exp2_poly2(a2, e0, e1);
                } else {
                    float a0, a1;
                    unf2(a2, a0, a1);
                    e0 = ex2_approx(a0);
                    e1 = ex2_approx(a1);
                }
                sum2 = fadd2(sum2, f2(e0, e1));
                pk[i] = pack_bf16x2(e0, e1);
            }
        };
        if constexpr (Geo<D>::kSBufs >= 3) {
            // With three S buffers the MMA warp runs two items ahead and the softmax is the
            // critical path: the exponentials are taken against the running max m_used (which
            // only moves when the item's max exceeds it by more than 2^8) while the item's max
            // is formed in the same pass, so they do not wait for it.  When it moves (always on
            // a row's first item, where m_used is -inf) the row repeats the pass against the new
            // max; S stays in registers meanwhile.  The decisions and arguments are those of the
            // max-first order below, so the results are identical.
            float mref = m_used == -INFINITY ? 0.0f : m_used;
            for (;;) {
                exp_pass(mref, std::true_type{});
                if constexpr (kKind != kItemCorr) mx *= p.scale_log2;
                if (!(mx > m_used + kRescaleLog2)) break;
                factor = ex2_approx(m_used - mx);
                rescale = m_used != -INFINITY;
                m_used = mx;
                mref = mx;
            }
        } else {
            // Max first.  With two S buffers the item chain through the MMA warp is the critical
            // path, and the single-pass order above measured slower here.
            mx = max3f(__uint_as_float(r[0]), __uint_as_float(r[1]), __uint_as_float(r[2]));
#pragma unroll
            for (int i = 3; i < 63; i += 2) mx = max3f(mx, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
            mx = fmaxf(mx, __uint_as_float(r[63]));
            if constexpr (kKind != kItemCorr) mx *= p.scale_log2;
            const float m_new = fmaxf(m_used, mx);
            if (m_new > m_used + kRescaleLog2) {
                factor = ex2_approx(m_used - m_new);
                rescale = m_used != -INFINITY;
                m_used = m_new;
            }
            exp_pass(m_used == -INFINITY ? 0.0f : m_used, std::false_type{});
        }
        float s0, s1;
        unf2(sum2, s0, s1);
        l = l * factor + (s0 + s1);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
    }
    if (__any_sync(0xFFFFFFFFu, rescale) && it > 0) {
        // PV(it-1) must be done before O is touched; its completion is the phase
        // (it-1)>>1 of v_empty[(it-1)&1].  Here PV(it-3) has completed (s_full for item it
        // was committed after PV(it-kSBufs), it-3 at the latest, was issued) and PV(it+1)
        // waits for this thread's p_full arrival, so that barrier is either one phase short
        // or complete: the parity is unambiguous.
        ok = wait_bar(&m.v_empty[(it - 1) & 1], ((it - 1) >> 1) & 1, m, p, kSiteSoftO);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (!ok) return false;
        tc_fence_after();
        const float f = rescale ? factor : 1.0f;
#pragma unroll 1
        for (int ch = 0; ch < Geo<D>::kOChunks; ++ch) {
            uint32_t o[32];
            const uint32_t oaddr = tmem + lane_base + Geo<D>::kTmemO + ch * 32;
            tmem_ld32(oaddr, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(oaddr, o);
        }
    }
    tmem_st32(s_addr, pk);
    tmem_wait_st();
    tc_fence_before();
    // one arrival per warp, after every lane's P stores have completed
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&m.p_full[b]);
    return true;
}

// Arrival of one half of a split unit on its counter, which holds (launch tag << 2) | count.  A
// counter whose tag is not this launch's counts as 0: a launch that gave up part way (a wait ran
// out) may leave its counters at 1 or 2, and a later launch on the same workspace must not read
// them as arrivals.  Returns the count before this arrival.
__device__ __forceinline__ int split_arrive(int *cnt, int gen)
{
    int old = *reinterpret_cast<volatile int *>(cnt);
    for (;;) {
        const int c = (old >> 2) == gen ? (old & 3) : 0;
        const int prev = atomicCAS(cnt, old, (gen << 2) | (c + 1));
        if (prev == old) return c;
        old = prev;
    }
}

// Epilogue of a unit split over two CTAs; softmax threads, one per row (TMEM lane).  Each half
// counts its arrival on the unit's counter.  The first to arrive writes its rows' unnormalised
// output O (relative to 2^m), running max m (log2 domain) and sum l to its partial slot and counts
// again; the second waits until the counter reads 3 (a bounded wait on a CTA that has already
// arrived, so is running, and has nothing left to wait for), brings those rows into shared memory
// and merges:
//   out = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)),
//   M = max(m_0, m_1),
// the online-softmax combination of two disjoint sets of terms.  A half without items (has_o
// false) contributes m = -inf, l = 0 and O = 0.  If any softmax warp's waits failed (ok false),
// the CTA does not arrive (the other half then arrives first and publishes) and the status words
// hold the timeout.
template <int D>
__device__ __forceinline__ void split_epilogue(uint32_t tmem, Misc &m, const Params &p, int bh, int row0,
                                            uint32_t lane_base, bool ok, bool has_o, float m_used, float l)
{
    uint32_t all_ok;
    asm volatile("{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\t"
                 "bar.red.and.pred b, 1, %2, a;\n\tselp.u32 %0, 1, 0, b;\n\t}"
                 : "=r"(all_ok)
                 : "r"(static_cast<uint32_t>(ok)), "r"(kSoftmaxThreads)
                 : "memory");
    if (!all_ok) return;
    constexpr int kRow = D + 4;   // floats per partial row: O[D], m, l, 2 unused (16-byte rows)
    const int row = threadIdx.x;
    const int slot = m.split_slot, half = m.split_half;
    int *cnt = p.split_cnt + slot;
    // Arrival first: the first half to arrive publishes its rows and counts again (the counter
    // reaches 3 once both halves have arrived and the rows are out); the second merges and never
    // writes its own partial rows.
    if (row == 0) m.split_old = split_arrive(cnt, p.split_gen);
    asm volatile("bar.sync 1, %0;" ::"r"(kSoftmaxThreads) : "memory");
    if (m.split_old == 0) {
        float *mine = p.split_part + (static_cast<size_t>(2 * slot + half) * kBM + row) * kRow;
#pragma unroll 1
        for (int ch = 0; ch < Geo<D>::kOChunks; ++ch) {
            uint32_t o[32];
            if (has_o) {
                tmem_ld32(tmem + lane_base + Geo<D>::kTmemO + ch * 32, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
            float4 *dst = reinterpret_cast<float4 *>(mine + ch * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                     __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
        }
        mine[D] = m_used;
        mine[D + 1] = l;
        __threadfence();                                           // the rows are visible ...
        asm volatile("bar.sync 1, %0;" ::"r"(kSoftmaxThreads) : "memory");
        // ... before this count (debug fault flag 4 withholds it, so the other half's wait runs
        // out); the counter already carries this launch's tag
        if (row == 0 && !(p.fault_flags & 4)) atomicAdd(cnt, 1);
        return;
    }
    // Second: wait (bounded) until the first half's rows are out.  The first half has already
    // arrived, so it is running and its publication ends.
    if (row == 0) {
        const uint64_t t0 = globaltimer_ns();
        const int done = (p.split_gen << 2) | 3;
        int seen;
        for (;;) {
            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(seen) : "l"(cnt) : "memory");
            if (seen == done) break;
            if (globaltimer_ns() - t0 > p.timeout_ns) {
                if (atomicCAS(&p.status->code, 0, 5) == 0) atomicExch(&p.status->where, kSiteMerge);
                break;
            }
            __nanosleep(256);
        }
        m.split_old = seen == done ? 1 : -1;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kSoftmaxThreads) : "memory");
    if (m.split_old < 0) return;
    __threadfence();
    // The other half's 128 rows are one contiguous block: one bulk copy brings them into shared
    // memory (the Q tile and the K/V ring are idle: every MMA of this CTA has completed).
    constexpr uint32_t kRowsBytes = kBM * kRow * 4;
    static_assert(kRowsBytes <= Geo<D>::kOffMisc && kRowsBytes % 16 == 0, "partial rows fit the idle tiles");
    float *rows = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(&m) - Geo<D>::kOffMisc);
    if (row == 0) {
        fence_proxy_async_global();
        mbar_arrive_expect_tx(&m.merge_full, kRowsBytes);
        bulk_load(rows, p.split_part + static_cast<size_t>(2 * slot + (half ^ 1)) * kBM * kRow, kRowsBytes,
                  &m.merge_full);
    }
    if (!wait_bar(&m.merge_full, 0, m, p, kSiteMerge, false)) return;
    const float *theirs = rows + row * kRow;
    const float mo = theirs[D], lo = theirs[D + 1];
    const float M = fmaxf(m_used, mo);
    const float wa = m_used == -INFINITY ? 0.0f : ex2_approx(m_used - M);
    const float wb = mo == -INFINITY ? 0.0f : ex2_approx(mo - M);
    // half 0's term first whichever half merges, so the rounding (one fused multiply-add) and
    // hence the output do not depend on which CTA finished second
    auto sum2 = [&](float own_x, float own_w, float their_x, float their_w) {
        return half == 0 ? fmaf(own_x, own_w, their_x * their_w) : fmaf(their_x, their_w, own_x * own_w);
    };
    const float inv = 1.0f / sum2(l, wa, lo, wb);
    const int grow = row0 + row;
    const bool store = grow < p.N;
    uint4 *dst = reinterpret_cast<uint4 *>(p.out + (static_cast<size_t>(bh) * p.N + (store ? grow : 0)) * D);
#pragma unroll 1
    for (int ch = 0; ch < Geo<D>::kOChunks; ++ch) {
        uint32_t o[32];
        if (has_o) {
            tmem_ld32(tmem + lane_base + Geo<D>::kTmemO + ch * 32, o);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        const float4 *src = reinterpret_cast<const float4 *>(theirs + ch * 32);
        auto mix = [&](int i, float t) { return sum2(__uint_as_float(o[i]), wa, t, wb) * inv; };
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const float4 t0 = src[2 * q4], t1 = src[2 * q4 + 1];
            uint4 w;
            w.x = pack_bf16x2(mix(8 * q4 + 0, t0.x), mix(8 * q4 + 1, t0.y));
            w.y = pack_bf16x2(mix(8 * q4 + 2, t0.z), mix(8 * q4 + 3, t0.w));
            w.z = pack_bf16x2(mix(8 * q4 + 4, t1.x), mix(8 * q4 + 5, t1.y));
            w.w = pack_bf16x2(mix(8 * q4 + 6, t1.z), mix(8 * q4 + 7, t1.w));
            if (store) dst[ch * 4 + q4] = w;
        }
    }
    if (row == 0) p.split_cnt[slot] = 0;   // ready for the next call
}

// Softmax warps 0-3: thread r owns row r of the 128-row tile (TMEM lane r).
template <int D>
__device__ __forceinline__ void softmax_role(uint32_t tmem, Misc &m, const Params &p, int bh, int row0)
{
    const int row = threadIdx.x;                       // 0..127 == TMEM lane
    const int warp = row >> 5;
    const bool in_b = row >= 64;
    const uint32_t *mymask = in_b ? m.mask_b : m.mask_a;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_used = -INFINITY, l = 0.0f;
    Walker w(p);
    int it = 0;
    bool ok = true;
    bool more = w.next(m);
    for (; ok && more && w.phase == 0; more = w.next(m)) {
        ok = softmax_item<D, kItemCorr>(tmem, m, p, mymask, lane_base, it, w.idx, m_used, l);
        it += ok;
    }
    const int partial = p.N % kTile ? p.Nk - 1 : -1;   // the last block when it is partial
    for (; ok && more && w.idx != partial; more = w.next(m)) {
        ok = softmax_item<D, kItemFull>(tmem, m, p, mymask, lane_base, it, w.idx, m_used, l);
        it += ok;
    }
    if (ok && more) {   // the partial last block is the last item when it is kept
        ok = softmax_item<D, kItemPartial>(tmem, m, p, mymask, lane_base, it, w.idx, m_used, l);
        it += ok;
    }
    // o_final is single-use: at this point two PVs may still be outstanding (the QK of the last
    // item is issued before the PV of the one before it), so no per-stage parity identifies the
    // last PV.
    if (m.split_n > 1) {
        // Every softmax warp enters the split epilogue, whose barriers count all four, even after
        // a failed wait (every wait is bounded, so every warp gets here).  Half of a unit may
        // have no item.
        if (ok && it > 0) {
            ok = wait_bar(&m.o_final, 0, m, p, kSiteEpilogue);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (ok) tc_fence_after();
        }
        split_epilogue<D>(tmem, m, p, bh, row0, lane_base, ok, it > 0, m_used, l);
        return;
    }
    if (!ok || it == 0) return;   // (a whole unit always has an item)
    ok = wait_bar(&m.o_final, 0, m, p, kSiteEpilogue);
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (!ok) return;
    tc_fence_after();
    const int grow = row0 + row;
    const bool store = grow < p.N;
    const float inv_l = 1.0f / l;
    uint4 *dst = reinterpret_cast<uint4 *>(p.out + (static_cast<size_t>(bh) * p.N + (store ? grow : 0)) * D);
#pragma unroll 1
    for (int ch = 0; ch < Geo<D>::kOChunks; ++ch) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + Geo<D>::kTmemO + ch * 32, o);
        tmem_wait_ld();
        if (store) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(o[8 * q4 + 0]) * inv_l, __uint_as_float(o[8 * q4 + 1]) * inv_l);
                v.y = pack_bf16x2(__uint_as_float(o[8 * q4 + 2]) * inv_l, __uint_as_float(o[8 * q4 + 3]) * inv_l);
                v.z = pack_bf16x2(__uint_as_float(o[8 * q4 + 4]) * inv_l, __uint_as_float(o[8 * q4 + 5]) * inv_l);
                v.w = pack_bf16x2(__uint_as_float(o[8 * q4 + 6]) * inv_l, __uint_as_float(o[8 * q4 + 7]) * inv_l);
                dst[ch * 4 + q4] = v;
            }
        }
    }
}

// ----------------------------------------------------------------------------- kernel

// Vector of LC consecutive floats loaded with one 8- or 16-byte access.
// ----------------------------------------------------------------------------- top-k / top-p

// Order-preserving 32-bit key of a score: a larger float gives a larger key; -0.0 and +0.0 (equal
// scores) share the key of +0.0.
__device__ __forceinline__ uint32_t score_key(float x)
{
    const uint32_t u = __float_as_uint(x == 0.0f ? 0.0f : x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_score(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Radix selection (four 8-bit digits, most significant first) of the last kept block of the
// top-k or top-p rule, for both routing tiles at once; all threads of the CTA take part.
// Blocks are ranked by score, highest first, equal scores by ascending index.  Top-k keeps the
// first k; top-p keeps the shortest prefix whose softmax mass (float64, w_j = exp(S_j - max S))
// reaches p * Z.  Each pass histograms the digit of the blocks whose higher digits equal the
// selected prefix (counts, and for top-p masses) and one warp per tile walks the histogram from
// the top bin down to the bin that holds the last kept block.  Result per tile t: sel_key[t] and
// sel_neq[t] -- keep key > sel_key, and the first sel_neq[t] (by index) of the sel_ceq[t] blocks
// whose key equals sel_key -- or sel_state[t] = kSelNone / kSelAll.
__device__ void radix_select(const float *row_a, const float *row_b, bool has_b, int Nk, Misc &m,
                             const Params &p)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool topp = p.route == kRouteTopP;
    if (topp) {   // row maxima for the softmax masses
        float ma = -INFINITY, mb = -INFINITY;
        for (int j = tid; j < Nk; j += kThreads) {
            ma = fmaxf(ma, row_a[j]);
            mb = fmaxf(mb, row_b[j]);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            ma = fmaxf(ma, __shfl_xor_sync(0xFFFFFFFFu, ma, o));
            mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
        }
        if (lane == 0) {
            m.red[0][warp] = ma;
            m.red[1][warp] = mb;
        }
    }
    __syncthreads();
    if (tid < 2) {
        const int t = tid;
        if (topp) {
            float mx = -INFINITY;
            for (int w = 0; w < kNumWarps; ++w) mx = fmaxf(mx, static_cast<float>(m.red[t][w]));
            m.row_max[t] = mx;
        }
        int state = kSelRun;
        double target = 0.0;
        if (t == 1 && !has_b) {
            state = kSelNone;
        } else if (topp) {
            if (p.topp >= 1.0f) state = kSelAll;
            else if (!(p.topp > 0.0f)) state = kSelNone;   // target p*Z is set in the first pass
        } else {
            const int need = min(p.topk, Nk);
            if (need <= 0) state = kSelNone;
            else if (need >= Nk) state = kSelAll;
            target = need;
        }
        m.sel_state[t] = state;
        m.sel_target[t] = target;
        m.sel_key[t] = 0u;
        m.sel_min[t] = 0xFFFFFFFFu;
        m.sel_ceq[t] = 0;
        m.sel_neq[t] = 0;
    }
    __syncthreads();
    if (m.sel_state[0] != kSelRun && m.sel_state[1] != kSelRun) return;

    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
        for (int i = tid; i < 256; i += kThreads) {
            m.hist_cnt[0][i] = 0u;
            m.hist_cnt[1][i] = 0u;
            m.hist_mass[0][i] = 0.0;
            m.hist_mass[1][i] = 0.0;
        }
        __syncthreads();
        for (int t = 0; t < 2; ++t) {
            if (m.sel_state[t] != kSelRun) continue;
            const float *row = t ? row_b : row_a;
            const uint32_t pre = m.sel_key[t];
            const double mx = m.row_max[t];
            for (int j = tid; j < Nk; j += kThreads) {
                const float sc = row[j];
                const uint32_t key = score_key(sc);
                if ((key ^ pre) & hi_mask) continue;
                const int dig = (key >> shift) & 255;
                atomicAdd(&m.hist_cnt[t][dig], 1u);
                if (topp) atomicAdd(&m.hist_mass[t][dig], exp(static_cast<double>(sc) - mx));
            }
        }
        __syncthreads();
        if (warp < 2 && m.sel_state[warp] == kSelRun) {
            const int t = warp;
            // lane l holds bins 8l..8l+7; higher bins hold higher scores
            double v[8];
            uint32_t c[8];
            double tot = 0.0;
            uint32_t ctot = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = m.hist_cnt[t][8 * lane + i];
                v[i] = topp ? m.hist_mass[t][8 * lane + i] : static_cast<double>(c[i]);
                tot += v[i];
                ctot += c[i];
            }
            double incl = tot;   // sum over lanes l..31
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const double n = __shfl_down_sync(0xFFFFFFFFu, incl, o);
                if (lane + o < 32) incl += n;
            }
            double target = m.sel_target[t];
            if (topp && pass == 0) target = static_cast<double>(p.topp) * __shfl_sync(0xFFFFFFFFu, incl, 0);
            // the bin of the last kept block is in the highest lane whose suffix sum reaches the
            // target; if rounding leaves every lane short, the lowest non-empty lane is used
            const uint32_t reach = __ballot_sync(0xFFFFFFFFu, incl >= target);
            const uint32_t nonempty = __ballot_sync(0xFFFFFFFFu, ctot != 0u);
            const int sel_lane = reach ? 31 - __clz(reach) : __ffs(nonempty) - 1;
            if (lane == sel_lane) {
                double acc = incl - tot;          // mass/count of the higher lanes
                // first bin (from the top) whose running sum reaches the target; if rounding
                // leaves every bin just short, the lowest non-empty bin
                int bin = -1, low = -1;
                uint32_t cnt = 0u, low_cnt = 0u;
                double before = acc, low_before = acc;
#pragma unroll
                for (int i = 7; i >= 0; --i) {
                    if (bin >= 0 || c[i] == 0u) continue;
                    if (acc + v[i] >= target) {
                        bin = i;
                        cnt = c[i];
                        before = acc;
                    } else {
                        low = i;
                        low_cnt = c[i];
                        low_before = acc;
                        acc += v[i];
                    }
                }
                if (bin < 0) {
                    bin = low;
                    cnt = low_cnt;
                    before = low_before;
                }
                m.sel_key[t] |= static_cast<uint32_t>(8 * lane + bin) << shift;
                m.sel_target[t] = target - before;
                m.sel_ceq[t] = static_cast<int>(cnt);
            }
        }
        __syncthreads();
    }
    if (tid < 2 && m.sel_state[tid] == kSelRun) {
        const int t = tid;
        const int ceq = m.sel_ceq[t];
        const double rem = m.sel_target[t];
        int n;
        if (topp) {
            // blocks with the selected key have equal masses; add them in index order until the
            // remaining mass is covered
            const double w = exp(static_cast<double>(key_score(m.sel_key[t])) - static_cast<double>(m.row_max[t]));
            double acc = 0.0;
            n = 0;
            while (n < ceq && acc < rem) {
                acc += w;
                ++n;
            }
            n = max(n, 1);
        } else {
            n = static_cast<int>(rem);
        }
        m.sel_neq[t] = min(max(n, 1), ceq);
    }
    __syncthreads();
}

// Keep decision of the top-k / top-p rules before ties at the selected key are thinned out.
__device__ __forceinline__ bool sel_keep(const Misc &m, int t, uint32_t key)
{
    const int st = m.sel_state[t];
    return st == kSelAll || (st == kSelRun && key >= m.sel_key[t]);
}

// Blocks whose key equals the selected key are all marked kept by sel_keep; keep only the first
// sel_neq of them (by index).  One thread per tile; runs only when such ties exist.
__device__ void thin_ties(uint32_t *mask, const float *row, int Nk, Misc &m, int t, int *count)
{
    if (m.sel_state[t] != kSelRun || m.sel_neq[t] >= m.sel_ceq[t]) return;
    const uint32_t ks = m.sel_key[t];
    int seen = 0;
    for (int j = 0; j < Nk; ++j) {
        if (score_key(row[j]) != ks) continue;
        if (seen >= m.sel_neq[t]) {
            mask[j >> 5] &= ~(1u << (j & 31));
            --*count;
        }
        ++seen;
    }
}

template <int LC>
__device__ __forceinline__ void load_vec(const float *src, float (&x)[LC])
{
    if constexpr (LC == 4) {
        const float4 t = __ldg(reinterpret_cast<const float4 *>(src));
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
    } else {
        static_assert(LC == 2, "2 or 4 channels per lane");
        const float2 t = __ldg(reinterpret_cast<const float2 *>(src));
        x[0] = t.x; x[1] = t.y;
    }
}

// One warp.  The walk visits the set bits of `need` (correction chunks) and then of `mask_u` (kept
// blocks), each in ascending order; this keeps the items at even (half 0) or odd (half 1)
// positions of the walk and clears the others, so every role of this CTA walks its half with the
// ordinary walker.
__device__ __forceinline__ void keep_half_of_walk(Misc &m, const Params &p, int half)
{
    const int lane = threadIdx.x & 31;
    int parity = 0;   // walk position of the first set bit of the current group of words, mod 2
    for (int phase = 0; phase < 2; ++phase) {
        uint32_t *bits = phase == 0 ? m.need : m.mask_u;
        const int nw = ((phase == 0 ? p.nchunks : p.Nk) + 31) >> 5;
        for (int w0 = 0; w0 < nw; w0 += 32) {
            const int w = w0 + lane;
            const uint32_t x = w < nw ? bits[w] : 0u;
            const int c = __popc(x);
            int incl = c;   // inclusive prefix over the lanes of the set-bit counts
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            int pos = parity + incl - c;
            uint32_t keep = 0u, rest = x;
            while (rest) {
                const uint32_t b = rest & (0u - rest);
                if ((pos & 1) == half) keep |= b;
                rest ^= b;
                ++pos;
            }
            if (w < nw) bits[w] = keep;
            parity = (parity + __shfl_sync(0xFFFFFFFFu, incl, 31)) & 1;
        }
    }
}

// kRank: the top-k / top-p rules (radix selection) are compiled in; the threshold rule's kernel is
// a separate instantiation without that code, which otherwise costs it about 3 % (measured).
template <int D, bool kRank>
__global__ void __launch_bounds__(kThreads, 2)
sol_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kb,
               const __grid_constant__ CUtensorMap tm_vb, const Params p)
{
    using G = Geo<D>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned by pointer arithmetic on the shared array, so that the compiler keeps
    // everything derived from it in the shared address space (an integer round trip would make
    // every Misc, mask and proxy-row access a generic one)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Misc &m = *reinterpret_cast<Misc *>(smem + G::kOffMisc);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // With p.pair, CTAs run in clusters of two (block indices 2c, 2c+1) that share the routing's
    // reads of the pooled keys.  A last CTA past grid_real exists only to complete a cluster: it
    // takes part in the shared routing (scoring its partner's tiles) and leaves.
    const bool paired = p.pair != 0;
    const bool real = static_cast<int>(blockIdx.x) < p.grid_real;
    const uint32_t partner = paired ? cluster_rank() ^ 1u : 0u;
    // Work unit: a pair of query tiles of one head.  The units from split_first on run as two
    // CTAs each (halves 0 and 1 on adjacent block indices), every other item of the unit's walk
    // on each; the second to finish merges the two partial results.
    int unit = real ? static_cast<int>(blockIdx.x) : 0, split_n = 1, split_half = 0;
    if (unit >= p.split_first) {
        const int r = unit - p.split_first;
        unit = p.split_first + (r >> 1);
        split_half = r & 1;
        split_n = 2;
    }
    const int pair = unit % p.npairs;
    const int bh = unit / p.npairs;
    const int tile_a = 2 * pair, tile_b = 2 * pair + 1;
    const bool has_b = tile_b < p.Nq;
    const int row0 = tile_a * kTile;
    const int n_a = min(kTile, p.N - row0);
    const int n_b = has_b ? min(kTile, p.N - row0 - kTile) : 0;
    const int Nk = p.Nk;

    if (tid == 0) {
        mbar_init(&m.q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&m.k_full[s], 1);
            mbar_init(&m.v_full[s], 1);
            mbar_init(&m.v_empty[s], 1);
        }
        for (int b = 0; b < kMaxSBufs; ++b) {
            mbar_init(&m.s_full[b], 1);
            mbar_init(&m.p_full[b], kSoftmaxThreads / 32);
        }
        mbar_init(&m.o_final, 1);
        mbar_init(&m.merge_full, 1);
        mbar_init(&m.drain, 1);
        mbar_init(&m.never, 1);
        m.abort_flag = 0;
        m.count_a = 0;
        m.count_b = 0;
        m.split_n = split_n;
        m.split_half = split_half;
        m.split_slot = unit - p.split_first + p.split_slot0;
        fence_mbar_init();
    }
    for (int i = tid; i < kMaskWords; i += kThreads) {
        m.mask_a[i] = 0u;
        m.mask_b[i] = 0u;
        m.mask_u[i] = 0u;
    }
    if (tid < kChunkWords) m.need[tid] = 0u;
    if (warp == kWarpTma && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_kb);
        tma_prefetch_desc(&tm_vb);
    }
    if (warp == kWarpMma && real) {
        tmem_alloc(&m.tmem_base, kTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m.tmem_base;

    if (warp == kWarpTma && lane == 0 && real) {
        mbar_arrive_expect_tx(&m.q_full, G::kQBytes);
#pragma unroll
        for (int h = 0; h < G::kHalves; ++h)
            tma_load_3d(smem + G::kOffQ + h * kQHalfBytes, &tm_q, &m.q_full, 64 * h, row0, bh);
    }

    // ---------------- routing 1: q_bar of both routing tiles (float32, ascending rows), also
    // written into the partner CTA's qbar_x
    if (tid < D) {
        if (!real) {
            m.qbar[0][tid] = 0.0f;
            m.qbar[1][tid] = 0.0f;
        } else if (wait_bar(&m.q_full, 0, m, p, kSiteQ)) {
            const int c = tid, half = c >> 6, cc = c & 63, chunk = cc >> 3, within = cc & 7;
            const uint8_t *qh = smem + G::kOffQ + half * kQHalfBytes + within * 2;
            float sa = 0.0f, sb = 0.0f;
            // unrolled so that the shared-memory loads run ahead of the (ordered) additions
#pragma unroll 8
            for (int r = 0; r < n_a; ++r) sa += bf16_at(qh + r * 128 + ((chunk ^ (r & 7)) << 4));
#pragma unroll 8
            for (int r = 0; r < n_b; ++r) {
                const int rr = kTile + r;
                sb += bf16_at(qh + rr * 128 + ((chunk ^ (rr & 7)) << 4));
            }
            m.qbar[0][c] = __fmul_rn(sa, __frcp_rn(static_cast<float>(n_a)));
            m.qbar[1][c] = has_b ? __fmul_rn(sb, __frcp_rn(static_cast<float>(n_b))) : 0.0f;
        }
        if (paired) {
            st_cluster_f32(cluster_addr(&m.qbar_x[0][tid], partner), m.qbar[0][tid]);
            st_cluster_f32(cluster_addr(&m.qbar_x[1][tid], partner), m.qbar[1][tid]);
        }
    }
    if (paired) {
        if (tid == 0) {
            const int mine = real ? bh : -1;
            asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(cluster_addr(&m.bh_x, partner)), "r"(mine) : "memory");
        }
        cluster_sync();
    } else {
        __syncthreads();
    }
    // A pair shares the scoring when both CTAs hold tiles of the same head (always, except at a
    // head boundary or for a CTA that only completes a cluster); otherwise each scores its own
    // tiles over every key block.
    const bool shared_head = paired && real && m.bh_x == bh;

    // ---------------- routing 2: proxy rows S_j = (q_bar . k_bar_j) * (1/sqrt d)
    float *row_a = reinterpret_cast<float *>(smem + G::kOffRowA);
    float *row_b = reinterpret_cast<float *>(smem + G::kOffRowB);
    const size_t unit_a = static_cast<size_t>(bh) * p.Nq + tile_a;
    if (paired) {
        {
            // The two CTAs of the cluster split the key blocks: rank 0 scores groups of 8 blocks
            // [0, G/2), rank 1 the rest, each for its own tiles A, B and its partner's (q_bar from
            // qbar_x), so each pooled key row is read from L2 once per cluster.  Within a CTA each
            // warp takes groups lo + w, lo + w + 6, ...  Lane l holds channels LC*l..LC*l+LC-1
            // (LC = d/32) and forms 32 partial dot products (8 blocks x 4 tiles); a reduce-scatter
            // over the lanes (31 shuffles) leaves the full sum of value l in lane l: block l & 7 of
            // tile l >> 3 (0, 1: own A, B; 2, 3: the partner's A, B, stored into its shared memory).
            // The next group's rows are loaded before the current group is reduced.
            constexpr int LC = G::kLaneCh;
            float qa[LC], qb[LC], xa[LC], xb[LC];
    #pragma unroll
            for (int c = 0; c < LC; ++c) {
                qa[c] = m.qbar[0][LC * lane + c];
                qb[c] = m.qbar[1][LC * lane + c];
                xa[c] = m.qbar_x[0][LC * lane + c];
                xb[c] = m.qbar_x[1][LC * lane + c];
            }
            const int ngroups = (Nk + 7) >> 3;
            const int half_groups = (ngroups + 1) >> 1;
            double sum_a = 0.0, sum_b = 0.0, sum_xa = 0.0, sum_xb = 0.0;
            float x[8][LC];
            const float *kb = p.kbar32 + static_cast<size_t>(bh) * Nk * D + LC * lane;
            auto load_group = [&](int grp) {
    #pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int j = 8 * grp + u;
                    if (j < Nk) {
                        load_vec<LC>(kb + static_cast<size_t>(j) * D, x[u]);
                    } else {
    #pragma unroll
                        for (int c = 0; c < LC; ++c) x[u][c] = 0.0f;
                    }
                }
            };
            const uint32_t xrow_a = cluster_addr(row_a, partner), xrow_b = cluster_addr(row_b, partner);
            const int lo = shared_head ? (cluster_rank() == 0 ? 0 : half_groups) : 0;
            const int hi = !real ? 0 : shared_head ? (cluster_rank() == 0 ? half_groups : ngroups) : ngroups;
            int g = lo + warp;
            if (g < hi) load_group(g);
            for (; g < hi; g += kNumWarps) {
                float v[32];
    #pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float da = qa[0] * x[u][0], db = qb[0] * x[u][0];
                    float ea = xa[0] * x[u][0], eb = xb[0] * x[u][0];
    #pragma unroll
                    for (int c = 1; c < LC; ++c) {
                        da = fmaf(qa[c], x[u][c], da);
                        db = fmaf(qb[c], x[u][c], db);
                        ea = fmaf(xa[c], x[u][c], ea);
                        eb = fmaf(xb[c], x[u][c], eb);
                    }
                    v[u] = da;
                    v[8 + u] = db;
                    v[16 + u] = ea;
                    v[24 + u] = eb;
                }
                const int gn = g + kNumWarps;
                if (gn < hi) load_group(gn);
                float k16[16], k8[8], k4[4], k2[2];
                const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4, h2 = lane & 2, h1 = lane & 1;
    #pragma unroll
                for (int i = 0; i < 16; ++i)
                    k16[i] = (h16 ? v[i + 16] : v[i]) + __shfl_xor_sync(0xFFFFFFFFu, h16 ? v[i] : v[i + 16], 16);
    #pragma unroll
                for (int i = 0; i < 8; ++i)
                    k8[i] = (h8 ? k16[i + 8] : k16[i]) + __shfl_xor_sync(0xFFFFFFFFu, h8 ? k16[i] : k16[i + 8], 8);
    #pragma unroll
                for (int i = 0; i < 4; ++i)
                    k4[i] = (h4 ? k8[i + 4] : k8[i]) + __shfl_xor_sync(0xFFFFFFFFu, h4 ? k8[i] : k8[i + 4], 4);
    #pragma unroll
                for (int i = 0; i < 2; ++i)
                    k2[i] = (h2 ? k4[i + 2] : k4[i]) + __shfl_xor_sync(0xFFFFFFFFu, h2 ? k4[i] : k4[i + 2], 2);
                const float tot = (h1 ? k2[1] : k2[0]) + __shfl_xor_sync(0xFFFFFFFFu, h1 ? k2[0] : k2[1], 1);
                const int j = 8 * g + (lane & 7);
                const int t = lane >> 3;   // 0, 1: own tile A, B; 2, 3: the partner's tile A, B
                if (j < Nk && (t < 2 || shared_head)) {
                    const float sc = tot * p.scale;
                    if (t == 0) {
                        row_a[j] = sc;
                        sum_a += sc;
                    } else if (t == 1) {
                        row_b[j] = sc;
                        sum_b += sc;
                    } else if (t == 2) {
                        st_cluster_f32(xrow_a + 4u * j, sc);
                        sum_xa += sc;
                    } else {
                        st_cluster_f32(xrow_b + 4u * j, sc);
                        sum_xb += sc;
                    }
                }
            }
    #pragma unroll
            for (int o = 16; o; o >>= 1) {
                sum_a += __shfl_xor_sync(0xFFFFFFFFu, sum_a, o);
                sum_b += __shfl_xor_sync(0xFFFFFFFFu, sum_b, o);
                sum_xa += __shfl_xor_sync(0xFFFFFFFFu, sum_xa, o);
                sum_xb += __shfl_xor_sync(0xFFFFFFFFu, sum_xb, o);
            }
            if (lane == 0) {
                m.red[0][warp] = sum_a;
                m.red[1][warp] = sum_b;
                st_cluster_f64(cluster_addr(&m.red_x[0][warp], partner), shared_head ? sum_xa : 0.0);
                st_cluster_f64(cluster_addr(&m.red_x[1][warp], partner), shared_head ? sum_xb : 0.0);
            }
        }
        cluster_sync();
        if (!real) return;   // a CTA that only completed the cluster (its smem is no longer read)
    } else {
        {
            // Each warp takes groups of 8 key blocks (group g = blocks 8g..8g+7; warp w takes groups
            // w, w+6, ...).  Lane l holds channels LC*l..LC*l+LC-1 (LC = d/32): it forms 16 partial
            // dot products (8 blocks x tiles A/B) and a reduce-scatter over the lanes (16 shuffles)
            // leaves the full sum of value (l >> 1) & 15 in lanes l and l^1.  The next group's rows are
            // loaded before the current group is reduced.
            constexpr int LC = G::kLaneCh;
            float qa[LC], qb[LC];
    #pragma unroll
            for (int c = 0; c < LC; ++c) {
                qa[c] = m.qbar[0][LC * lane + c];
                qb[c] = m.qbar[1][LC * lane + c];
            }
            const float *kb = p.kbar32 + static_cast<size_t>(bh) * Nk * D + LC * lane;
            const int ngroups = (Nk + 7) >> 3;
            const int my_idx = (lane >> 1) & 15;
            double sum_a = 0.0, sum_b = 0.0;
            float x[8][LC];
            auto load_group = [&](int grp) {
    #pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int j = 8 * grp + u;
                    if (j < Nk) {
                        load_vec<LC>(kb + static_cast<size_t>(j) * D, x[u]);
                    } else {
    #pragma unroll
                        for (int c = 0; c < LC; ++c) x[u][c] = 0.0f;
                    }
                }
            };
            int g = warp;
            if (g < ngroups) load_group(g);
            for (; g < ngroups; g += kNumWarps) {
                float v[16];
    #pragma unroll
                for (int u = 0; u < 8; ++u) {
                    float da = qa[0] * x[u][0], db = qb[0] * x[u][0];
    #pragma unroll
                    for (int c = 1; c < LC; ++c) {
                        da = fmaf(qa[c], x[u][c], da);
                        db = fmaf(qb[c], x[u][c], db);
                    }
                    v[u] = da;
                    v[8 + u] = db;
                }
                const int gn = g + kNumWarps;
                if (gn < ngroups) load_group(gn);
                float k8[8], k4[4], k2[2];
                const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4, h2 = lane & 2;
    #pragma unroll
                for (int i = 0; i < 8; ++i)
                    k8[i] = (h16 ? v[i + 8] : v[i]) + __shfl_xor_sync(0xFFFFFFFFu, h16 ? v[i] : v[i + 8], 16);
    #pragma unroll
                for (int i = 0; i < 4; ++i)
                    k4[i] = (h8 ? k8[i + 4] : k8[i]) + __shfl_xor_sync(0xFFFFFFFFu, h8 ? k8[i] : k8[i + 4], 8);
    #pragma unroll
                for (int i = 0; i < 2; ++i)
                    k2[i] = (h4 ? k4[i + 2] : k4[i]) + __shfl_xor_sync(0xFFFFFFFFu, h4 ? k4[i] : k4[i + 2], 4);
                const float k1 = (h2 ? k2[1] : k2[0]) + __shfl_xor_sync(0xFFFFFFFFu, h2 ? k2[0] : k2[1], 2);
                const float tot = k1 + __shfl_xor_sync(0xFFFFFFFFu, k1, 1);
                const int j = 8 * g + (my_idx & 7);
                if ((lane & 1) == 0 && j < Nk) {
                    const float sc = tot * p.scale;
                    if (my_idx < 8) {
                        row_a[j] = sc;
                        sum_a += sc;
                    } else {
                        row_b[j] = sc;
                        sum_b += sc;
                    }
                }
            }
    #pragma unroll
            for (int o = 16; o; o >>= 1) {
                sum_a += __shfl_xor_sync(0xFFFFFFFFu, sum_a, o);
                sum_b += __shfl_xor_sync(0xFFFFFFFFu, sum_b, o);
            }
            if (lane == 0) {
                m.red[0][warp] = sum_a;
                m.red[1][warp] = sum_b;
                m.red_x[0][warp] = 0.0;
                m.red_x[1][warp] = 0.0;
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        double sa = 0.0, sb = 0.0;
        for (int w = 0; w < kNumWarps; ++w) { sa += m.red[0][w]; sb += m.red[1][w]; }
        for (int w = 0; w < kNumWarps; ++w) { sa += m.red_x[0][w]; sb += m.red_x[1][w]; }
        m.mu[0] = sa / Nk;
        m.mu[1] = sb / Nk;
    }
    __syncthreads();
    // ---------------- routing 3: sigma (two-pass, double)
    {
        const double mu_a = m.mu[0], mu_b = m.mu[1];
        double ss_a = 0.0, ss_b = 0.0;
        for (int j = tid; j < Nk; j += kThreads) {
            const double da = static_cast<double>(row_a[j]) - mu_a;
            const double db = static_cast<double>(row_b[j]) - mu_b;
            ss_a += da * da;
            ss_b += db * db;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            ss_a += __shfl_xor_sync(0xFFFFFFFFu, ss_a, o);
            ss_b += __shfl_xor_sync(0xFFFFFFFFu, ss_b, o);
        }
        __syncthreads();   // everyone has read m.mu before m.red is reused
        if (lane == 0) {
            m.red[0][warp] = ss_a;
            m.red[1][warp] = ss_b;
        }
    }
    __syncthreads();
    if (tid == 0) {
        for (int t = 0; t < 2; ++t) {
            double ss = 0.0;
            for (int w = 0; w < kNumWarps; ++w) ss += m.red[t][w];
            const double sigma = sqrt(ss / Nk);
            double tau;
            const float beta = p.beta_head ? p.beta_head[bh] : p.beta;
            if (isinf(beta)) tau = beta < 0.0f ? -INFINITY : INFINITY;
            else tau = m.mu[t] + static_cast<double>(beta) * sigma;   // NaN beta: NaN tau, nothing kept
            m.sigma[t] = sigma;
            m.tau[t] = tau;
        }
        if (p.dbg_stats) {
            for (int t = 0; t < (has_b ? 2 : 1); ++t) {
                float *st = p.dbg_stats + (unit_a + t) * 3;
                st[0] = static_cast<float>(m.mu[t]);
                st[1] = static_cast<float>(m.sigma[t]);
                st[2] = static_cast<float>(m.tau[t]);
            }
        }
    }
    __syncthreads();
    // ---------------- routing 4: keep masks (ballot per 32 blocks), counts, debug rows
    constexpr bool by_rank = kRank;   // top-k / top-p instead of mu + beta*sigma
    if constexpr (by_rank) radix_select(row_a, row_b, has_b, Nk, m, p);
    const int nwords = (Nk + 31) >> 5;
    {
        const double tau_a = m.tau[0], tau_b = m.tau[1];
        int cnt_a = 0, cnt_b = 0;
        uint32_t min_a = 0xFFFFFFFFu, min_b = 0xFFFFFFFFu;
        for (int wd = warp; wd < nwords; wd += kNumWarps) {
            const int j = wd * 32 + lane;
            const bool inb = j < Nk;
            const float sa = inb ? row_a[j] : 0.0f;
            const float sb = inb ? row_b[j] : 0.0f;
            bool ka, kb;
            if constexpr (by_rank) {
                const uint32_t ya = score_key(sa), yb = score_key(sb);
                ka = inb && sel_keep(m, 0, ya);
                kb = inb && has_b && sel_keep(m, 1, yb);
                if (ka) min_a = min(min_a, ya);
                if (kb) min_b = min(min_b, yb);
            } else {
                ka = inb && static_cast<double>(sa) >= tau_a;
                kb = inb && has_b && static_cast<double>(sb) >= tau_b;
            }
            const uint32_t wa = __ballot_sync(0xFFFFFFFFu, ka);
            const uint32_t wb = __ballot_sync(0xFFFFFFFFu, kb);
            if (lane == 0) {
                m.mask_a[wd] = wa;
                m.mask_b[wd] = wb;
                m.mask_u[wd] = wa | wb;
                cnt_a += __popc(wa);
                cnt_b += __popc(wb);
            }
            if (inb && p.dbg_proxy) {
                p.dbg_proxy[unit_a * Nk + j] = sa;
                if (has_b) p.dbg_proxy[(unit_a + 1) * Nk + j] = sb;
            }
        }
        if (lane == 0) {
            atomicAdd(&m.count_a, cnt_a);
            atomicAdd(&m.count_b, cnt_b);
        }
        if constexpr (by_rank) {
            min_a = __reduce_min_sync(0xFFFFFFFFu, min_a);
            min_b = __reduce_min_sync(0xFFFFFFFFu, min_b);
            if (lane == 0) {
                atomicMin(&m.sel_min[0], min_a);
                atomicMin(&m.sel_min[1], min_b);
            }
        }
    }
    __syncthreads();
    if constexpr (by_rank) {
        if (tid == 0) thin_ties(m.mask_a, row_a, Nk, m, 0, &m.count_a);
        if (tid == 32) thin_ties(m.mask_b, row_b, Nk, m, 1, &m.count_b);
        __syncthreads();
        for (int wd = tid; wd < nwords; wd += kThreads) m.mask_u[wd] = m.mask_a[wd] | m.mask_b[wd];
        if (tid == 0 && p.dbg_stats) {
            // threshold statistic of a rank rule: the score of the last kept block
            for (int t = 0; t < (has_b ? 2 : 1); ++t)
                p.dbg_stats[(unit_a + t) * 3 + 2] =
                    (t ? m.count_b : m.count_a) == 0 ? INFINITY : key_score(m.sel_min[t]);
        }
        __syncthreads();
    }
    if (p.dbg_mask) {
        for (int j = tid; j < Nk; j += kThreads) {
            p.dbg_mask[unit_a * Nk + j] = (m.mask_a[j >> 5] >> (j & 31)) & 1u;
            if (has_b) p.dbg_mask[(unit_a + 1) * Nk + j] = (m.mask_b[j >> 5] >> (j & 31)) & 1u;
        }
    }
    // correction chunks that still hold a block skipped by tile A (or by an existing tile B)
    {
        for (int c = tid; c < p.nchunks; c += kThreads) {
            uint32_t need = 0;
            for (int h = 0; h < 2; ++h) {
                const int wd = 2 * c + h;
                if (wd >= nwords) continue;
                const int rem = Nk - wd * 32;
                const uint32_t valid = rem >= 32 ? 0xFFFFFFFFu : ((1u << rem) - 1u);
                need |= valid & ~(m.mask_a[wd] & (has_b ? m.mask_b[wd] : 0xFFFFFFFFu));
            }
            if (need) atomicOr(&m.need[c >> 5], 1u << (c & 31));
        }
        if (tid == 0 && p.density) {
            p.density[unit_a] = m.count_a;
            if (has_b) p.density[unit_a + 1] = m.count_b;
        }
    }
    if (split_n > 1) {
        __syncthreads();                          // need and mask_u are complete
        if (warp == 0) keep_half_of_walk(m, p, split_half);
    }
    fence_proxy_async_smem();   // generic writes to the ring happen-before the TMA overwrites it
    __syncthreads();

    // ---------------- pipeline
    const bool aborted = volatile_load(&m.abort_flag) != 0;
    if (warp == kWarpTma) {
        if (lane == 0) {
            if (!aborted) producer_role<D>(&tm_k, &tm_v, &tm_kb, &tm_vb, smem, m, p, bh);
            wait_bar(&m.q_full, 0, m, p, kSiteProdDrain, false);   // the Q copy has landed
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        if (lane == 0 && !aborted) mma_role<D>(tmem, smem, m, p);
        __syncwarp();
    } else if (!aborted) {
        softmax_role<D>(tmem, m, p, bh, row0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Work units run as two CTAs each when they do not fill the last wave of CTAs (two resident per
// SM): about 1.5 times the units of a last wave that is at most half full.  On the 12-head,
// 16384-token call that splits 84 of 1536 units (56 past five full waves of 296): 1.9 % faster at
// d = 128 and 3 % at d = 64, measured with the merge (without it, 84 to 150 split units were
// equally good).  A fuller last wave, or a call of less than one wave, splits nothing.
long long split_units(long long units, int slots, int cap)
{
    if (cap <= 0 || slots <= 0 || units <= slots) return 0;
    const long long tail = units % slots;
    if (tail == 0 || 2 * tail > slots) return 0;
    return std::min<long long>(std::min<long long>(cap, units), tail + tail / 2);
}

template <int D, bool kRank>
cudaError_t launch_d(const FwdLaunch &L, cudaStream_t stream)
{
    static std::once_flag attr_once[64];
    static int sm_count[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    constexpr uint32_t kSmem = smem_bytes<D>();
    cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once[dev], [&] {
        attr_err = cudaFuncSetAttribute(sol_fwd_kernel<D, kRank>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kSmem));
        if (attr_err == cudaSuccess)
            attr_err = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
    });
    if (attr_err != cudaSuccess) return attr_err;

    Params p{};
    p.BH = L.BH;
    p.N = L.N;
    p.Nk = L.Nk;
    p.Nq = L.Nq;
    p.npairs = (L.Nq + 1) / 2;
    p.nchunks = (L.Nk + 63) / 64;
    p.beta = L.beta;
    p.beta_head = L.beta_head;
    p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    const int n_last = L.N - (L.Nk - 1) * kTile;
    p.last_bias_log2 = static_cast<float>(std::log2(static_cast<double>(n_last)));
    p.kbar32 = L.kbar32;
    p.out = static_cast<__nv_bfloat16 *>(L.out);
    p.density = L.density;
    p.status = L.status;
    p.dbg_proxy = L.dbg_proxy;
    p.dbg_mask = L.dbg_mask;
    p.dbg_stats = L.dbg_stats;
    p.fault_flags = L.fault_flags;
    p.timeout_ns = L.timeout_ns;
    p.route = L.route;
    p.topk = L.topk;
    p.topp = L.topp;
    // The split is decided for the whole call (a launch may cover one head group of it) and each
    // launch splits its own units that fall among the call's last ones, so that a call run in
    // head groups gives the same output as one launch.
    const long long units = static_cast<long long>(p.npairs) * L.BH;
    const long long call_units = L.call_units > 0 ? L.call_units : units;
    const long long S_call = L.split_all ? std::min<long long>(call_units, std::max(L.split_cap, 0))
                                         : split_units(call_units, 2 * sm_count[dev], L.split_cap);
    const long long first_call = call_units - S_call;
    const long long first_local = std::min(units, std::max(0LL, first_call - L.unit0));
    const long long S = units - first_local;
    p.split_first = static_cast<int>(first_local);
    p.split_slot0 = static_cast<int>(L.unit0 + first_local - first_call);
    p.split_cnt = L.split_cnt;
    p.split_part = L.split_part;
    // a fresh tag per launch, 1 .. 2^29 - 1 (tag << 2 | count stays a positive int)
    static std::atomic<unsigned> launch_tag{0};
    p.split_gen = static_cast<int>(launch_tag.fetch_add(1u, std::memory_order_relaxed) % 0x1FFFFFFFu) + 1;
    // Clusters of two share the proxy scoring's reads of the pooled keys.  Measured on B200: the
    // 32-head 262144-token call (4096 key blocks) ran 2.2 % faster, the 12-head 16384-token and
    // 40-head 75600-token calls (256 and 1182 blocks) 1-5 % slower (a cluster needs two free CTA
    // slots at once), so only calls with at least kPairMinBlocks key blocks use them.
    constexpr int kPairMinBlocks = 2048;
    p.pair = L.Nk >= kPairMinBlocks ? 1 : 0;
    const long long grid_real = units + S;
    const long long grid = p.pair ? (grid_real + 1) & ~1LL : grid_real;
    if (units <= 0 || grid > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    p.grid_real = static_cast<int>(grid_real);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.pair ? 2 : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, sol_fwd_kernel<D, kRank>, *L.tm_q, *L.tm_k, *L.tm_v, *L.tm_kb, *L.tm_vb, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sol_fwd(const FwdLaunch &L, cudaStream_t stream)
{
    const bool rank = L.route != kRouteThreshold;
    if (L.d == 128) return rank ? launch_d<128, true>(L, stream) : launch_d<128, false>(L, stream);
    if (L.d == 64) return rank ? launch_d<64, true>(L, stream) : launch_d<64, false>(L, stream);
    return cudaErrorInvalidValue;
}

}  // namespace sol
