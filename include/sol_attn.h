/*
 * sol_attn.h: C ABI of the Sol-Attn block-sparse attention forward for NVIDIA B200 (sm_100a).
 *
 * The operation is the forward pass of "Sol-Attn: Accelerating Video Generation Inference via
 * On-the-Fly Attention Sparsification" (Li et al., 2026).  Its routing paragraphs define the
 * block choice: a query's pre-softmax proxy scores against key blocks are reduced to a row mean
 * mu and standard deviation sigma, and a block is computed exactly iff its score is at least
 * tau = mu + beta*sigma (one global beta).  The fused-operator paragraph puts routing, the exact
 * sparse attention and an approximation of every skipped block into one online-softmax pass.
 * Readings fixed by this library where the page is silent:
 *   - query tiles and key blocks are T = 64 tokens; Nq = Nk = ceil(N / 64); the last tile/block
 *     may be partial with n_j = N - 64*(Nk-1) tokens;
 *   - routing is per query tile i: S_ij = (q_bar_i . k_bar_j) / sqrt(d) with q_bar_i, k_bar_j the
 *     float32 means of the tile's queries / the block's keys; mu_i and population sigma_i of row i
 *     (accumulated in double); block j is kept for tile i iff S_ij >= tau_i; beta = -inf keeps
 *     every block, beta = +inf keeps none;
 *   - a skipped block j contributes one softmax term to each row r of the tile, with logit
 *     (q_r . k_bar_j)/sqrt(d) + ln(n_j) and value v_bar_j (so it adds n_j*exp(q.k_bar/sqrt d - m)
 *     to the denominator and that weight times v_bar_j to the numerator);
 *   - bidirectional (no causal mask), forward only.
 *
 * Conventions for every entry point:
 *   - q, k, v, out: bfloat16, contiguous [B, H, N, d] (token rows of d elements), device
 *     pointers, 16-byte aligned.  d is 64 or 128 (the video DiT head sizes; the paper's models
 *     use 128).  1 <= N <= 524288.  B*H*ceil(Nq/2) < 2^31.
 *   - The caller owns all memory.  The library allocates no device or host memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     stream-ordered.  sol_attn_fwd needs a prior sol_attn_pool on the same K, V and workspace,
 *     earlier in stream order.
 *   - Errors are returned, never thrown.  Argument errors are detected on the host before any
 *     launch.  SOL_ERR_CUDA means a CUDA runtime/driver call or launch failed.
 *   - Device-side failures (a pipeline wait that ran out of time) are recorded in a status word
 *     inside the workspace; sol_attn_read_status() synchronises the stream and returns it.
 *   - The library keeps no state between calls apart from per-device one-time set-up (kernel
 *     attributes, the SM count that sizes the split of the last wave of CTAs, the driver entry
 *     point for tensor-map encoding, and the two copy streams and the events sol_attn_fwd_host
 *     pipelines its copies with) and a process-wide launch counter (it tags the workspace's
 *     split counters, so that counters a failed call left behind never count for a later call);
 *     it is thread-safe.  Calls that share a workspace must not overlap on the GPU.
 */
#ifndef SOL_ATTN_H
#define SOL_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SOL_OK = 0,
    SOL_ERR_INVALID_ARG = 1, /* null pointer, non-positive or too large size, NaN beta */
    SOL_ERR_UNSUPPORTED = 2, /* d not 64 or 128, N above the supported maximum */
    SOL_ERR_ALIGNMENT = 3,   /* a tensor pointer that is not 16-byte aligned */
    SOL_ERR_CUDA = 4,        /* a CUDA call or kernel launch failed */
    SOL_ERR_TIMEOUT = 5,     /* a device pipeline wait gave up (see sol_attn_read_status) */
    SOL_ERR_SCRATCH_LIMIT = 6 /* sol_attn_fwd_noalloc: the shape needs more scratch than it has */
} sol_status;

/* Bytes of device workspace sol_attn_pool/sol_attn_fwd need for this shape: a 1 KB header
 * (status words and the counters of split tile pairs), the pooled keys and values, float32
 * [B,H,Nk,d] each, their bfloat16 copies [B,H,Nk,d] each, and room for the partial output rows
 * of up to 128 tile pairs that the forward splits over two CTAs to fill its last wave of CTAs
 * (2 x 128 rows x (d + 4) float32 per pair; 17 MB at d = 128 once the call has 128 tile pairs).
 * Returns 0 for an invalid or unsupported shape. */
size_t sol_attn_workspace_bytes(int B, int H, int N, int d);

/* Mean-pool K and V into 64-token blocks (the k_bar_j / v_bar_j of the routing and of the
 * correction of skipped blocks).  k_bar_j[c] = (float32 sum of k_t[c] over the block's tokens in
 * ascending order) * (1.0f / n_j); the same for v; the bfloat16 copies are round-to-nearest-even
 * of the float32 values.  Also clears the workspace status words.
 * workspace: device, >= sol_attn_workspace_bytes(B,H,N,d) bytes, 256-byte aligned. */
sol_status sol_attn_pool(const void *k, const void *v, int B, int H, int N, int d,
                         void *workspace, void *stream);

/* Fused Sol-Attn forward: per query tile, builds the proxy row against the pooled keys in shared
 * memory (never in global memory), reduces it to mu/sigma, keeps the blocks at or above tau, runs
 * exact attention over the kept blocks and one pooled term per skipped block in a single
 * online-softmax pass, and writes out = softmax-weighted values rounded to bfloat16.
 * beta: any non-NaN float, +-inf allowed.
 * density_out: device int32 [B,H,Nq], number of kept blocks per query tile, or NULL.
 * workspace: the one sol_attn_pool filled for this K, V (its status words may be written, and
 * the split region is used as scratch; calls that share a workspace must not overlap on the GPU).
 * Work unit: a pair of query tiles of one head per CTA.  When the units do not fill the last wave
 * of CTAs (two per SM), the last units run as two CTAs each, every other item of the unit's work
 * list on each; the second of the two to finish merges both partial rows (their own running max
 * and sum) into the output.  Calls with at least 2048 key blocks (N > 131008) launch the CTAs in
 * clusters of two that split the proxy scoring's reads of the pooled keys.  The result is the
 * same attention up to float rounding order. */
sol_status sol_attn_fwd(const void *q, const void *k, const void *v, int B, int H, int N, int d,
                        float beta, void *workspace, void *out, int32_t *density_out,
                        void *stream);

/* sol_attn_fwd with one beta per head: beta_per_head is a device float array [B*H] (index
 * b*H + h), 4-byte aligned.  Entries may be +-inf; a NaN entry gives a NaN threshold, so that
 * head keeps no block.  This is the per-head form of the threshold paragraph's single global
 * offset, used to hold every head at the same target density (see the Python helper
 * calibrate_betas). */
sol_status sol_attn_fwd_betas(const void *q, const void *k, const void *v, int B, int H, int N,
                              int d, const float *beta_per_head, void *workspace, void *out,
                              int32_t *density_out, void *stream);

/* Block-selection rules.  SOL_ROUTE_THRESHOLD is the paper's rule (keep S_ij >= mu_i + beta*sigma_i).
 * SOL_ROUTE_TOPK and SOL_ROUTE_TOPP are the two prior-art rules the paper's routing paragraph
 * contrasts it with (a fixed number of blocks per query; blocks until their cumulative probability
 * reaches a threshold).  They run on the same proxy row inside the same fused kernel; only the
 * keep decision differs.  Readings fixed by this library:
 *   - blocks are ranked by proxy score, highest first; equal scores (-0.0 equals +0.0) rank the
 *     lower block index first;
 *   - top-k keeps the first min(k, Nk) blocks of every query tile's row;
 *   - top-p gives block j the probability w_j / Z, w_j = exp(S_ij - max_j S_ij) in double,
 *     Z = sum_j w_j (no weighting by token count), and keeps the shortest prefix of the ranking
 *     whose probability reaches p (block j is kept iff the mass ranked before it is < p*Z);
 *     p <= 0 keeps none, p >= 1 keeps every block.  The float64 sums are accumulated in an
 *     unspecified order, so a prefix whose mass lies within about 1e-12*Z of p*Z may end one
 *     block earlier or later than an exact evaluation;
 *   - skipped blocks get the same pooled correction term as under the threshold rule. */
typedef enum {
    SOL_ROUTE_THRESHOLD = 0,
    SOL_ROUTE_TOPK = 1,
    SOL_ROUTE_TOPP = 2
} sol_route;

/* sol_attn_fwd with the top-k rule: k_blocks >= 0 blocks kept per query tile (values above Nk keep
 * every block).  density_out then holds min(k_blocks, Nk) for every tile.  Negative k_blocks:
 * SOL_ERR_INVALID_ARG.  Other arguments as for sol_attn_fwd. */
sol_status sol_attn_fwd_topk(const void *q, const void *k, const void *v, int B, int H, int N,
                             int d, int k_blocks, void *workspace, void *out,
                             int32_t *density_out, void *stream);

/* sol_attn_fwd with the top-p rule: p is the probability mass to cover per query tile (any
 * non-NaN float; see sol_route for <= 0 and >= 1).  NaN p: SOL_ERR_INVALID_ARG. */
sol_status sol_attn_fwd_topp(const void *q, const void *k, const void *v, int B, int H, int N,
                             int d, float p, void *workspace, void *out, int32_t *density_out,
                             void *stream);

/* sol_attn_fwd_debug for any rule: route selects the rule and param is its parameter (beta for
 * SOL_ROUTE_THRESHOLD, k for SOL_ROUTE_TOPK -- an integral value >= 0 --, p for SOL_ROUTE_TOPP).
 * Debug outputs as for sol_attn_fwd_debug; for the rank rules stats_out[...,2] holds the score of
 * the last kept block (+inf when none is kept) instead of mu + beta*sigma.  Synchronises the
 * stream and returns the device status.  An unknown route or an invalid param:
 * SOL_ERR_INVALID_ARG. */
sol_status sol_attn_fwd_debug_route(const void *q, const void *k, const void *v, int B, int H,
                                    int N, int d, int route, float param, void *workspace,
                                    void *out, int32_t *density_out, float *proxy_out,
                                    uint8_t *mask_out, float *stats_out, void *stream);

/* Test/diagnostic variant of sol_attn_fwd: the same computation plus optional debug outputs,
 * then a stream synchronisation and a read of the device status.  Not for production use.
 *   proxy_out  device float [B,H,Nq,Nk]: the proxy rows S_ij (or NULL)
 *   mask_out   device uint8 [B,H,Nq,Nk]: 1 = block kept (or NULL)
 *   stats_out  device float [B,H,Nq,3]: mu_i, sigma_i, tau_i (or NULL)
 *   fault_flags bit 0: the MMA issuer waits on a barrier nothing signals, so the pipeline wait
 *               runs out and the call must return SOL_ERR_TIMEOUT with the context intact.
 *               bit 1: split every work unit the workspace has room for (up to 128 tile pairs)
 *               over two CTAs, whatever the wave shape (tests of the merge on small shapes).
 *               bit 2: the first half of a split unit publishes its rows but not its final
 *               count, so the other half's wait for them runs out (SOL_ERR_TIMEOUT).
 *   timeout_ms: limit for each device wait; <= 0 selects the production default (2000 ms).
 * Returns SOL_ERR_TIMEOUT if any device wait ran out, else the launch status. */
sol_status sol_attn_fwd_debug(const void *q, const void *k, const void *v, int B, int H, int N,
                              int d, float beta, void *workspace, void *out,
                              int32_t *density_out, float *proxy_out, uint8_t *mask_out,
                              float *stats_out, int fault_flags, int timeout_ms, void *stream);

/* Synchronise `stream`, read the device status words in the workspace header and clear them.
 * workspace NULL reads the status words of sol_attn_fwd_noalloc's built-in scratch on the current
 * device instead.  Returns SOL_OK, SOL_ERR_TIMEOUT (a device wait gave up) or SOL_ERR_CUDA.  If
 * where_out is not NULL it receives an internal code naming the wait that gave up (0 if none).
 * A call that gave up leaves no state that misleads a later call on the same workspace, whether or
 * not its status was read: the counters of split tile pairs carry a tag of the launch that wrote
 * them, and another launch's tag counts as zero. */
sol_status sol_attn_read_status(void *workspace, int *where_out, void *stream);

/* One end-to-end call on host buffers: copies q, k, v from (preferably pinned) host memory into
 * the caller's device buffers, pools, runs the forward, and copies out and density back, without
 * synchronising.  The heads are split into contiguous groups (about one per 32 MiB of upload, at
 * most 32 when one head's tile pairs fill their last wave of CTAs at least 90 %, else at most 8;
 * the first and the last group half the size of the others) and the copies are pipelined
 * with the compute: group g+1 uploads on an internal copy stream while `stream` pools and runs
 * group g, and group g's output downloads on a second internal copy stream while later groups
 * compute.  The uploads wait for all work queued on `stream` before this call, and everything
 * (the last download included) is ordered before work queued on `stream` after it, so the device
 * buffers may be reused by the next call.  Host buffers must stay valid until `stream` reaches
 * that point.  An error returned after copies were queued keeps that ordering (as far as the
 * failing CUDA runtime allows), so the same rule applies.  h_density / d_density may both be NULL.
 * workspace: 256-byte aligned, as for sol_attn_pool.  Results are bit-identical to sol_attn_pool +
 * sol_attn_fwd. */
sol_status sol_attn_fwd_host(const void *h_q, const void *h_k, const void *h_v, int B, int H,
                             int N, int d, float beta, void *d_q, void *d_k, void *d_v,
                             void *workspace, void *d_out, int32_t *d_density, void *h_out,
                             int32_t *h_density, void *stream);

/* Bytes of scratch built into the library for sol_attn_fwd_noalloc (16 MiB, one array per GPU
 * that loads the library, held until the process exits). */
#define SOL_ATTN_NOALLOC_MAX_BYTES (16u * 1024u * 1024u)

/* sol_attn_pool + sol_attn_fwd for callers that cannot allocate device memory: code that runs
 * inside a fixed memory budget, a host framework whose allocator must not be called back from
 * here, or a plugin without an allocator of its own.  The paper has no counterpart; this is a
 * packaging of the same two kernels.  Inputs and outputs are the caller's (as for sol_attn_fwd);
 * the pooled keys/values and status words go to a scratch array inside the library instead of a
 * caller workspace.  This entry point calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Limit: the call's pooled keys and values (12 bytes per pooled channel) and a 1 KB header
 *     fit in SOL_ATTN_NOALLOC_MAX_BYTES, i.e. B*H*ceil(N/64) <= 10922 pooled rows at d = 128,
 *     21844 at d = 64 (a 12-head, 16384-token call fits); larger shapes return
 *     SOL_ERR_SCRATCH_LIMIT without launching anything.  This entry point never splits a tile
 *     pair over two CTAs (the scratch has no room for the partial rows), so its last wave of
 *     CTAs may run less full than sol_attn_fwd's.
 *   - The first call on each device looks up the scratch array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before any stream
 *     capture.  A lookup that fails returns SOL_ERR_CUDA and is retried by the next call.
 *   - Every call on a device shares the one array and leaves its contents behind; each call
 *     clears the status words and rewrites all pooled rows it reads before use.  Calls whose
 *     execution overlaps on the GPU (different streams, or graphs launched concurrently) race on
 *     the array: serialise them.
 *   - Device-side wait timeouts are recorded in the scratch status words; sol_attn_read_status
 *     with a NULL workspace synchronises the stream and reads (and clears) them.
 * Other arguments, errors and asynchrony as for sol_attn_fwd. */
sol_status sol_attn_fwd_noalloc(const void *q, const void *k, const void *v, int B, int H, int N,
                                int d, float beta, void *out, int32_t *density_out, void *stream);

/* Static English description of a status code. */
const char *sol_attn_error_string(sol_status status);

#ifdef __cplusplus
}
#endif

#endif /* SOL_ATTN_H */
