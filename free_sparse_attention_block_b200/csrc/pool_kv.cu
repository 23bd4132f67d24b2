// K/V block pooling: k_bar_j = (sum of the block's keys, float32, ascending token order) * (1/n_j),
// the same for values, plus round-to-nearest-even bfloat16 copies for the tensor-core correction.
// ("Sol-Attn", routing paragraphs: a block is scored through a block-level summary of its keys;
// skipped blocks are approximated by their pooled key and value.)
//
// HBM-bound streaming kernel: a group of d/CPL lanes (CPL = 4 channels per lane: a full warp for
// d = 128, a half-warp for d = 64) owns one 64-token block of K or V; lane l of the group owns
// channels CPL*l .. CPL*l+CPL-1 and reads them as one 8-byte vector per token, so a warp
// instruction reads 256 contiguous bytes of rows.  Each channel is summed sequentially over the
// block's tokens, which fixes the float32 rounding order.  Measured on B200 (12 heads x 16384
// tokens / 40 heads x 75600 tokens): CPL = 8 3.0 / 6.3 TB/s, CPL = 4 3.4 / 6.4 TB/s, CPL = 2
// 3.4 / 6.4 TB/s -- at small sizes more lanes per block keep more loads in flight.
#include <cuda_bf16.h>

#include "internal.h"

namespace sol {
namespace {

constexpr int kPoolThreads = 256;

// CPL bf16 channels of one token row, loaded as one 4/8/16-byte vector.
template <int CPL> struct RowVec;
template <> struct RowVec<8> { using T = uint4; };
template <> struct RowVec<4> { using T = uint2; };
template <> struct RowVec<2> { using T = uint32_t; };

template <int CPL>
__device__ __forceinline__ void add_bf16(float (&acc)[CPL], const typename RowVec<CPL>::T &u)
{
    const uint32_t *w = reinterpret_cast<const uint32_t *>(&u);
#pragma unroll
    for (int i = 0; i < CPL / 2; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

#ifndef SOL_POOL_CPL
#define SOL_POOL_CPL 4
#endif

template <int D, int CPL>
__global__ void __launch_bounds__(kPoolThreads) pool_kv_kernel(
    const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v, int BH, int N, int Nk,
    float *__restrict__ kbar32, float *__restrict__ vbar32, __nv_bfloat16 *__restrict__ kbar16,
    __nv_bfloat16 *__restrict__ vbar16, int *__restrict__ clear, int clear_words)
{
    if (blockIdx.x == 0 && clear != nullptr) {
        for (int i = threadIdx.x; i < clear_words; i += kPoolThreads) clear[i] = 0;
    }
    using Vec = typename RowVec<CPL>::T;
    constexpr int kLanes = D / CPL;                        // lanes per block = vectors per token row
    const long long grp = (static_cast<long long>(blockIdx.x) * kPoolThreads + threadIdx.x) / kLanes;
    const int sub = threadIdx.x & (kLanes - 1);            // channels CPL*sub .. CPL*sub+CPL-1
    const long long per_tensor = static_cast<long long>(BH) * Nk;
    if (grp >= 2 * per_tensor) return;
    const bool is_v = grp >= per_tensor;
    const long long blk = is_v ? grp - per_tensor : grp;   // bh * Nk + j
    const int bh = static_cast<int>(blk / Nk);
    const int j = static_cast<int>(blk - static_cast<long long>(bh) * Nk);
    const int n = min(kTile, N - j * kTile);

    const Vec *src = reinterpret_cast<const Vec *>((is_v ? v : k) + (static_cast<long long>(bh) * N + j * kTile) * D) + sub;
    float acc[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) acc[i] = 0.0f;
    if (n == kTile) {
#pragma unroll 16
        for (int t = 0; t < kTile; ++t) add_bf16<CPL>(acc, __ldg(src + t * kLanes));
    } else {
        for (int t = 0; t < n; ++t) add_bf16<CPL>(acc, __ldg(src + t * kLanes));
    }
    const float inv = __frcp_rn(static_cast<float>(n));
    float r[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) r[i] = __fmul_rn(acc[i], inv);

    float *d32 = (is_v ? vbar32 : kbar32) + blk * D + sub * CPL;
#pragma unroll
    for (int i = 0; i < CPL; i += 2) reinterpret_cast<float2 *>(d32)[i / 2] = make_float2(r[i], r[i + 1]);
    Vec packed;
    uint32_t *pw = reinterpret_cast<uint32_t *>(&packed);
#pragma unroll
    for (int i = 0; i < CPL / 2; ++i) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(r[2 * i], r[2 * i + 1]);
        pw[i] = *reinterpret_cast<uint32_t *>(&h2);
    }
    __nv_bfloat16 *d16 = (is_v ? vbar16 : kbar16) + blk * D + sub * CPL;
    *reinterpret_cast<Vec *>(d16) = packed;
}

}  // namespace

cudaError_t launch_pool_kv(const void *k, const void *v, int BH, int N, int Nk, int d, float *kbar32,
                           float *vbar32, void *kbar16, void *vbar16, int *clear, int clear_words,
                           cudaStream_t stream)
{
    if (!head_dim_supported(d)) return cudaErrorInvalidValue;
    constexpr int kCpl = SOL_POOL_CPL;
    const long long threads = 2LL * BH * Nk * (d / kCpl);
    const long long blocks = (threads + kPoolThreads - 1) / kPoolThreads;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    auto kern = d == 64 ? pool_kv_kernel<64, kCpl> : pool_kv_kernel<128, kCpl>;
    kern<<<static_cast<unsigned>(blocks), kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), BH, N, Nk,
        kbar32, vbar32, static_cast<__nv_bfloat16 *>(kbar16), static_cast<__nv_bfloat16 *>(vbar16), clear,
        clear_words);
    return cudaGetLastError();
}

}  // namespace sol
