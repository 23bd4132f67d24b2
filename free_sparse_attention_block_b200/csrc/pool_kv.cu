// K/V block pooling: k_bar_j = (sum of the block's keys, float32, ascending token order) * (1/n_j),
// the same for values, plus round-to-nearest-even bfloat16 copies for the tensor-core correction.
// ("Sol-Attn", routing paragraphs: a block is scored through a block-level summary of its keys;
// skipped blocks are approximated by their pooled key and value.)
//
// HBM-bound streaming kernel: a group of d/8 lanes (a half-warp for d = 128, a quarter-warp for
// d = 64) owns one 64-token block of K or V; lane l of the group owns channels 8l..8l+7 and reads
// them as one 16-byte vector per token, so a warp instruction reads 512 contiguous bytes of rows.
// Each channel is summed sequentially over the block's tokens, which fixes the float32 rounding
// order.
#include <cuda_bf16.h>

#include "internal.h"

namespace sol {
namespace {

constexpr int kPoolThreads = 256;

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 &u)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kv_kernel(
    const uint4 *__restrict__ k, const uint4 *__restrict__ v, int BH, int N, int Nk,
    float *__restrict__ kbar32, float *__restrict__ vbar32, __nv_bfloat16 *__restrict__ kbar16,
    __nv_bfloat16 *__restrict__ vbar16)
{
    constexpr int kLanes = D / 8;                          // lanes per block = uint4 per token row
    const long long grp = (static_cast<long long>(blockIdx.x) * kPoolThreads + threadIdx.x) / kLanes;
    const int sub = threadIdx.x & (kLanes - 1);            // channel group: 8*sub .. 8*sub+7
    const long long per_tensor = static_cast<long long>(BH) * Nk;
    if (grp >= 2 * per_tensor) return;
    const bool is_v = grp >= per_tensor;
    const long long blk = is_v ? grp - per_tensor : grp;   // bh * Nk + j
    const int bh = static_cast<int>(blk / Nk);
    const int j = static_cast<int>(blk - static_cast<long long>(bh) * Nk);
    const int n = min(kTile, N - j * kTile);

    const uint4 *src = (is_v ? v : k) + (static_cast<long long>(bh) * N + j * kTile) * kLanes + sub;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    if (n == kTile) {
#pragma unroll 16
        for (int t = 0; t < kTile; ++t) add_bf16x8(acc, __ldg(src + t * kLanes));
    } else {
        for (int t = 0; t < n; ++t) add_bf16x8(acc, __ldg(src + t * kLanes));
    }
    const float inv = __frcp_rn(static_cast<float>(n));
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = __fmul_rn(acc[i], inv);

    float *d32 = (is_v ? vbar32 : kbar32) + blk * D + sub * 8;
    reinterpret_cast<float4 *>(d32)[0] = make_float4(r[0], r[1], r[2], r[3]);
    reinterpret_cast<float4 *>(d32)[1] = make_float4(r[4], r[5], r[6], r[7]);
    uint4 packed;
    uint32_t *pw = reinterpret_cast<uint32_t *>(&packed);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(r[2 * i], r[2 * i + 1]);
        pw[i] = *reinterpret_cast<uint32_t *>(&h2);
    }
    __nv_bfloat16 *d16 = (is_v ? vbar16 : kbar16) + blk * D + sub * 8;
    *reinterpret_cast<uint4 *>(d16) = packed;
}

}  // namespace

cudaError_t launch_pool_kv(const void *k, const void *v, int BH, int N, int Nk, int d, float *kbar32,
                           float *vbar32, void *kbar16, void *vbar16, cudaStream_t stream)
{
    if (!head_dim_supported(d)) return cudaErrorInvalidValue;
    const long long threads = 2LL * BH * Nk * (d / 8);
    const long long blocks = (threads + kPoolThreads - 1) / kPoolThreads;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    auto kern = d == 64 ? pool_kv_kernel<64> : pool_kv_kernel<128>;
    kern<<<static_cast<unsigned>(blocks), kPoolThreads, 0, stream>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), BH, N, Nk, kbar32, vbar32,
        static_cast<__nv_bfloat16 *>(kbar16), static_cast<__nv_bfloat16 *>(vbar16));
    return cudaGetLastError();
}

}  // namespace sol
