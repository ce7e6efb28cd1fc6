// lb_pack.cu - sign packing: float / int8 factors -> packed +-1 words.
//
// Layout (include/lb.h): word w of a packed row holds columns 32w .. 32w+31;
// bit j is 1 iff column 32w + j is strictly negative.  Every entry of a
// binarized factor is +1 or -1 and costs one bit (sesamedisk.com, "Samsung
// LittleBit 13B Model", section "How low-rank binarization works").
//
// U is packed along its rows (along r).  V [n_in x r] is packed as V^T: one
// packed row per latent index k, along n_in, so both contractions of the
// forward pass stream their factor with the contraction index innermost.
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"

namespace lb {
namespace {

// Strictly negative: sign bit set, not +-0, not NaN.  Integer tests on the bit
// pattern, so the result does not depend on denormal flushing.
__device__ __forceinline__ bool neg_f32(uint32_t b)
{
    return (b >> 31) && (b & 0x7fffffffu) && !(((b & 0x7f800000u) == 0x7f800000u) && (b & 0x007fffffu));
}
__device__ __forceinline__ bool neg_f16(uint32_t b)
{
    return (b & 0x8000u) && (b & 0x7fffu) && !(((b & 0x7c00u) == 0x7c00u) && (b & 0x03ffu));
}
__device__ __forceinline__ bool neg_bf16(uint32_t b)
{
    return (b & 0x8000u) && (b & 0x7fffu) && !(((b & 0x7f80u) == 0x7f80u) && (b & 0x007fu));
}

template <int DT>
__device__ __forceinline__ bool is_negative(const void *src, int64_t idx)
{
    if constexpr (DT == LB_F32) return neg_f32(static_cast<const uint32_t *>(src)[idx]);
    else if constexpr (DT == LB_F16) return neg_f16(static_cast<const uint16_t *>(src)[idx]);
    else if constexpr (DT == LB_BF16) return neg_bf16(static_cast<const uint16_t *>(src)[idx]);
    else return static_cast<const int8_t *>(src)[idx] < 0;
}

// Pack along the rows of the source (factor U): one warp per destination
// word; lane j tests column 32w + j; the ballot is the word.
template <int DT>
__global__ void pack_rows_kernel(const void *__restrict__ src, int64_t rows, int64_t cols,
                                 int64_t src_ld, uint32_t *__restrict__ dst, int64_t dst_ld)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t total = rows * dst_ld;
    for (int64_t item = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); item < total;
         item += warps) {
        const int64_t row = item / dst_ld, w = item - row * dst_ld;
        const int64_t col = w * 32 + lane;
        const bool neg = col < cols && is_negative<DT>(src, row * src_ld + col);
        const uint32_t word = __ballot_sync(0xffffffffu, neg);
        if (lane == 0) dst[row * dst_ld + w] = word;
    }
}

// Pack along the columns of the source (factor V -> V^T).  A block owns one
// destination word column w and 32 latent indices k0 .. k0+31: it reads the
// 32 x 32 tile V[32w .. 32w+31][k0 .. k0+31] with k innermost (coalesced),
// then thread k assembles its word from the 32 flags of column k.
template <int DT>
__global__ void pack_cols_kernel(const void *__restrict__ src, int64_t rows, int64_t cols,
                                 int64_t src_ld, uint32_t *__restrict__ dst, int64_t dst_ld)
{
    __shared__ uint8_t flag[32][33];
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    const int64_t w = blockIdx.x;
    const int64_t k = (int64_t)blockIdx.y * 32 + tx;
    for (int i = ty; i < 32; i += 8) {
        const int64_t row = w * 32 + i;
        flag[i][tx] = (row < rows && k < cols) ? (uint8_t)is_negative<DT>(src, row * src_ld + k) : 0;
    }
    __syncthreads();
    if (ty == 0 && k < cols) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) word |= (uint32_t)flag[i][tx] << i;
        dst[k * dst_ld + w] = word;
    }
}

template <int DT>
cudaError_t launch_pack(const void *src, lb_factor kind, int64_t rows, int64_t cols, int64_t src_ld,
                        uint32_t *dst, int64_t dst_ld, cudaStream_t stream)
{
    if (kind == LB_FACTOR_U) {
        const int64_t words = rows * dst_ld;
        const int threads = 256;
        int64_t blocks = (words + 7) / 8;
        if (blocks > 148 * 64) blocks = 148 * 64;
        pack_rows_kernel<DT><<<(unsigned)blocks, threads, 0, stream>>>(src, rows, cols, src_ld, dst, dst_ld);
    } else {
        dim3 grid((unsigned)dst_ld, (unsigned)((cols + 31) / 32));
        pack_cols_kernel<DT><<<grid, dim3(32, 8), 0, stream>>>(src, rows, cols, src_ld, dst, dst_ld);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t pack_signs_launch(const void *src, lb_dtype dtype, lb_factor kind, int64_t rows, int64_t cols,
                              int64_t src_ld, uint32_t *dst, int64_t dst_ld, cudaStream_t stream)
{
    switch (dtype) {
    case LB_F32: return launch_pack<LB_F32>(src, kind, rows, cols, src_ld, dst, dst_ld, stream);
    case LB_F16: return launch_pack<LB_F16>(src, kind, rows, cols, src_ld, dst, dst_ld, stream);
    case LB_BF16: return launch_pack<LB_BF16>(src, kind, rows, cols, src_ld, dst, dst_ld, stream);
    case LB_I8: return launch_pack<LB_I8>(src, kind, rows, cols, src_ld, dst, dst_ld, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace lb
