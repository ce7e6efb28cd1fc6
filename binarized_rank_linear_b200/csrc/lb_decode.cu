// lb_decode.cu - the forward pass for 1..128 tokens: dispatch between the
// CUDA-core path (1..4 tokens, lb_gemv.cu) and the tcgen05 path (5..128
// tokens, lb_mid.cu).  Also the dispatch of either contraction on
// its own (the split latent entry points).
//
// The layer (sesamedisk.com, "Samsung LittleBit 13B Model", section "What the
// method actually computes", Proposition 1) is computed by a pair of
// launches per slice, contraction 1 then contraction 2, chained with
// programmatic dependent launch; both paths of residual compensation run in
// the same pair.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_internal.h"

namespace lb {

cudaError_t decode_prepare_device(const DeviceInfo &dev)
{
    cudaError_t e = small_prepare_device(dev);
    if (e == cudaSuccess) e = mid_prepare_device(dev);
    return e;
}

size_t decode_workspace_bytes(int tokens, int n_in, int n_out, const int *ranks, int npaths)
{
    (void)n_in;
    (void)n_out;
    const int M = std::min(tokens, kMidMaxTokens);
    return std::max(mid_workspace_bytes(M, ranks, npaths),
                    small_workspace_bytes(std::min(M, kSmallMaxTokens), ranks, npaths));
}

cudaError_t decode_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    const int ranks[2] = {a.path[0].rank, a.npaths > 1 ? a.path[1].rank : 0};
    for (int m0 = 0; m0 < a.tokens; m0 += kMidMaxTokens) {
        const int M = std::min(kMidMaxTokens, a.tokens - m0);
        const cudaError_t e = M <= kSmallMaxTokens && small_fits(M, a.n_in, a.n_out, ranks, a.npaths, dev)
                                  ? small_forward(a, dev, stream, m0, M)
                                  : mid_forward(a, dev, stream, m0, M);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t latent_launch(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, uint16_t *z, int64_t ldz)
{
    return a.tokens > kMidMaxTokens ? prefill_latent(a, dev, stream, z, ldz)
                                       : mid_latent(a, dev, stream, 0, a.tokens, z, ldz);
}

cudaError_t expand_launch(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, const uint16_t *z,
                          int64_t ldz)
{
    return a.tokens > kMidMaxTokens ? prefill_expand(a, dev, stream, z, ldz)
                                       : mid_expand(a, dev, stream, 0, a.tokens, z, ldz);
}

}  // namespace lb
