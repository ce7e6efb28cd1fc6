// lb_decode.cu - the forward pass for 1..128 tokens: dispatch between the
// CUDA-core path (1..4 tokens, lb_gemv.cu) and the tcgen05 path (5..128
// tokens, lb_mid.cu).  Also the dispatch of either contraction on its own
// (the split latent entry points) and of sibling projections that share x.
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

GroupArgs group_of_one(const ForwardArgs &a)
{
    GroupArgs g{};
    g.x = a.x;
    g.ldx = a.ldx;
    g.tokens = a.tokens;
    g.n_in = a.n_in;
    g.nproj = 1;
    g.proj[0].n_out = a.n_out;
    g.proj[0].npaths = a.npaths;
    g.proj[0].path[0] = a.path[0];
    g.proj[0].path[1] = a.path[1];
    g.proj[0].y = a.y;
    g.proj[0].ldy = a.ldy;
    g.workspace = a.workspace;
    g.workspace_bytes = a.workspace_bytes;
    return g;
}

ForwardArgs layer_of(const GroupArgs &g, int j)
{
    ForwardArgs a{};
    a.x = g.x;
    a.ldx = g.ldx;
    a.tokens = g.tokens;
    a.n_in = g.n_in;
    a.n_out = g.proj[j].n_out;
    a.npaths = g.proj[j].npaths;
    a.path[0] = g.proj[j].path[0];
    a.path[1] = g.proj[j].path[1];
    a.y = g.proj[j].y;
    a.ldy = g.proj[j].ldy;
    a.workspace = g.workspace;
    a.workspace_bytes = g.workspace_bytes;
    return a;
}

namespace {

// A group of one layer with only the sizes filled in (enough for workspace sizes).
GroupArgs sizes_only(int tokens, int n_in, int n_out, const int *ranks, int npaths)
{
    ForwardArgs a{};
    a.tokens = tokens;
    a.n_in = n_in;
    a.n_out = n_out;
    a.npaths = npaths;
    a.path[0].rank = ranks[0];
    a.path[1].rank = npaths > 1 ? ranks[1] : 0;
    return group_of_one(a);
}

// 1-4 tokens go to the CUDA-core kernels when they fit, except 3-4 tokens on
// wide layers: their tables and lookups grow with the tokens while the
// tcgen05 kernels cost about the same at 1-16 tokens (B200, Llama-2-7B
// gate/up: 6.9, 9.6, 14.9, 19.4 us at 1-4 tokens against 15.2 on tcgen05;
// q_proj 12.3 against 14.8 at 4 tokens).  The switch is at tokens x sign
// bits (sum of r (n_in + n_out) over the group's paths) above 80 M.
bool small_preferred(int M, const GroupArgs &g, const DeviceInfo &dev)
{
    if (M > kSmallMaxTokens || !small_fits(M, g, dev)) return false;
    if (M <= 2) return true;
    int64_t bits = 0;
    for (int j = 0; j < g.nproj; ++j)
        for (int q = 0; q < g.proj[j].npaths; ++q)
            bits += (int64_t)g.proj[j].path[q].rank * (g.n_in + g.proj[j].n_out);
    return (int64_t)M * bits <= 80000000;
}

size_t layer_workspace_bytes(const ForwardArgs &a)
{
    const int ranks[2] = {a.path[0].rank, a.npaths > 1 ? a.path[1].rank : 0};
    return a.tokens > kMidMaxTokens ? prefill_workspace_bytes(a.tokens, ranks, a.npaths)
                                    : decode_workspace_bytes(a.tokens, a.n_in, a.n_out, ranks, a.npaths);
}

}  // namespace

size_t decode_workspace_bytes(int tokens, int n_in, int n_out, const int *ranks, int npaths)
{
    const int M = std::min(tokens, kMidMaxTokens);
    return std::max(mid_workspace_bytes(M, ranks, npaths),
                    small_workspace_bytes(std::min(M, kSmallMaxTokens), sizes_only(M, n_in, n_out, ranks, npaths)));
}

cudaError_t decode_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    const GroupArgs g = group_of_one(a);
    for (int m0 = 0; m0 < a.tokens; m0 += kMidMaxTokens) {
        const int M = std::min(kMidMaxTokens, a.tokens - m0);
        const cudaError_t e = small_preferred(M, g, dev) ? small_forward(g, dev, stream, m0, M)
                                                                             : mid_forward(a, dev, stream, m0, M);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

size_t group_workspace_bytes(const GroupArgs &g)
{
    // enough for whichever path the call takes, and for each layer alone
    size_t need = g.tokens <= kSmallMaxTokens ? small_workspace_bytes(g.tokens, g) : 0;
    if (g.tokens <= kMidMaxTokens) need = std::max(need, mid_group_workspace_bytes(g.tokens, g));
    for (int j = 0; j < g.nproj; ++j) need = std::max(need, layer_workspace_bytes(layer_of(g, j)));
    return need;
}

cudaError_t group_forward(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream)
{
    if (small_preferred(g.tokens, g, dev)) return small_forward(g, dev, stream, 0, g.tokens);
    if (g.tokens <= kMidMaxTokens) return mid_group_forward(g, dev, stream, 0, g.tokens);
    for (int j = 0; j < g.nproj; ++j) {
        const cudaError_t e = prefill_forward(layer_of(g, j), dev, stream);
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
