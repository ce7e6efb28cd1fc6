// lb_host_io.cu - moving a call's activations between host and device memory
// inside the forward chain, for the host-buffer entry point.
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"

namespace lb {
namespace {

constexpr int kGatherThreads = 256;

// dst[i] = src[i] for i < n16 (16-byte units).  src is pinned host memory
// reached through its device mapping.  The next kernel is released at entry,
// so its weight loads overlap this copy (it waits for the copy before it
// reads dst).  Both the load and the store come after the dependency wait:
// the previous kernel on the stream may still write src (a chain of host
// calls in which one call's y_host is the next call's x_host: the last
// kernel of a call stores y after releasing its dependents) or read dst (the
// previous call's first kernel reads x_dev).
__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                                int64_t n16)
{
    pdl_launch_dependents();
    const int64_t i = (int64_t)blockIdx.x * kGatherThreads + threadIdx.x;
    pdl_wait();
    if (i < n16) dst[i] = src[i];
}

}  // namespace

cudaError_t host_gather_launch(const void *src, void *dst, size_t bytes, cudaStream_t stream)
{
    const int64_t n16 = (int64_t)(bytes / 16);
    if (n16 == 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)((n16 + kGatherThreads - 1) / kGatherThreads));
    cfg.blockDim = dim3(kGatherThreads);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gather_kernel, static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), n16);
}

}  // namespace lb
