// lb_fixed_scratch.cu - lb_linear_forward_fixed_scratch: the decode forward
// pass (1..32 tokens) with its scratch in a fixed device array that the
// library owns, instead of a workspace passed in by the caller.
//
// Who needs it: callers that cannot hand the library device memory at call
// time.  For example, a plain C host program with no device allocator of its
// own; a runtime whose device memory is reserved once, up front, under a fixed
// budget; or a latency-critical loop where allocation (and the implicit
// device synchronisation of cudaMalloc/cudaFree) is not allowed.  This file
// allocates nothing either: no cudaMalloc, no cudaFree, no allocating library
// routine.  The array below is part of the library's device image, created
// when the module is loaded on a device.
//
// The decode path is the only one served: its scratch (the latent between
// the two contractions) is at most a few hundred KB at the sizes in use; the
// prefill path needs tokens x rank x 2 bytes, far beyond a fixed array.
#include <mutex>

#include <cuda_runtime.h>

#include "lb.h"
#include "lb_internal.h"

namespace {

// One copy per device.  Nothing in it has to start at zero: every byte a call
// reads, the same call wrote earlier (the first contraction writes the latent
// that the second reads).
static __device__ __align__(256) unsigned char g_fixed_scratch[LB_FIXED_SCRATCH_BYTES];

using lb::kMaxDevices;
std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices];  // device address of g_fixed_scratch, per device; set once

// Device address of this device's array, looked up on the first call made
// with the device current and cached after that.  The stream must belong to
// the current device (the legacy default stream, NULL, always does): the
// kernels run on the stream's device, and the address is this device's.
lb_status scratch_address(cudaStream_t stream, void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return LB_ERR_CUDA;
    }
    if (stream) {
        int sdev = -1;
        if (cudaStreamGetDevice(stream, &sdev) != cudaSuccess) {
            (void)cudaGetLastError();
            return LB_ERR_INVALID_ARGUMENT;
        }
        if (sdev != dev) return LB_ERR_INVALID_ARGUMENT;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_fixed_scratch);
        if (e != cudaSuccess || !p) {
            (void)cudaGetLastError();  // do not leave the error for the caller's next call
            return LB_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return LB_OK;
}

}  // namespace

extern "C" lb_status lb_linear_forward_fixed_scratch(const uint16_t *x, int64_t tokens, int64_t n_in,
                                                     int64_t n_out, int64_t ldx, const lb_path *main,
                                                     const lb_path *residual, uint16_t *y, int64_t ldy,
                                                     void *stream)
{
    if (tokens < 0) return LB_ERR_INVALID_ARGUMENT;
    if (tokens == 0) return LB_OK;
    if (tokens > lb::kDecodeMaxTokens) return LB_ERR_UNSUPPORTED_SHAPE;
    if (!x || !y || !main) return LB_ERR_INVALID_ARGUMENT;
    const size_t need = lb_forward_workspace_bytes(tokens, n_in, n_out, main->rank, residual ? residual->rank : 0);
    if (need > LB_FIXED_SCRATCH_BYTES) return LB_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    const lb_status st = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (st != LB_OK) return st;
    // Everything else (shapes, strides, alignment, the paths) is checked by
    // lb_linear_forward before it launches anything.
    return lb_linear_forward(x, tokens, n_in, n_out, ldx, main, residual, y, ldy, scratch,
                             LB_FIXED_SCRATCH_BYTES, stream);
}
