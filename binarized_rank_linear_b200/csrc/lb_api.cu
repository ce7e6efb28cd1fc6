// lb_api.cu - the C ABI (include/lb.h): argument checks, per-device set-up,
// dispatch by token count, and the device status word.
#include <array>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "lb.h"
#include "lb_internal.h"

// One status word per device (each device that loads the library has its own
// copy of this variable).  Kernels set it with atomicCAS(0 -> code).
__device__ int g_lb_status = 0;

namespace {

using lb::kMaxDevices;
constexpr int64_t kMaxDim = int64_t(1) << 20;     // n_in, n_out
constexpr int64_t kMaxRank = 32768;
constexpr int64_t kMaxTokens = int64_t(1) << 24;

std::mutex g_mutex;
std::atomic<int> g_prefill_pairs{1};  // lb_set_prefill_pairs
std::array<lb::DeviceInfo, kMaxDevices> g_dev;
std::array<bool, kMaxDevices> g_ready{};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_words(int64_t cols) { return (cols + 31) / 32; }

// Set-up for the current device, once: check it is an sm_100 part, read its
// SM count and shared-memory limit, resolve the status word's device address
// and raise the kernels' dynamic shared-memory limits.
lb_status device_info(lb::DeviceInfo *out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return LB_ERR_NOT_SUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_ready[dev]) {
        *out = g_dev[dev];
        return LB_OK;
    }
    int major = 0, minor = 0;
    lb::DeviceInfo info;
    info.device = dev;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&info.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return LB_ERR_NOT_SUPPORTED_DEVICE;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&info.status), g_lb_status) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    if (lb::decode_prepare_device(info) != cudaSuccess || lb::prefill_prepare_device(info) != cudaSuccess ||
        lb::wgrad_prepare_device(info) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    g_dev[dev] = info;
    g_ready[dev] = true;
    *out = info;
    return LB_OK;
}

// Checks one path against the layer's sizes; fills `d` on success.
lb_status check_path(const lb_path *p, int64_t n_in, int64_t n_out, lb::PathDesc *d)
{
    if (!p || !p->u_bits || !p->vt_bits || !p->h || !p->g || !p->l) return LB_ERR_INVALID_ARGUMENT;
    if (p->rank <= 0 || p->u_ld < 0 || p->vt_ld < 0) return LB_ERR_INVALID_ARGUMENT;
    if (p->rank % 32 != 0 || p->rank > kMaxRank) return LB_ERR_UNSUPPORTED_SHAPE;
    const int64_t u_ld = p->u_ld ? p->u_ld : ceil_words(p->rank);
    const int64_t vt_ld = p->vt_ld ? p->vt_ld : ceil_words(n_in);
    if (u_ld < ceil_words(p->rank) || vt_ld < ceil_words(n_in)) return LB_ERR_INVALID_ARGUMENT;
    if (!aligned16(p->u_bits) || !aligned16(p->vt_bits) || !aligned16(p->h) || !aligned16(p->g) ||
        !aligned16(p->l))
        return LB_ERR_MISALIGNED;
    (void)n_out;
    d->u_bits = p->u_bits;
    d->vt_bits = p->vt_bits;
    d->h = p->h;
    d->g = p->g;
    d->l = p->l;
    d->rank = (int)p->rank;
    d->u_ld = u_ld;
    d->vt_ld = vt_ld;
    return LB_OK;
}

// Checks the half of a path that one contraction alone uses: the V side
// (vt_bits, g, l against n_in) for the latent, the U side (u_bits, h) for the
// expansion; the other half is not read and may be null.
lb_status check_half(const lb_path *p, bool v_side, int64_t n_in, lb::PathDesc *d)
{
    if (!p) return LB_ERR_INVALID_ARGUMENT;
    if (p->rank <= 0 || p->u_ld < 0 || p->vt_ld < 0) return LB_ERR_INVALID_ARGUMENT;
    if (p->rank % 32 != 0 || p->rank > kMaxRank) return LB_ERR_UNSUPPORTED_SHAPE;
    *d = lb::PathDesc{};
    d->rank = (int)p->rank;
    if (v_side) {
        if (!p->vt_bits || !p->g || !p->l) return LB_ERR_INVALID_ARGUMENT;
        const int64_t vt_ld = p->vt_ld ? p->vt_ld : ceil_words(n_in);
        if (vt_ld < ceil_words(n_in)) return LB_ERR_INVALID_ARGUMENT;
        if (!aligned16(p->vt_bits) || !aligned16(p->g) || !aligned16(p->l)) return LB_ERR_MISALIGNED;
        d->vt_bits = p->vt_bits;
        d->g = p->g;
        d->l = p->l;
        d->vt_ld = vt_ld;
    } else {
        if (!p->u_bits || !p->h) return LB_ERR_INVALID_ARGUMENT;
        const int64_t u_ld = p->u_ld ? p->u_ld : ceil_words(p->rank);
        if (u_ld < ceil_words(p->rank)) return LB_ERR_INVALID_ARGUMENT;
        if (!aligned16(p->u_bits) || !aligned16(p->h)) return LB_ERR_MISALIGNED;
        d->u_bits = p->u_bits;
        d->h = p->h;
        d->u_ld = u_ld;
    }
    return LB_OK;
}

size_t workspace_for(int64_t tokens, int64_t n_in, int64_t n_out, const int *ranks, int npaths)
{
    if (tokens > lb::kMidMaxTokens) return lb::prefill_workspace_bytes((int)tokens, ranks, npaths);
    return lb::decode_workspace_bytes((int)tokens, (int)n_in, (int)n_out, ranks, npaths);
}

}  // namespace

bool lb::prefill_pairs_enabled() { return g_prefill_pairs.load(std::memory_order_relaxed) != 0; }

namespace {
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;
std::atomic<unsigned long long> g_debug_wait_ns{kDefaultWaitNs};  // lb_debug_inject_stall
std::atomic<int> g_debug_skip{0};
}  // namespace

unsigned long long lb::debug_wait_ns() { return g_debug_wait_ns.load(std::memory_order_relaxed); }
int lb::debug_skip_arrival() { return g_debug_skip.load(std::memory_order_relaxed); }

extern "C" {

const char *lb_status_string(lb_status s)
{
    switch (s) {
    case LB_OK: return "LB_OK";
    case LB_ERR_INVALID_ARGUMENT: return "LB_ERR_INVALID_ARGUMENT";
    case LB_ERR_UNSUPPORTED_SHAPE: return "LB_ERR_UNSUPPORTED_SHAPE";
    case LB_ERR_MISALIGNED: return "LB_ERR_MISALIGNED";
    case LB_ERR_CUDA: return "LB_ERR_CUDA";
    case LB_ERR_DEVICE_TIMEOUT: return "LB_ERR_DEVICE_TIMEOUT";
    case LB_ERR_NOT_SUPPORTED_DEVICE: return "LB_ERR_NOT_SUPPORTED_DEVICE";
    case LB_ERR_WORKSPACE_TOO_SMALL: return "LB_ERR_WORKSPACE_TOO_SMALL";
    case LB_ERR_RANGE: return "LB_ERR_RANGE";
    }
    return "LB_ERR_UNKNOWN";
}

int64_t lb_packed_ld_words(int64_t cols)
{
    return cols <= 0 ? -1 : ceil_words(cols);
}

size_t lb_packed_bytes(lb_factor kind, int64_t n_in_or_out, int64_t rank)
{
    if (n_in_or_out <= 0 || rank <= 0 || n_in_or_out > kMaxDim * 64 || rank > kMaxDim * 64) return 0;
    if (kind == LB_FACTOR_U) return (size_t)n_in_or_out * (size_t)ceil_words(rank) * 4u;
    if (kind == LB_FACTOR_V) return (size_t)rank * (size_t)ceil_words(n_in_or_out) * 4u;
    return 0;
}

lb_status lb_rank_for_budget(int64_t n_in, int64_t n_out, int64_t eff_num, int64_t eff_den, int paths,
                             int align, int64_t *rank)
{
    if (!rank) return LB_ERR_INVALID_ARGUMENT;
    *rank = 0;
    if (n_in <= 0 || n_out <= 0 || eff_num <= 0 || eff_den <= 0 || (paths != 1 && paths != 2) || align < 1)
        return LB_ERR_INVALID_ARGUMENT;
    // numerator eff_num * n_in * n_out and denominator eff_den * paths * (n_in + n_out)
    // in unsigned 128-bit arithmetic: no overflow for any int64 inputs.
    const unsigned __int128 num = (unsigned __int128)eff_num * (unsigned __int128)n_in * (unsigned __int128)n_out;
    const unsigned __int128 den =
        (unsigned __int128)eff_den * (unsigned __int128)paths * ((unsigned __int128)n_in + (unsigned __int128)n_out);
    unsigned __int128 r = num / den;
    r -= r % (unsigned __int128)align;
    if (r > (unsigned __int128)INT64_MAX) return LB_ERR_INVALID_ARGUMENT;
    *rank = (int64_t)r;
    return r == 0 ? LB_ERR_UNSUPPORTED_SHAPE : LB_OK;
}

lb_status lb_pack_signs(const void *src, lb_dtype dtype, lb_factor kind, int64_t rows, int64_t cols,
                        int64_t src_ld, uint32_t *dst, int64_t dst_ld_words, void *stream)
{
    if (!src || !dst) return LB_ERR_INVALID_ARGUMENT;
    if (dtype != LB_F32 && dtype != LB_F16 && dtype != LB_BF16 && dtype != LB_I8) return LB_ERR_INVALID_ARGUMENT;
    if (kind != LB_FACTOR_U && kind != LB_FACTOR_V) return LB_ERR_INVALID_ARGUMENT;
    if (rows <= 0 || cols <= 0 || src_ld < cols) return LB_ERR_INVALID_ARGUMENT;
    if (rows > kMaxDim * 64 || cols > kMaxDim * 64) return LB_ERR_UNSUPPORTED_SHAPE;
    const int64_t packed_cols = kind == LB_FACTOR_U ? cols : rows;
    if (dst_ld_words < ceil_words(packed_cols)) return LB_ERR_INVALID_ARGUMENT;
    const size_t esize = dtype == LB_F32 ? 4 : (dtype == LB_I8 ? 1 : 2);
    if ((reinterpret_cast<uintptr_t>(src) % esize) != 0 || (reinterpret_cast<uintptr_t>(dst) & 3u) != 0)
        return LB_ERR_MISALIGNED;
    lb::DeviceInfo dev;
    const lb_status st = device_info(&dev);
    if (st != LB_OK) return st;
    const cudaError_t e = lb::pack_signs_launch(src, dtype, kind, rows, cols, src_ld, dst, dst_ld_words,
                                                static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    return LB_OK;
}

size_t lb_forward_workspace_bytes(int64_t tokens, int64_t n_in, int64_t n_out, int64_t rank_main,
                                  int64_t rank_residual)
{
    if (tokens < 0 || n_in <= 0 || n_out <= 0 || rank_main <= 0 || rank_residual < 0) return 0;
    if (tokens > kMaxTokens || n_in > kMaxDim || n_out > kMaxDim || rank_main > kMaxRank ||
        rank_residual > kMaxRank)
        return 0;
    if (tokens == 0) return 0;
    const int ranks[2] = {(int)rank_main, (int)rank_residual};
    return workspace_for(tokens, n_in, n_out, ranks, rank_residual > 0 ? 2 : 1);
}

// Every host-side check of lb_linear_forward (tokens > 0).
// Every host-side check of a forward call (sizes, pointers, alignment,
// workspace); on success fills `a`.  Launches nothing.
static lb_status make_forward(const uint16_t *x, int64_t tokens, int64_t n_in, int64_t n_out, int64_t ldx,
                              const lb_path *main, const lb_path *residual, uint16_t *y, int64_t ldy,
                              void *workspace, size_t workspace_bytes, lb::ForwardArgs *a)
{
    if (!x || !y || !main) return LB_ERR_INVALID_ARGUMENT;
    if (ldx < n_in || ldy < n_out) return LB_ERR_INVALID_ARGUMENT;
    if (n_in % 32 != 0 || n_out % 32 != 0 || n_in > kMaxDim || n_out > kMaxDim || tokens > kMaxTokens)
        return LB_ERR_UNSUPPORTED_SHAPE;
    if (ldx % 8 != 0 || ldy % 8 != 0 || !aligned16(x) || !aligned16(y)) return LB_ERR_MISALIGNED;
    *a = lb::ForwardArgs{};
    a->npaths = residual ? 2 : 1;
    lb_status st = check_path(main, n_in, n_out, &a->path[0]);
    if (st == LB_OK && residual) st = check_path(residual, n_in, n_out, &a->path[1]);
    if (st != LB_OK) return st;
    const int ranks[2] = {a->path[0].rank, a->npaths > 1 ? a->path[1].rank : 0};
    const size_t need = workspace_for(tokens, n_in, n_out, ranks, a->npaths);
    if (need > 0 && !workspace) return LB_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < need) return LB_ERR_WORKSPACE_TOO_SMALL;
    if (workspace && !aligned16(workspace)) return LB_ERR_MISALIGNED;
    a->x = x;
    a->ldx = ldx;
    a->tokens = (int)tokens;
    a->n_in = (int)n_in;
    a->n_out = (int)n_out;
    a->y = y;
    a->ldy = ldy;
    a->workspace = workspace;
    a->workspace_bytes = workspace_bytes;
    return LB_OK;
}

static lb_status run_forward(const lb::ForwardArgs &a, const lb::DeviceInfo &dev, void *stream)
{
    const cudaError_t e = a.tokens > lb::kMidMaxTokens ? lb::prefill_forward(a, dev, static_cast<cudaStream_t>(stream))
                                                       : lb::decode_forward(a, dev, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    return LB_OK;
}

lb_status lb_linear_forward(const uint16_t *x, int64_t tokens, int64_t n_in, int64_t n_out, int64_t ldx,
                            const lb_path *main, const lb_path *residual, uint16_t *y, int64_t ldy,
                            void *workspace, size_t workspace_bytes, void *stream)
{
    if (tokens < 0 || n_in <= 0 || n_out <= 0) return LB_ERR_INVALID_ARGUMENT;
    if (tokens == 0) return LB_OK;
    lb::ForwardArgs a;
    lb_status st = make_forward(x, tokens, n_in, n_out, ldx, main, residual, y, ldy, workspace, workspace_bytes, &a);
    if (st != LB_OK) return st;
    lb::DeviceInfo dev;
    st = device_info(&dev);
    if (st != LB_OK) return st;
    return run_forward(a, dev, stream);
}

// Fills g from the caller's projections; checks everything a siblings call
// checks on the host (sizes, pointers, alignment), not the workspace.
static lb_status build_group(const uint16_t *x, int64_t tokens, int64_t n_in, int64_t ldx, int nproj,
                             const lb_projection *proj, bool sizes_only, lb::GroupArgs *g)
{
    if (tokens < 0 || n_in <= 0 || nproj < 1 || nproj > LB_MAX_SIBLINGS || !proj) return LB_ERR_INVALID_ARGUMENT;
    if (n_in % 32 != 0 || n_in > kMaxDim || tokens > kMaxTokens) return LB_ERR_UNSUPPORTED_SHAPE;
    if (!sizes_only) {
        if (!x || ldx < n_in) return LB_ERR_INVALID_ARGUMENT;
        if (ldx % 8 != 0 || !aligned16(x)) return LB_ERR_MISALIGNED;
    }
    *g = lb::GroupArgs{};
    g->x = x;
    g->ldx = ldx;
    g->tokens = (int)tokens;
    g->n_in = (int)n_in;
    g->nproj = nproj;
    for (int j = 0; j < nproj; ++j) {
        const lb_projection &pj = proj[j];
        lb::ProjDesc &d = g->proj[j];
        if (pj.n_out <= 0 || !pj.main) return LB_ERR_INVALID_ARGUMENT;
        if (pj.n_out % 32 != 0 || pj.n_out > kMaxDim) return LB_ERR_UNSUPPORTED_SHAPE;
        d.n_out = (int)pj.n_out;
        d.npaths = pj.residual ? 2 : 1;
        if (sizes_only) {
            const lb_path *ps[2] = {pj.main, pj.residual};
            for (int q = 0; q < d.npaths; ++q) {
                if (ps[q]->rank <= 0) return LB_ERR_INVALID_ARGUMENT;
                if (ps[q]->rank % 32 != 0 || ps[q]->rank > kMaxRank) return LB_ERR_UNSUPPORTED_SHAPE;
                d.path[q].rank = (int)ps[q]->rank;
            }
            continue;
        }
        if (!pj.y || pj.ldy < pj.n_out) return LB_ERR_INVALID_ARGUMENT;
        if (pj.ldy % 8 != 0 || !aligned16(pj.y)) return LB_ERR_MISALIGNED;
        lb_status st = check_path(pj.main, n_in, pj.n_out, &d.path[0]);
        if (st == LB_OK && pj.residual) st = check_path(pj.residual, n_in, pj.n_out, &d.path[1]);
        if (st != LB_OK) return st;
        d.y = pj.y;
        d.ldy = pj.ldy;
    }
    return LB_OK;
}

size_t lb_siblings_workspace_bytes(int64_t tokens, int64_t n_in, int nproj, const lb_projection *proj)
{
    lb::GroupArgs g;
    if (build_group(nullptr, tokens, n_in, n_in, nproj, proj, true, &g) != LB_OK || tokens == 0) return 0;
    return lb::group_workspace_bytes(g);
}

lb_status lb_linear_forward_siblings(const uint16_t *x, int64_t tokens, int64_t n_in, int64_t ldx, int nproj,
                                     const lb_projection *proj, void *workspace, size_t workspace_bytes,
                                     void *stream)
{
    if (tokens < 0 || n_in <= 0 || nproj < 1 || nproj > LB_MAX_SIBLINGS || !proj) return LB_ERR_INVALID_ARGUMENT;
    if (tokens == 0) return LB_OK;
    lb::GroupArgs g;
    lb_status st = build_group(x, tokens, n_in, ldx, nproj, proj, false, &g);
    if (st != LB_OK) return st;
    const size_t need = lb::group_workspace_bytes(g);
    if (need > 0 && !workspace) return LB_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < need) return LB_ERR_WORKSPACE_TOO_SMALL;
    if (workspace && !aligned16(workspace)) return LB_ERR_MISALIGNED;
    g.workspace = workspace;
    g.workspace_bytes = workspace_bytes;
    lb::DeviceInfo dev;
    st = device_info(&dev);
    if (st != LB_OK) return st;
    if (lb::group_forward(g, dev, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    return LB_OK;
}

// The device's view of host memory: the address under which kernels reach
// `p` when it lies in pinned host memory mapped into the device's address
// space (as page-locked allocations are with unified addressing); null
// otherwise (pageable memory, device memory, an unknown pointer).
static void *device_view(const void *p)
{
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

lb_status lb_linear_forward_host(const uint16_t *x_host, int64_t tokens, int64_t n_in, int64_t n_out,
                                 const lb_path *main, const lb_path *residual, uint16_t *y_host, uint16_t *x_dev,
                                 uint16_t *y_dev, void *workspace, size_t workspace_bytes, void *stream)
{
    if (tokens < 0 || n_in <= 0 || n_out <= 0) return LB_ERR_INVALID_ARGUMENT;
    if (tokens == 0) return LB_OK;
    if (!x_host || !y_host) return LB_ERR_INVALID_ARGUMENT;
    // every check on the device side first: nothing moves when the call is refused
    lb::ForwardArgs a;
    lb_status st = make_forward(x_dev, tokens, n_in, n_out, n_in, main, residual, y_dev, n_out, workspace,
                                workspace_bytes, &a);
    if (st != LB_OK) return st;
    lb::DeviceInfo dev;
    st = device_info(&dev);
    if (st != LB_OK) return st;
    // Up to 128 tokens (the decode kernels, whose last kernel stores y with
    // plain coalesced stores), with both host buffers pinned and mapped: x
    // reaches x_dev through one gather kernel (a single round trip over the
    // host link, chained into the forward kernels, where a DMA copy and the
    // switch from copy engine to kernels cost several times that), and the
    // last kernel writes y straight into y_host
    if (tokens <= lb::kMidMaxTokens) {
        const void *xd = device_view(x_host);
        void *yd = device_view(y_host);
        if (xd && yd && aligned16(xd) && aligned16(yd)) {
            lb::ForwardArgs h = a;
            h.y = static_cast<uint16_t *>(yd);
            if (lb::host_gather_launch(xd, x_dev, (size_t)tokens * (size_t)n_in * 2,
                                       static_cast<cudaStream_t>(stream)) != cudaSuccess) {
                cudaGetLastError();
                return LB_ERR_CUDA;
            }
            return run_forward(h, dev, stream);
        }
    }
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(x_dev, x_host, (size_t)tokens * (size_t)n_in * 2, cudaMemcpyHostToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    st = run_forward(a, dev, stream);
    if (st != LB_OK) return st;
    if (cudaMemcpyAsync(y_host, y_dev, (size_t)tokens * (size_t)n_out * 2, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    return LB_OK;
}

lb_status lb_latent_forward(const uint16_t *x, int64_t tokens, int64_t n_in, int64_t ldx, const lb_path *main,
                            const lb_path *residual, uint16_t *z, int64_t ldz, void *stream)
{
    if (tokens < 0 || n_in <= 0) return LB_ERR_INVALID_ARGUMENT;
    if (tokens == 0) return LB_OK;
    if (!x || !z || !main) return LB_ERR_INVALID_ARGUMENT;
    if (ldx < n_in) return LB_ERR_INVALID_ARGUMENT;
    if (n_in % 32 != 0 || n_in > kMaxDim || tokens > kMaxTokens) return LB_ERR_UNSUPPORTED_SHAPE;
    lb::ForwardArgs a{};
    a.npaths = residual ? 2 : 1;
    lb_status st = check_half(main, true, n_in, &a.path[0]);
    if (st == LB_OK && residual) st = check_half(residual, true, n_in, &a.path[1]);
    if (st != LB_OK) return st;
    const int64_t R = a.path[0].rank + (a.npaths > 1 ? a.path[1].rank : 0);
    if (ldz < R) return LB_ERR_INVALID_ARGUMENT;
    if (ldx % 8 != 0 || ldz % 8 != 0 || !aligned16(x) || !aligned16(z)) return LB_ERR_MISALIGNED;
    a.x = x;
    a.ldx = ldx;
    a.tokens = (int)tokens;
    a.n_in = (int)n_in;
    lb::DeviceInfo dev;
    st = device_info(&dev);
    if (st != LB_OK) return st;
    if (lb::latent_launch(a, dev, static_cast<cudaStream_t>(stream), z, ldz) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    return LB_OK;
}

lb_status lb_expand_forward(const uint16_t *z, int64_t tokens, int64_t n_out, int64_t ldz, const lb_path *main,
                            const lb_path *residual, uint16_t *y, int64_t ldy, void *stream)
{
    if (tokens < 0 || n_out <= 0) return LB_ERR_INVALID_ARGUMENT;
    if (tokens == 0) return LB_OK;
    if (!z || !y || !main) return LB_ERR_INVALID_ARGUMENT;
    if (ldy < n_out) return LB_ERR_INVALID_ARGUMENT;
    if (n_out % 32 != 0 || n_out > kMaxDim || tokens > kMaxTokens) return LB_ERR_UNSUPPORTED_SHAPE;
    lb::ForwardArgs a{};
    a.npaths = residual ? 2 : 1;
    lb_status st = check_half(main, false, 0, &a.path[0]);
    if (st == LB_OK && residual) st = check_half(residual, false, 0, &a.path[1]);
    if (st != LB_OK) return st;
    const int64_t R = a.path[0].rank + (a.npaths > 1 ? a.path[1].rank : 0);
    if (ldz < R) return LB_ERR_INVALID_ARGUMENT;
    if (ldz % 8 != 0 || ldy % 8 != 0 || !aligned16(z) || !aligned16(y)) return LB_ERR_MISALIGNED;
    a.tokens = (int)tokens;
    a.n_out = (int)n_out;
    a.y = y;
    a.ldy = ldy;
    lb::DeviceInfo dev;
    st = device_info(&dev);
    if (st != LB_OK) return st;
    if (lb::expand_launch(a, dev, static_cast<cudaStream_t>(stream), z, ldz) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    return LB_OK;
}

size_t lb_backward_workspace_bytes(int64_t tokens, int64_t n_in, int64_t n_out, int64_t rank_main,
                                   int64_t rank_residual)
{
    if (tokens < 0 || n_in <= 0 || n_out <= 0 || rank_main <= 0 || rank_residual < 0) return 0;
    if (tokens > kMaxTokens || n_in > kMaxDim || n_out > kMaxDim || rank_main > kMaxRank || rank_residual > kMaxRank)
        return 0;
    if (tokens == 0 || n_in % 32 != 0 || n_out % 32 != 0 || rank_main % 32 != 0 || rank_residual % 32 != 0) return 0;
    const int ranks[2] = {(int)rank_main, (int)rank_residual};
    return lb::backward_workspace_bytes((int)tokens, (int)n_in, (int)n_out, ranks, rank_residual > 0 ? 2 : 1);
}

lb_status lb_linear_backward(const uint16_t *x, const uint16_t *dy, int64_t tokens, int64_t n_in, int64_t n_out,
                             int64_t ldx, int64_t lddy, const lb_path *main, const lb_path *residual, uint16_t *dx,
                             int64_t lddx, float *dh, float *dg, float *dl, void *workspace, size_t workspace_bytes,
                             void *stream)
{
    if (tokens < 0 || n_in <= 0 || n_out <= 0) return LB_ERR_INVALID_ARGUMENT;
    if (!main || !dh || !dg || !dl) return LB_ERR_INVALID_ARGUMENT;
    if (tokens > 0 && (!x || !dy)) return LB_ERR_INVALID_ARGUMENT;  // no tokens: x and dy are not read
    if (ldx < n_in || lddy < n_out || (dx && lddx < n_in)) return LB_ERR_INVALID_ARGUMENT;
    if (n_in % 32 != 0 || n_out % 32 != 0 || n_in > kMaxDim || n_out > kMaxDim || tokens > kMaxTokens)
        return LB_ERR_UNSUPPORTED_SHAPE;
    if (ldx % 8 != 0 || lddy % 8 != 0 || !aligned16(x) || !aligned16(dy)) return LB_ERR_MISALIGNED;  // null is aligned
    if (dx && (lddx % 8 != 0 || !aligned16(dx))) return LB_ERR_MISALIGNED;
    if ((reinterpret_cast<uintptr_t>(dh) | reinterpret_cast<uintptr_t>(dg) | reinterpret_cast<uintptr_t>(dl)) & 3u)
        return LB_ERR_MISALIGNED;
    lb::BackwardArgs b{};
    b.npaths = residual ? 2 : 1;
    lb_status st = check_path(main, n_in, n_out, &b.path[0]);
    if (st == LB_OK && residual) st = check_path(residual, n_in, n_out, &b.path[1]);
    if (st != LB_OK) return st;
    const int ranks[2] = {b.path[0].rank, b.npaths > 1 ? b.path[1].rank : 0};
    const size_t need = tokens > 0 ? lb::backward_workspace_bytes((int)tokens, (int)n_in, (int)n_out, ranks, b.npaths) : 0;
    if (need > 0 && !workspace) return LB_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < need) return LB_ERR_WORKSPACE_TOO_SMALL;
    if (workspace && !aligned16(workspace)) return LB_ERR_MISALIGNED;
    lb::DeviceInfo dev;
    st = device_info(&dev);
    if (st != LB_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tokens == 0) {
        // no tokens: every scale gradient is an empty sum
        const int R = ranks[0] + ranks[1];
        if (cudaMemsetAsync(dh, 0, sizeof(float) * (size_t)b.npaths * (size_t)n_out, s) != cudaSuccess ||
            cudaMemsetAsync(dg, 0, sizeof(float) * (size_t)b.npaths * (size_t)n_in, s) != cudaSuccess ||
            cudaMemsetAsync(dl, 0, sizeof(float) * (size_t)R, s) != cudaSuccess) {
            cudaGetLastError();
            return LB_ERR_CUDA;
        }
        return LB_OK;
    }
    b.x = x;
    b.ldx = ldx;
    b.dy = dy;
    b.lddy = lddy;
    b.tokens = (int)tokens;
    b.n_in = (int)n_in;
    b.n_out = (int)n_out;
    b.dx = dx;
    b.lddx = lddx;
    b.dh = dh;
    b.dg = dg;
    b.dl = dl;
    b.workspace = workspace;
    b.workspace_bytes = workspace_bytes;
    if (lb::backward_launch(b, dev, s) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    return LB_OK;
}

lb_status lb_device_status(void *stream, lb_status *out)
{
    if (!out) return LB_ERR_INVALID_ARGUMENT;
    *out = LB_OK;
    lb::DeviceInfo dev;
    const lb_status st = device_info(&dev);
    if (st != LB_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_lb_status, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return LB_ERR_CUDA;
    }
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_lb_status, &zero, sizeof(int)) != cudaSuccess) {
            cudaGetLastError();
            return LB_ERR_CUDA;
        }
    }
    *out = static_cast<lb_status>(v);
    return LB_OK;
}

lb_status lb_debug_inject_stall(int enable, uint64_t wait_limit_ns)
{
    if (enable != 0 && enable != 1) return LB_ERR_INVALID_ARGUMENT;
    if (enable && (wait_limit_ns < 1000ull || wait_limit_ns > kDefaultWaitNs)) return LB_ERR_INVALID_ARGUMENT;
    g_debug_wait_ns.store(enable ? wait_limit_ns : kDefaultWaitNs, std::memory_order_relaxed);
    g_debug_skip.store(enable, std::memory_order_relaxed);
    return LB_OK;
}

lb_status lb_set_prefill_pairs(int enable)
{
    if (enable != 0 && enable != 1) return LB_ERR_INVALID_ARGUMENT;
    g_prefill_pairs.store(enable, std::memory_order_relaxed);
    return LB_OK;
}

}  // extern "C"
