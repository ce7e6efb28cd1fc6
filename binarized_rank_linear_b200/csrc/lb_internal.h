// lb_internal.h - host-side interfaces between the C ABI (lb_api.cu) and the
// kernel translation units.  Not installed; not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "lb.h"

namespace lb {

// Devices the library serves per process: ordinals 0 .. kMaxDevices - 1 (its
// per-device tables have this many entries).
constexpr int kMaxDevices = 64;

// Per-device facts the launchers need (cached by lb_api.cu).
struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int max_smem_optin = 0;  // bytes of dynamic shared memory a block may opt into
    int *status = nullptr;   // device address of this device's status word
    int pair_slots = 0;      // CTA pairs of the prefill pair kernels resident at once
};

// ----------------------------------------------------------------- packing
cudaError_t pack_signs_launch(const void *src, lb_dtype dtype, lb_factor kind, int64_t rows, int64_t cols,
                              int64_t src_ld, uint32_t *dst, int64_t dst_ld, cudaStream_t stream);

// ----------------------------------------------------------------- forward
// Up to two paths, already validated, with their strides resolved.
struct PathDesc {
    const uint32_t *u_bits;
    const uint32_t *vt_bits;
    const uint16_t *h, *g, *l;
    int rank;
    int64_t u_ld, vt_ld;
};

struct ForwardArgs {
    const uint16_t *x;
    int64_t ldx;
    int tokens;
    int n_in, n_out;
    int npaths;
    PathDesc path[2];
    uint16_t *y;
    int64_t ldy;
    void *workspace;
    size_t workspace_bytes;
};

// Sibling projections: layers that share x (lb_linear_forward_siblings),
// each with its own paths, output width and output buffer.
constexpr int kMaxSiblings = LB_MAX_SIBLINGS;
struct ProjDesc {
    int n_out;
    int npaths;
    PathDesc path[2];
    uint16_t *y;
    int64_t ldy;
};
struct GroupArgs {
    const uint16_t *x;
    int64_t ldx;
    int tokens;
    int n_in;
    int nproj;
    ProjDesc proj[kMaxSiblings];
    void *workspace;
    size_t workspace_bytes;
};
// The single-layer call as a group of one.
GroupArgs group_of_one(const ForwardArgs &a);
// The layer of projection j alone, for the paths that run one layer at a time.
ForwardArgs layer_of(const GroupArgs &g, int j);

// Decode path (up to kMidMaxTokens tokens per launch pair; lb_decode.cu).
// Up to kSmallMaxTokens tokens run on CUDA cores (nibble tables, lb_gemv.cu)
// when the shapes fit it, the rest on tcgen05 (lb_mid.cu).  kDecodeMaxTokens
// bounds the fixed-scratch entry point.
constexpr int kSmallMaxTokens = 4;
size_t small_workspace_bytes(int M, const GroupArgs &g);
// One launch pair for the whole group (a single layer is a group of one).
cudaError_t small_forward(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream, int m0, int M);
// False when the shapes do not fit the small path (its latent tables must fit
// shared memory); the tensor-core decode path takes those.
bool small_fits(int M, const GroupArgs &g, const DeviceInfo &dev);
cudaError_t small_prepare_device(const DeviceInfo &dev);
constexpr int kDecodeMaxTokens = 32;
size_t decode_workspace_bytes(int tokens, int n_in, int n_out, const int *ranks, int npaths);
cudaError_t decode_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream);
cudaError_t decode_prepare_device(const DeviceInfo &dev);
// A group of siblings at any token count: one launch pair for the whole group
// up to kMidMaxTokens tokens (small path when it fits, else tcgen05), each
// projection's own prefill launches beyond.
size_t group_workspace_bytes(const GroupArgs &g);
cudaError_t group_forward(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream);

// Fault injection for tests (lb_debug_inject_stall): the limit of the
// tcgen05 decode kernels' bounded waits (ns) and whether their first
// producer warp skips one arrival.  Read when a launch is prepared.
unsigned long long debug_wait_ns();
int debug_skip_arrival();

// Up to kMidMaxTokens tokens per launch pair on tcgen05 with the sign matrix
// as the 128-row MMA operand and the tokens as N (lb_mid.cu).
constexpr int kMidMaxTokens = 128;
size_t mid_workspace_bytes(int tokens, const int *ranks, int npaths);
cudaError_t mid_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M);
cudaError_t mid_prepare_device(const DeviceInfo &dev);
// One launch pair for a whole group of siblings (the latent of every layer in
// one workspace z [M][sum of ranks], fp16).
size_t mid_group_workspace_bytes(int tokens, const GroupArgs &g);
cudaError_t mid_group_forward(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream, int m0, int M);
cudaError_t mid_latent(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M, uint16_t *z,
                       int64_t ldz);
cudaError_t mid_expand(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M,
                       const uint16_t *z, int64_t ldz);

// Prefill path (more than kMidMaxTokens tokens): two tcgen05 GEMMs with the
// binary operand expanded in shared memory (lb_prefill.cu).
size_t prefill_workspace_bytes(int tokens, const int *ranks, int npaths);
cudaError_t prefill_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream);
cudaError_t prefill_prepare_device(DeviceInfo &dev);  // also fills dev.pair_slots
bool prefill_pairs_enabled();                          // lb_set_prefill_pairs

// ----------------------------------------------------------------- host buffers (lb_host_io.cu)
// Copies `bytes` (a multiple of 16) from pinned host memory, given by its
// device mapping, to device memory with one kernel on `stream`, chained to
// the kernels before and after it by programmatic dependent launch.
cudaError_t host_gather_launch(const void *src, void *dst, size_t bytes, cudaStream_t stream);
cudaError_t prefill_latent(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, uint16_t *z, int64_t ldz);
cudaError_t prefill_expand(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, const uint16_t *z,
                           int64_t ldz);

// ---------------------------------------------------------------- backward (lb_backward.cu, lb_prefill.cu)
// The backward pass's contraction-1-shaped steps on the prefill kernels:
// C[m, n] = sum_k A[m, k] B[n, k] with A bf16 [M x K], B[n, k] =
// sign(row n of bits_p)[k] s_p[k] (rows n < r0 from path 0, the rest from
// path 1), stored as l (.) C (l_p per column; C itself where l is null) in
// fp16, or bf16 with out_bf16, [M x (r0 + r1)]; with aux (fp16, or bf16 with
// aux_bf16, [M x N]) also part[m / 32][n] = sum over the 32-row block of the
// unscaled C * aux.
struct Bwd1Args {
    int M, K, r0, r1;
    const uint16_t *a;
    int64_t lda;
    const uint32_t *bits0, *bits1;  // packed rows along K (bits1 null: one path)
    int64_t ld0, ld1;
    const uint16_t *s0, *s1;  // per-K scale of each path's rows (fp16, length K)
    const uint16_t *l0, *l1;  // per-column scale of the stored output, or null
    uint16_t *out;
    int64_t ldo;
    const uint16_t *aux;
    int64_t ldaux;
    float *part;
    int out_bf16, aux_bf16;
};
cudaError_t bwd_contraction1(const Bwd1Args &b, const DeviceInfo &dev, cudaStream_t stream);

// A scale gradient as a weight-gradient product (lb_wgrad.cu): for every row
// o of a path's sign matrix S_p (packed along the latent) and every path p,
// the sum over k in path p of sign(S_p[o, k]) l_p[k] G[o, k], G = A^T B with
// A bf16 [tokens x rows] and B bf16 [tokens x R] (the paths side by side), the
// tokens as the MMA's K; l_p null means 1.  dh: A = dy, B = c, S = U, l.
// dg: A = x, B = l (.) a, S = V, no l.  One partial per tile column and
// token part: part_p[row][o], rows = WgradPlan::rows.
struct WgradPlan {
    int bn, ntn, nsplit, kps, rows;
};
WgradPlan wgrad_plan(int rows, int R, int tokens, int sms);
int wgrad_max_parts(int R, int tokens);  // the most partial rows any plan takes
struct WgradArgs {
    int tokens, rows, R, r0;
    const uint16_t *a;
    int64_t lda;
    const uint16_t *b;
    int64_t ldb;
    const uint32_t *bits0, *bits1;  // packed rows o along the path's latent (bits1 null: one path)
    int64_t bld0, bld1;
    const uint16_t *l0, *l1;  // latent scale of each path, or null for 1
    float *part0, *part1;     // part1 null: one path
};
cudaError_t wgrad_prepare_device(const DeviceInfo &dev);
cudaError_t wgrad_scale_grad(const WgradArgs &w, const DeviceInfo &dev, cudaStream_t stream);
// dx = sum_p g_p (.) S_V,p (l_p (.) a_p): the forward's contraction-2 shape in
// bf16 (A = l (.) a bf16 [M x R], B rows i = +-bf16(g_p[i]) by V packed along
// the latent), out bf16 [M x n_in].
struct BwdDxArgs {
    int M, n_in, r0, r1;
    const uint16_t *a;
    int64_t lda;
    const uint32_t *bits0, *bits1;
    int64_t ld0, ld1;
    const uint16_t *g0, *g1;
    uint16_t *dx;
    int64_t lddx;
};
cudaError_t bwd_dx(const BwdDxArgs &b, const DeviceInfo &dev, cudaStream_t stream);

// The whole backward pass (lb_linear_backward), already validated.
struct BackwardArgs {
    const uint16_t *x;
    int64_t ldx;
    const uint16_t *dy;
    int64_t lddy;
    int tokens, n_in, n_out, npaths;
    PathDesc path[2];
    uint16_t *dx;  // may be null
    int64_t lddx;
    float *dh, *dg, *dl;
    void *workspace;
    size_t workspace_bytes;
};
size_t backward_workspace_bytes(int tokens, int n_in, int n_out, const int *ranks, int npaths);
cudaError_t backward_launch(const BackwardArgs &b, const DeviceInfo &dev, cudaStream_t stream);

// Either contraction alone, the latent in caller memory: z fp16 [tokens][ldz]
// (token-major, the paths side by side, path 0 first); any number of tokens
// (up to 32 on the lb_mid.cu kernels, more on the prefill kernels).
cudaError_t latent_launch(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, uint16_t *z, int64_t ldz);
cudaError_t expand_launch(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, const uint16_t *z,
                          int64_t ldz);

}  // namespace lb
