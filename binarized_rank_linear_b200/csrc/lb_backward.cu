// lb_backward.cu - the backward pass of the layer: the gradients with respect
// to x and to every path's scale vectors h, g and l, given dy = dL/dy.
//
// The forward pass (sesamedisk.com, "Samsung LittleBit 13B Model", section
// "What the method actually computes", Proposition 1) per path p is
//     t = g (.) x,  c = S_V^T t,  z = l (.) c,  e = S_U z,  y = sum_p h (.) e,
// and quantization-aware training runs back through it (littlebitllm.com,
// "Pipeline").  With the signs held fixed the chain rule gives, per path,
//     a  = S_U^T (h (.) dy)            (the gradient with respect to z)
//     dl = sum over tokens of a (.) c
//     dt = S_V (l (.) a)               (the gradient with respect to t)
//     dg = sum over tokens of x (.) dt,   dx = sum_p g (.) dt
//     dh = sum over tokens of dy (.) e
// Five tcgen05 products compute them:
//   K1  c = S_V^T (g (.) x)            x [M x n_in] against the packed rows of
//                                      V^T (lb_prefill.cu, mode 3); bf16
//   K2  a_s = l (.) S_U^T (h (.) dy)   dy [M x n_out] against the rows of U^T
//                                      (mode 3), scaled by l on the way out;
//                                      the epilogue also forms a (.) c per
//                                      32-token block (dl partials); bf16
//   K3  dh_p[o] = sum_k sign(U_p[o, k]) l_p[k] (dy^T c)[o, k]
//   K4  dg_p[i] = sum_k sign(V_p[i, k]) (x^T a_s)[i, k]
//                                      both with the tokens as the MMA's K
//                                      (lb_wgrad.cu): per row a sum over k in
//                                      the epilogue (partials per tile column)
//   K5  dx = sum_p g_p (.) S_V,p a_s,p the forward's contraction-2 shape in
//                                      bf16 (mode 2), V packed along r
// then one kernel adds each partial column over its rows in order, so the
// results do not depend on timing.  K2, K4 and K5 read the factors along the
// other axis from the forward pass: U^T packed along n_out and V packed along
// r, which one bit-transpose launch makes from the forward's packed words
// into the workspace, so the call takes the forward pass's lb_path as it is.
// c and a_s travel between the products in bf16, the type of x and dy that
// K3 and K4 multiply them with.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"

namespace lb {
namespace {

// ------------------------------------------------------------ bit transpose
// out[col][row / 32] bit (row % 32) = in[row][col / 32] bit (col % 32), for a
// packed matrix of `rows` x `cols` bits (both multiples of 32).  One warp per
// column word cb and up to kRowBlocks consecutive 32-row blocks rb: for each
// block, lane l loads row 32 rb + l's word cb, and the ballot of bit j over
// the lanes is output row 32 cb + j's word rb, kept by lane j.  Each lane
// then stores its consecutive output words together (one 32-byte sector).
constexpr int kTransposeWarps = 8;
constexpr int kRowBlocks = 8;

// Up to four transposes in one launch: matrix q takes the CTAs first_cta[q] ..
constexpr int kMaxTransposes = 4;
struct TransposeJob {
    const uint32_t *in;
    int64_t ld_in;
    int rows, cols;
    uint32_t *out;
    int64_t ld_out;
    int first_cta;
};
struct TransposeBatch {
    TransposeJob job[kMaxTransposes];
    int n;
};

__global__ void __launch_bounds__(32 * kTransposeWarps) transpose_bits_kernel(const __grid_constant__ TransposeBatch b)
{
    int q = 0;
    while (q + 1 < b.n && (int)blockIdx.x >= b.job[q + 1].first_cta) ++q;
    const TransposeJob &t = b.job[q];
    const int lane = threadIdx.x & 31;
    const int64_t job = (int64_t)((int)blockIdx.x - t.first_cta) * kTransposeWarps + (threadIdx.x >> 5);
    const int rbs = t.rows >> 5, cbs = t.cols >> 5;
    const int groups = (rbs + kRowBlocks - 1) / kRowBlocks;
    if (job >= (int64_t)groups * cbs) return;  // whole warps leave together
    const int rg = (int)(job % groups), cb = (int)(job / groups);
    const int rb0 = rg * kRowBlocks, nrb = min(kRowBlocks, rbs - rb0);
    uint32_t w[kRowBlocks];
#pragma unroll
    for (int r = 0; r < kRowBlocks; ++r)
        w[r] = r < nrb ? __ldg(t.in + (int64_t)(32 * (rb0 + r) + lane) * t.ld_in + cb) : 0u;
    uint32_t mine[kRowBlocks];
#pragma unroll
    for (int r = 0; r < kRowBlocks; ++r) {
        mine[r] = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const uint32_t v = __ballot_sync(0xffffffffu, (w[r] >> j) & 1u);
            if (lane == j) mine[r] = v;
        }
    }
    uint32_t *dst = t.out + (int64_t)(32 * cb + lane) * t.ld_out + rb0;
#pragma unroll
    for (int r = 0; r < kRowBlocks; ++r)
        if (r < nrb) dst[r] = mine[r];
}

// Adds one matrix to a batch; returns its CTA count.
int add_transpose(TransposeBatch &b, const uint32_t *in, int64_t ld_in, int rows, int cols, uint32_t *out,
                  int64_t ld_out, int first_cta)
{
    const int64_t jobs = (int64_t)((rows / 32 + kRowBlocks - 1) / kRowBlocks) * (cols / 32);
    b.job[b.n++] = TransposeJob{in, ld_in, rows, cols, out, ld_out, first_cta};
    return (int)((jobs + kTransposeWarps - 1) / kTransposeWarps);
}

// ------------------------------------------------------------ partial sums
// out[n] = sum over the rows rb = 0 .. blocks - 1 of part[rb][n],
// for up to kMaxSegments vectors in one launch.  A CTA takes 32 columns; its
// kGroups warps take the blocks rb = g, g + kGroups, ... of those columns
// (each in block order), and warp 0 adds the kGroups sums in group order:
// a fixed order, so the result does not depend on timing.
constexpr int kMaxSegments = 5;
constexpr int kGroups = 8;
struct ReduceSeg {
    const float *part;
    float *out;
    int n;
    int blocks;  // rows of partials: 32-token blocks, or K3's tile columns and token parts
};
struct ReduceParams {
    ReduceSeg seg[kMaxSegments];
    int nseg;
};

__global__ void __launch_bounds__(32 * kGroups) reduce_partials_kernel(const __grid_constant__ ReduceParams p)
{
    __shared__ float sums[kGroups][32];
    const int lane = threadIdx.x & 31, g = threadIdx.x >> 5;
    int64_t col = (int64_t)blockIdx.x * 32 + lane;
    const ReduceSeg *seg = nullptr;
    for (int s = 0; s < p.nseg; ++s) {
        if (col < p.seg[s].n) {
            seg = &p.seg[s];
            break;
        }
        col -= p.seg[s].n;
    }
    float acc = 0.0f;
    if (seg != nullptr)
        for (int rb = g; rb < seg->blocks; rb += kGroups) acc += __ldg(seg->part + (int64_t)rb * seg->n + col);
    sums[g][lane] = acc;
    __syncthreads();
    if (g == 0 && seg != nullptr) {
        float t = 0.0f;
#pragma unroll
        for (int q = 0; q < kGroups; ++q) t += sums[q][lane];
        seg->out[col] = t;
    }
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// Workspace layout of one call (every piece 256-byte aligned).
struct BwdLayout {
    size_t ut[2], v[2];     // transposed sign words of each path
    size_t c, a;            // bf16 [M x R]: c, and l (.) a
    size_t pl, ph[2], pg[2];  // partials
    size_t total;
};

BwdLayout layout(int M, int n_in, int n_out, const int *ranks, int npaths)
{
    BwdLayout L{};
    size_t off = 0;
    const int R = ranks[0] + (npaths > 1 ? ranks[1] : 0);
    const size_t RB = (size_t)((M + 31) / 32);
    for (int q = 0; q < npaths; ++q) {
        L.ut[q] = off;
        off += align256((size_t)ranks[q] * (size_t)(n_out / 32) * 4);
        L.v[q] = off;
        off += align256((size_t)n_in * (size_t)(ranks[q] / 32) * 4);
    }
    L.c = off;
    off += align256((size_t)M * R * 2);
    L.a = off;
    off += align256((size_t)M * R * 2);
    L.pl = off;
    off += align256(RB * R * 4);
    // dh's and dg's partial rows (K3, K4): at most wgrad_max_parts; dl's: the 32-token blocks
    const size_t HB = std::max(RB, (size_t)wgrad_max_parts(R, M));
    for (int q = 0; q < npaths; ++q) {
        L.ph[q] = off;
        off += align256(HB * (size_t)n_out * 4);
        L.pg[q] = off;
        off += align256(HB * (size_t)n_in * 4);
    }
    L.total = off;
    return L;
}

}  // namespace

size_t backward_workspace_bytes(int tokens, int n_in, int n_out, const int *ranks, int npaths)
{
    return layout(tokens, n_in, n_out, ranks, npaths).total;
}

cudaError_t backward_launch(const BackwardArgs &b, const DeviceInfo &dev, cudaStream_t stream)
{
    const int M = b.tokens, npaths = b.npaths;
    const int ranks[2] = {b.path[0].rank, npaths > 1 ? b.path[1].rank : 0};
    const int r0 = ranks[0], r1 = ranks[1], R = r0 + r1;
    const BwdLayout L = layout(M, b.n_in, b.n_out, ranks, npaths);
    uint8_t *ws = static_cast<uint8_t *>(b.workspace);
    uint32_t *ut[2] = {nullptr, nullptr}, *v[2] = {nullptr, nullptr};
    TransposeBatch tr{};
    int ctas = 0;
    for (int q = 0; q < npaths; ++q) {
        const PathDesc &P = b.path[q];
        ut[q] = reinterpret_cast<uint32_t *>(ws + L.ut[q]);
        v[q] = reinterpret_cast<uint32_t *>(ws + L.v[q]);
        // U [n_out x r] -> U^T [r x n_out]; V^T [r x n_in] -> V [n_in x r]
        ctas += add_transpose(tr, P.u_bits, P.u_ld, b.n_out, P.rank, ut[q], b.n_out / 32, ctas);
        ctas += add_transpose(tr, P.vt_bits, P.vt_ld, P.rank, b.n_in, v[q], P.rank / 32, ctas);
    }
    transpose_bits_kernel<<<(unsigned)ctas, 32 * kTransposeWarps, 0, stream>>>(tr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    uint16_t *c = reinterpret_cast<uint16_t *>(ws + L.c);
    uint16_t *a = reinterpret_cast<uint16_t *>(ws + L.a);
    float *pl = reinterpret_cast<float *>(ws + L.pl);
    float *ph[2] = {reinterpret_cast<float *>(ws + L.ph[0]), npaths > 1 ? reinterpret_cast<float *>(ws + L.ph[1]) : nullptr};
    float *pg[2] = {reinterpret_cast<float *>(ws + L.pg[0]), npaths > 1 ? reinterpret_cast<float *>(ws + L.pg[1]) : nullptr};
    const PathDesc &P0 = b.path[0], &P1 = b.path[1];
    const bool two = npaths > 1;

    // K1: c = S_V^T (g (.) x), unscaled
    Bwd1Args k1{};
    k1.M = M;
    k1.K = b.n_in;
    k1.r0 = r0;
    k1.r1 = r1;
    k1.a = b.x;
    k1.lda = b.ldx;
    k1.bits0 = P0.vt_bits;
    k1.ld0 = P0.vt_ld;
    k1.s0 = P0.g;
    if (two) {
        k1.bits1 = P1.vt_bits;
        k1.ld1 = P1.vt_ld;
        k1.s1 = P1.g;
    }
    k1.out = c;
    k1.ldo = R;
    k1.out_bf16 = 1;
    e = bwd_contraction1(k1, dev, stream);
    if (e != cudaSuccess) return e;

    // K2: a_s = l (.) S_U^T (h (.) dy), scaled by l on the way out; dl
    // partials sum a (.) c from the unscaled accumulator
    Bwd1Args k2{};
    k2.M = M;
    k2.K = b.n_out;
    k2.r0 = r0;
    k2.r1 = r1;
    k2.a = b.dy;
    k2.lda = b.lddy;
    k2.bits0 = ut[0];
    k2.ld0 = b.n_out / 32;
    k2.s0 = P0.h;
    k2.l0 = P0.l;
    if (two) {
        k2.bits1 = ut[1];
        k2.ld1 = b.n_out / 32;
        k2.s1 = P1.h;
        k2.l1 = P1.l;
    }
    k2.out = a;
    k2.ldo = R;
    k2.out_bf16 = 1;
    k2.aux = c;
    k2.ldaux = R;
    k2.aux_bf16 = 1;
    k2.part = pl;
    e = bwd_contraction1(k2, dev, stream);
    if (e != cudaSuccess) return e;

    // K3: dh_p[o] = sum_k sign(U_p[o, k]) l_p[k] G[o, k], G = dy^T c
    WgradArgs k3{};
    k3.tokens = M;
    k3.rows = b.n_out;
    k3.R = R;
    k3.r0 = r0;
    k3.a = b.dy;
    k3.lda = b.lddy;
    k3.b = c;
    k3.ldb = R;
    k3.bits0 = P0.u_bits;
    k3.bld0 = P0.u_ld;
    k3.l0 = P0.l;
    if (two) {
        k3.bits1 = P1.u_bits;
        k3.bld1 = P1.u_ld;
        k3.l1 = P1.l;
    }
    k3.part0 = ph[0];
    k3.part1 = ph[1];
    e = wgrad_scale_grad(k3, dev, stream);
    if (e != cudaSuccess) return e;

    // K4: dg_p[i] = sum_k sign(V_p[i, k]) H[i, k], H = x^T a_s (l already in a_s)
    WgradArgs k4{};
    k4.tokens = M;
    k4.rows = b.n_in;
    k4.R = R;
    k4.r0 = r0;
    k4.a = b.x;
    k4.lda = b.ldx;
    k4.b = a;
    k4.ldb = R;
    k4.bits0 = v[0];
    k4.bld0 = r0 / 32;
    if (two) {
        k4.bits1 = v[1];
        k4.bld1 = r1 / 32;
    }
    k4.part0 = pg[0];
    k4.part1 = pg[1];
    e = wgrad_scale_grad(k4, dev, stream);
    if (e != cudaSuccess) return e;

    // K5: dx = sum_p g_p (.) S_V,p a_s,p
    if (b.dx != nullptr) {
        BwdDxArgs k5{};
        k5.M = M;
        k5.n_in = b.n_in;
        k5.r0 = r0;
        k5.r1 = r1;
        k5.a = a;
        k5.lda = R;
        k5.bits0 = v[0];
        k5.ld0 = r0 / 32;
        k5.g0 = P0.g;
        if (two) {
            k5.bits1 = v[1];
            k5.ld1 = r1 / 32;
            k5.g1 = P1.g;
        }
        k5.dx = b.dx;
        k5.lddx = b.lddx;
        e = bwd_dx(k5, dev, stream);
        if (e != cudaSuccess) return e;
    }
    const int hrows = wgrad_plan(b.n_out, R, M, dev.sm_count).rows;
    const int grows = wgrad_plan(b.n_in, R, M, dev.sm_count).rows;

    // the partial sums, each added over its rows in row order
    ReduceParams rp{};
    const int tb = (M + 31) / 32;
    int total = 0;
    auto add = [&](const float *part, float *out, int n, int blocks) {
        rp.seg[rp.nseg++] = ReduceSeg{part, out, n, blocks};
        total += n;
    };
    add(pl, b.dl, R, tb);
    add(ph[0], b.dh, b.n_out, hrows);
    if (two) add(ph[1], b.dh + b.n_out, b.n_out, hrows);
    add(pg[0], b.dg, b.n_in, grows);
    if (two) add(pg[1], b.dg + b.n_in, b.n_in, grows);
    // every segment's length is a multiple of 32, so a CTA's 32 columns lie in one segment
    reduce_partials_kernel<<<(unsigned)(total / 32), 32 * kGroups, 0, stream>>>(rp);
    return cudaGetLastError();
}

}  // namespace lb
