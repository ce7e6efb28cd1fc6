// lb_decode.cu - the forward pass for 1..32 tokens.
//
// The layer (sesamedisk.com, "Samsung LittleBit 13B Model", section "What the
// method actually computes", Proposition 1), per path p:
//     z_p = l_p (.) (sign(V_p)^T (g_p (.) x))         contraction 1 (latent)
//     y   = sum_p h_p (.) (sign(U_p) z_p)             contraction 2 (expand)
// Both paths of residual compensation run in the same two launches.
//
// At batch 1 the layer is a 2-3 MB stream of packed sign bits, so a call is
// bound by latency: each kernel is one DRAM round trip for its weights plus
// one L2 round trip for its activations, and everything else is kept short.
//
//  * Tensor cores on sign bits.  Every factor entry is +-1, so a sign bit
//    becomes an fp16 MMA operand with two integer ops: shift the bit pair into
//    the fp16 sign positions and XOR it onto a constant.  Contraction 1 runs
//    A = +-1 (exact) against B = g (.) x in fp16 (one rounding); contraction 2
//    runs A = +-h_o (exact fp16) against B = z in fp16.  Products are exact in
//    fp32 and sums accumulate in fp32 (mma.m16n8k16, four independent chains).
//    Activations in fp16 follow the page ("activations X stay in FP16").
//  * The packed layout is plain (column 32w + j at bit j of word w).  The
//    MMA's k index is mapped to columns so that a lane's two k values of one A
//    register are columns c and c + 16 of a word: one shift puts both bits at
//    the fp16 sign positions (bits 15 and 31).  The B operand is built in
//    shared memory in the same column order; the contraction does not depend
//    on the order of k.
//  * Every global read of a kernel is an asynchronous copy issued at entry
//    (weights) or right after the dependency wait (activations), so each
//    kernel pays one DRAM and one L2 latency.  Kernel parameters are read with
//    static indices only (no dependent constant-bank loads at entry).
//  * The two kernels are chained with programmatic dependent launch.  Each
//    releases its dependent after its MMA loop, not at entry: released
//    dependents stay resident while they wait, and releasing at entry made
//    every later kernel of a chain resident at once and slowed the running
//    one down.  The dependent's prologue (its weight copies) overlaps the tail.
//  * Contraction 1 splits n_in across CTAs only when one CTA's slice would not
//    fit in shared memory; the CTAs then write fp32 partial latents and
//    contraction 2 sums them (fixed order) while it loads the latent.  There
//    are no atomics: results are deterministic.
#include <algorithm>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"

namespace lb {
namespace {

// 512 threads for up to 16 tokens, 256 for 17..32 (more accumulators).
template <int NT>
struct Shape {
    static constexpr int kThreads = NT == 4 ? 256 : 512;
    static constexpr int kWarps = kThreads / 32;
};

constexpr uint32_t kOnes = 0x3C003C00u;  // fp16 pair (+1, +1)
// Contraction 2 keeps the partial latents of a split contraction 1 in shared
// memory; this bounds their size (and with it the workspace).
constexpr size_t kMaxPartialBytes = 96 * 1024;

// A 16-byte fragment holds 8 fp16 values of 32 consecutive columns for the
// lane quad position tg: halves 0..7 are columns tg, tg+16, tg+4, tg+20,
// tg+8, tg+24, tg+12, tg+28.  Register j (halves 2j, 2j+1) is one MMA B
// register: j = 0, 1 for the k-step over columns {0..7, 16..23}, j = 2, 3 for
// the k-step over {8..15, 24..31}.
__device__ __forceinline__ int frag_half_of_col(int c) { return 2 * ((c >> 2) & 3) + (c >> 4); }
__device__ __forceinline__ int frag_col(int tg, int half) { return tg + 16 * (half & 1) + 4 * (half >> 1); }

// (+-1, +-1) from the sign bits at positions (15 - sh, 31 - sh) of w.
__device__ __forceinline__ uint32_t sign_pair(uint32_t w, int sh) { return kOnes ^ ((w << sh) & 0x80008000u); }
// (+-s, +-s') from a packed scale pair and the same two sign bits.
__device__ __forceinline__ uint32_t signed_pair(uint32_t scale2, uint32_t w, int sh)
{
    return scale2 ^ ((w << sh) & 0x80008000u);
}

// Number of 4-word (128-column) quads that cover n columns.
__host__ __device__ __forceinline__ int quads_of(int n) { return (n + 127) / 128; }

// Shared-memory row stride (words) for bit rows of `quads` quads: a multiple
// of 4 words whose quad count is odd, so the 8 rows one LDS.128 touches fall
// in distinct bank groups.
__host__ __device__ __forceinline__ int bit_row_stride(int quads) { return 4 * (quads | 1); }

// ============================================================ contraction 1
struct LatentParams {
    const uint16_t *x;
    int64_t ldx;
    int M, n_in;
    const uint32_t *vt0, *vt1;
    int64_t vt_ld0, vt_ld1;
    const uint16_t *g0, *g1, *l0, *l1;
    int rank0, rank1;
    int groups0;  // row groups of path 0 (path 1's follow)
    int rt;       // 16-row tiles per CTA; kWarps / rt warps per tile
    int cs;       // CTAs splitting n_in; > 1 writes fp32 partials
    int quads;    // quads of n_in
    int cq;       // quads staged per chunk
    int S;        // smem stride of a bit row, words
    uint4 *zf;    // cs == 1: latent fragments (fp16)
    int64_t zoff0, zoff1;
    float *part;  // cs > 1: [cs][rank0 + rank1][M]
    int *status;
};

template <int NT>
__global__ void __launch_bounds__(Shape<NT>::kThreads) latent_kernel(const LatentParams p)
{
    constexpr int T = Shape<NT>::kThreads, NW = Shape<NT>::kWarps, N8 = NT * 8;
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gr = lane >> 2, tg = lane & 3;
    const int cs = p.cs;
    const int group = blockIdx.x / cs, split_c = blockIdx.x - group * cs;
    const bool second = group >= p.groups0;
    const int row0 = (second ? group - p.groups0 : group) * 16 * p.rt;
    const int rank = second ? p.rank1 : p.rank0;
    const int rows = min(16 * p.rt, rank - row0);
    const int q0 = split_c * p.quads / cs, q1 = (split_c + 1) * p.quads / cs;
    const int W = p.n_in >> 5;
    const int w0 = 4 * q0;
    const int nw = min(4 * q1, W) - w0;  // real words (32 columns each) of this CTA
    const int M = p.M;
    const int cq = p.cq;
    const int nch = (q1 - q0 + cq - 1) / cq;
    const int64_t ld = second ? p.vt_ld1 : p.vt_ld0;
    const uint32_t *vt = (second ? p.vt1 : p.vt0) + (int64_t)row0 * ld + w0;
    const uint16_t *g = (second ? p.g1 : p.g0) + 32 * w0;
    const uint16_t *lsrc = (second ? p.l1 : p.l0) + row0;
    const uint16_t *xb = p.x + 32 * w0;
    const int cstride = 128 * cq;  // halves per staged row of a chunk

    uint32_t *sbits = reinterpret_cast<uint32_t *>(smem);                    // [16 rt][S]
    uint16_t *lraw = reinterpret_cast<uint16_t *>(sbits + 16 * p.rt * p.S);  // [16 rt]
    uint16_t *graw = lraw + 16 * p.rt;                                       // [2][128 cq]
    uint16_t *xraw = graw + 2 * cstride;                                     // [2][M][128 cq]
    uint4 *tf = reinterpret_cast<uint4 *>(xraw + 2 * cstride * M);           // [4 cq][M][4]
    float *sred = reinterpret_cast<float *>(tf + 16 * cq * M);               // [NW][16][N8]

    // (1) weights: every sign bit of this CTA, its l slice and the g slice of
    // the first chunk, all as asynchronous copies issued before any wait
    if ((ld & 3) == 0) {
        const int nqr = (nw + 3) >> 2;
        for (int r = warp; r < rows; r += NW)
            for (int qq = lane; qq < nqr; qq += 32) cp_async16(sbits + r * p.S + 4 * qq, vt + r * ld + 4 * qq);
    } else {
        for (int r = warp; r < rows; r += NW)
            for (int w = lane; w < nw; w += 32) cp_async4(sbits + r * p.S + w, vt + r * ld + w);
    }
    if (tid < rows / 8) cp_async16(lraw + 8 * tid, lsrc + 8 * tid);
    auto stage_g = [&](int ch) {
        const int wa = 4 * ch * cq, n16 = 4 * (min(nw, wa + 4 * cq) - wa);
        uint16_t *dst = graw + (ch & 1) * cstride;
        for (int e = tid; e < n16; e += T) cp_async16(dst + 8 * e, g + 32 * wa + 8 * e);
    };
    auto stage_x = [&](int ch) {
        const int wa = 4 * ch * cq, n16 = 4 * (min(nw, wa + 4 * cq) - wa);
        uint16_t *dst = xraw + (ch & 1) * cstride * M;
        for (int m = 0; m < M; ++m)
            for (int e = tid; e < n16; e += T)
                cp_async16(dst + m * cstride + 8 * e, xb + (int64_t)m * p.ldx + 32 * wa + 8 * e);
    };
    stage_g(0);
    cp_async_commit();

    // (2) x is produced by the previous kernel on the stream
    pdl_wait();
    stage_x(0);
    cp_async_commit();

    // four independent accumulator chains (word parity x k-step), summed in
    // a fixed order at the end
    float acc[NT][4], acc4[3][NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = acc4[0][nt][i] = acc4[1][nt][i] = acc4[2][nt][i] = 0.f;
    const int ws = NW / p.rt;
    const int tile = warp / ws, split = warp - tile * ws;
    const bool active = 16 * tile < rows;
    const uint32_t *b0 = sbits + (16 * tile + gr) * p.S;
    const uint32_t *b1 = b0 + 8 * p.S;
    bool overflow = false;

    for (int ch = 0; ch < nch; ++ch) {
        if (ch + 1 < nch) {
            stage_g(ch + 1);
            stage_x(ch + 1);
            cp_async_commit();
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_group<0>();
        }
        __syncthreads();

        // (3) B fragments of this chunk: t = g (.) x in fp16, in the MMA's column order
        const int cw = min(4 * cq, nw - 4 * ch * cq);
        const uint16_t *gbuf = graw + (ch & 1) * cstride;
        const uint16_t *xbuf = xraw + (ch & 1) * cstride * M;
        for (int e = tid; e < 16 * cq * M; e += T) {
            const int t = e & 3, wm = e >> 2;
            const int wl = wm / M, m = wm - wl * M;
            uint4 out = make_uint4(0u, 0u, 0u, 0u);
            if (wl < cw) {
                const uint16_t *gw = gbuf + 32 * wl;
                const uint16_t *xw = xbuf + m * cstride + 32 * wl;
                float f[8];
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    const int col = frag_col(t, h);
                    f[h] = f16_bits_to_float(gw[col]) * bf16_bits_to_float(xw[col]);
                    overflow |= beyond_f16(f[h]);
                }
                out = make_uint4(pack_half2(f[0], f[1]), pack_half2(f[2], f[3]), pack_half2(f[4], f[5]),
                                 pack_half2(f[6], f[7]));
            }
            tf[e] = out;  // == tf[(wl * M + m) * 4 + t]
        }
        __syncthreads();

        // (4) tensor-core contraction over this chunk
        if (active) {
            const int nqc = (cw + 3) >> 2;
            const int qa = split * nqc / ws, qb = (split + 1) * nqc / ws;
            for (int qq = qa; qq < qb; ++qq) {
                const int qb4 = 4 * (ch * cq + qq);
                const uint4 W0 = *reinterpret_cast<const uint4 *>(b0 + qb4);
                const uint4 W1 = *reinterpret_cast<const uint4 *>(b1 + qb4);
                const uint32_t wa[4] = {W0.x, W0.y, W0.z, W0.w};
                const uint32_t wb[4] = {W1.x, W1.y, W1.z, W1.w};
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    const int wl = 4 * qq + wi;
                    uint4 X[NT];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int m = gr + 8 * nt;
                        X[nt] = m < M ? tf[(wl * M + m) * 4 + tg] : make_uint4(0u, 0u, 0u, 0u);
                    }
                    float(&c0)[NT][4] = (wi & 1) ? acc4[1] : acc;
                    float(&c1)[NT][4] = (wi & 1) ? acc4[2] : acc4[0];
                    uint32_t a0 = sign_pair(wa[wi], 15 - tg), a1 = sign_pair(wb[wi], 15 - tg);
                    uint32_t a2 = sign_pair(wa[wi], 11 - tg), a3 = sign_pair(wb[wi], 11 - tg);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16_16816(c0[nt], a0, a1, a2, a3, X[nt].x, X[nt].y);
                    a0 = sign_pair(wa[wi], 7 - tg);
                    a1 = sign_pair(wb[wi], 7 - tg);
                    a2 = sign_pair(wa[wi], 3 - tg);
                    a3 = sign_pair(wb[wi], 3 - tg);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16_16816(c1[nt], a0, a1, a2, a3, X[nt].z, X[nt].w);
                }
            }
        }
    }
    pdl_launch_dependents();

    // (5) sum the chains, then the warps of each tile (fixed order)
    {
        float *mine = sred + warp * 16 * N8;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = (acc[nt][i] + acc4[0][nt][i]) + (acc4[1][nt][i] + acc4[2][nt][i]);
            const int c = 8 * nt + 2 * tg;
            mine[gr * N8 + c] = v[0];
            mine[gr * N8 + c + 1] = v[1];
            mine[(gr + 8) * N8 + c] = v[2];
            mine[(gr + 8) * N8 + c + 1] = v[3];
        }
    }
    __syncthreads();
    for (int e = tid; e < rows * M; e += T) {
        const int r = e / M, m = e - r * M;
        const int t = r >> 4, rr = r & 15;
        float s = 0.f;
        for (int j = 0; j < ws; ++j) s += sred[((t * ws + j) * 16 + rr) * N8 + m];
        const int k = row0 + r;
        if (cs == 1) {
            // (6a) whole rows here: scale by l and store the fp16 latent fragment
            const float z = s * f16_bits_to_float(lraw[r]);
            overflow |= beyond_f16(z);
            const int kw = k >> 5, cc = k & 31;
            uint16_t *dst = reinterpret_cast<uint16_t *>(p.zf + (second ? p.zoff1 : p.zoff0) +
                                                         ((int64_t)kw * M + m) * 4 + (cc & 3));
            dst[frag_half_of_col(cc)] = __half_as_ushort(__float2half_rn(z));
        } else {
            // (6b) a slice of n_in: store the fp32 partial; contraction 2 sums them
            const int kg = (second ? p.rank0 : 0) + k;
            p.part[((int64_t)split_c * (p.rank0 + p.rank1) + kg) * M + m] = s;
        }
    }
    if (overflow) set_status(p.status, LB_ERR_RANGE);
}

// ============================================================ contraction 2
struct ExpandParams {
    int zmode;  // 0: fp16 fragments from contraction 1; 1: fp32 partials to sum
    const uint4 *zf;
    int64_t zoff0, zoff1;
    const float *part;
    int cs;
    const uint16_t *l0, *l1;
    int M, n_out;
    const uint32_t *u0, *u1;
    int64_t u_ld0, u_ld1;
    const uint16_t *h0, *h1;
    int rank0, rank1;
    int npaths;
    int kq0, kq1;  // latent quads per path
    int S0, S1;    // smem stride of a bit row per path, words
    int flat0, flat1;  // 1: rows copied as one contiguous block (stride = u_ld, read word by word)
    int ks;        // warps splitting the latent; kWarps / ks tiles in flight
    int tiles_per_cta;
    uint16_t *y;
    int64_t ldy;
    int *status;
};

template <int NT>
__global__ void __launch_bounds__(Shape<NT>::kThreads) expand_kernel(const ExpandParams p)
{
    constexpr int T = Shape<NT>::kThreads, NW = Shape<NT>::kWarps, N8 = NT * 8;
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gr = lane >> 2, tg = lane & 3;
    const int M = p.M;
    const int tpc = p.tiles_per_cta;
    const int tile0 = blockIdx.x * tpc;
    const int ntiles = min(tpc, p.n_out / 16 - tile0);
    const int o0 = 16 * tile0;
    const bool two = p.npaths > 1;
    const int R = p.rank0 + p.rank1;

    uint32_t *const sb0 = reinterpret_cast<uint32_t *>(smem);
    uint32_t *const sb1 = sb0 + 16 * tpc * p.S0 + 4;
    uint16_t *const sh0 = reinterpret_cast<uint16_t *>(sb1 + (two ? 16 * tpc * p.S1 + 4 : 0));
    uint16_t *const sh1 = sh0 + 16 * tpc;
    uint4 *const sz = reinterpret_cast<uint4 *>(sh1 + (two ? 16 * tpc : 0));
    uint4 *const sz1 = sz + 16 * p.kq0 * M;
    float *const sred = reinterpret_cast<float *>(sz1 + (two ? 16 * p.kq1 * M : 0));
    // only with zmode 1: l of both paths and the partial latents
    uint16_t *const sl = reinterpret_cast<uint16_t *>(sred + NW * 16 * N8);  // [R]
    float *const spart = reinterpret_cast<float *>(sl + R);                  // [cs][R][M]

    // (1) this CTA's sign bits of U and its h slice (and l) -> shared memory
    const int rows = 16 * ntiles;
    for (int pp = 0; pp < p.npaths; ++pp) {
        const int64_t ld = pp ? p.u_ld1 : p.u_ld0;
        const uint32_t *u = (pp ? p.u1 : p.u0) + (int64_t)o0 * ld;
        uint32_t *sb = pp ? sb1 : sb0;
        const int S = pp ? p.S1 : p.S0;
        if (!(pp ? p.flat1 : p.flat0)) {
            const int nqr = pp ? p.kq1 : p.kq0;
            for (int r = warp; r < rows; r += NW)
                for (int qq = lane; qq < nqr; qq += 32) cp_async16(sb + r * S + 4 * qq, u + r * ld + 4 * qq);
        } else {
            // rows of a stride that is not a whole number of 16-byte chunks:
            // the CTA's rows are one contiguous block, copied in 16-byte pieces
            const int n16 = rows * (int)ld / 4;
            for (int e = tid; e < n16; e += T) cp_async16(sb + 4 * e, u + 4 * e);
        }
        const uint16_t *h = (pp ? p.h1 : p.h0) + o0;
        if (tid < 2 * ntiles) cp_async16((pp ? sh1 : sh0) + 8 * tid, h + 8 * tid);
    }
    if (p.zmode == 1) {
        for (int e = tid; e < p.rank0 / 8; e += T) cp_async16(sl + 8 * e, p.l0 + 8 * e);
        for (int e = tid; e < p.rank1 / 8; e += T) cp_async16(sl + p.rank0 + 8 * e, p.l1 + 8 * e);
    }
    cp_async_commit();

    // (2) the latent is produced by the previous kernel
    pdl_wait();
    if (p.zmode == 0) {
        // (3a) latent fragments; words past a path's rank are zero
        for (int pp = 0; pp < p.npaths; ++pp) {
            const int n = 16 * (pp ? p.kq1 : p.kq0) * M;
            const int Wp = (pp ? p.rank1 : p.rank0) >> 5;
            const uint4 *src = p.zf + (pp ? p.zoff1 : p.zoff0);
            uint4 *dst = pp ? sz1 : sz;
            for (int e = tid; e < n; e += T) {
                const bool real = e / (4 * M) < Wp;
                cp_async16(dst + e, real ? src + e : src, real ? 16u : 0u);
            }
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
    } else {
        // (3b) partial latents of a split contraction 1: sum them (fixed
        // order), scale by l, build the fp16 fragments
        const int n16 = p.cs * R * M / 4;
        for (int e = tid; e < n16; e += T) cp_async16(spart + 4 * e, p.part + 4 * e);
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        bool overflow = false;
        for (int pp = 0; pp < p.npaths; ++pp) {
            const int n = 16 * (pp ? p.kq1 : p.kq0) * M;
            const int rp = pp ? p.rank1 : p.rank0, kbase = pp ? p.rank0 : 0;
            uint4 *dst = pp ? sz1 : sz;
            for (int e = tid; e < n; e += T) {
                const int t = e & 3, wm = e >> 2;
                const int kw = wm / M, m = wm - kw * M;
                uint32_t v[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float z2[2];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int k = 32 * kw + frag_col(t, 2 * j + hh);
                        float s = 0.f;
                        if (k < rp) {
                            for (int c = 0; c < p.cs; ++c) s += spart[((int64_t)c * R + kbase + k) * M + m];
                            s *= f16_bits_to_float(sl[kbase + k]);
                        }
                        overflow |= beyond_f16(s);
                        z2[hh] = s;
                    }
                    v[j] = pack_half2(z2[0], z2[1]);
                }
                dst[e] = make_uint4(v[0], v[1], v[2], v[3]);
            }
        }
        if (overflow) set_status(p.status, LB_ERR_RANGE);
        __syncthreads();
    }

    // (4) tensor-core contraction, NW / ks tiles at a time
    const int rt_par = NW / p.ks;
    const int tw = warp / p.ks, split = warp - tw * p.ks;
    const int kq0 = p.kq0, KQ = p.kq0 + (two ? p.kq1 : 0);
    const int qa = split * KQ / p.ks, qb = (split + 1) * KQ / p.ks;
    for (int tb = 0; tb < ntiles; tb += rt_par) {
        const int t = tb + tw;
        float acc[NT][4], acc4[3][NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = acc4[0][nt][i] = acc4[1][nt][i] = acc4[2][nt][i] = 0.f;
        if (t < ntiles) {
            const int ro = 16 * t + gr;
            uint32_t hlo0 = sh0[ro], hhi0 = sh0[ro + 8], hlo1 = 0u, hhi1 = 0u;
            hlo0 |= hlo0 << 16;
            hhi0 |= hhi0 << 16;
            if (two) {
                hlo1 = sh1[ro];
                hhi1 = sh1[ro + 8];
                hlo1 |= hlo1 << 16;
                hhi1 |= hhi1 << 16;
            }
            for (int qf = qa; qf < qb; ++qf) {
                const bool sec = qf >= kq0;
                const int qq = sec ? qf - kq0 : qf;
                const int S = sec ? p.S1 : p.S0;
                const uint32_t *bb = (sec ? sb1 : sb0) + ro * S + 4 * qq;
                uint32_t wa[4], wb[4];
                if (!(sec ? p.flat1 : p.flat0)) {
                    const uint4 W0 = *reinterpret_cast<const uint4 *>(bb);
                    const uint4 W1 = *reinterpret_cast<const uint4 *>(bb + 8 * S);
                    wa[0] = W0.x; wa[1] = W0.y; wa[2] = W0.z; wa[3] = W0.w;
                    wb[0] = W1.x; wb[1] = W1.y; wb[2] = W1.z; wb[3] = W1.w;
                } else {
                    // words past the rank read the next row (or the next
                    // buffer); their latent entries are zero
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        wa[i] = bb[i];
                        wb[i] = bb[8 * S + i];
                    }
                }
                const uint32_t hl = sec ? hlo1 : hlo0, hh = sec ? hhi1 : hhi0;
                const uint4 *zp = sec ? sz1 : sz;
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    const int kw = 4 * qq + wi;
                    uint4 Z[NT];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int m = gr + 8 * nt;
                        Z[nt] = m < M ? zp[(kw * M + m) * 4 + tg] : make_uint4(0u, 0u, 0u, 0u);
                    }
                    float(&c0)[NT][4] = (wi & 1) ? acc4[1] : acc;
                    float(&c1)[NT][4] = (wi & 1) ? acc4[2] : acc4[0];
                    uint32_t a0 = signed_pair(hl, wa[wi], 15 - tg), a1 = signed_pair(hh, wb[wi], 15 - tg);
                    uint32_t a2 = signed_pair(hl, wa[wi], 11 - tg), a3 = signed_pair(hh, wb[wi], 11 - tg);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16_16816(c0[nt], a0, a1, a2, a3, Z[nt].x, Z[nt].y);
                    a0 = signed_pair(hl, wa[wi], 7 - tg);
                    a1 = signed_pair(hh, wb[wi], 7 - tg);
                    a2 = signed_pair(hl, wa[wi], 3 - tg);
                    a3 = signed_pair(hh, wb[wi], 3 - tg);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16_16816(c1[nt], a0, a1, a2, a3, Z[nt].z, Z[nt].w);
                }
            }
        }
        if (tb + rt_par >= ntiles) pdl_launch_dependents();
        float *mine = sred + warp * 16 * N8;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = (acc[nt][i] + acc4[0][nt][i]) + (acc4[1][nt][i] + acc4[2][nt][i]);
            const int c = 8 * nt + 2 * tg;
            mine[gr * N8 + c] = v[0];
            mine[gr * N8 + c + 1] = v[1];
            mine[(gr + 8) * N8 + c] = v[2];
            mine[(gr + 8) * N8 + c + 1] = v[3];
        }
        __syncthreads();
        // (5) sum the ks warps of each tile (fixed order) and store bf16 y
        for (int e = tid; e < rt_par * 16 * M; e += T) {
            const int r = e & 15, mt = e >> 4;
            const int m = mt % M, tl = mt / M;
            const int tt = tb + tl;
            if (tt < ntiles) {
                float s = 0.f;
                for (int j = 0; j < p.ks; ++j) s += sred[((tl * p.ks + j) * 16 + r) * N8 + m];
                p.y[(int64_t)m * p.ldy + o0 + 16 * tt + r] = float_to_bf16_bits(s);
            }
        }
        __syncthreads();
    }
}

// ============================================================ planning
struct LatentPlan {
    int rt, cs, groups0, groups, quads, nq_max, cq, S;
    size_t smem;
};
struct ExpandPlan {
    int ks, tiles_per_cta, ctas, S[2], flat[2];
    size_t smem;
};

int nt_of(int M) { return M <= 8 ? 1 : (M <= 16 ? 2 : 4); }
int threads_of(int M) { return nt_of(M) == 4 ? 256 : 512; }

size_t latent_smem(int rt, int S, int cq, int M, int NT, int warps)
{
    return (size_t)16 * rt * S * 4 + (size_t)32 * rt + (size_t)512 * cq + (size_t)512 * cq * M +
           (size_t)256 * cq * M + (size_t)warps * 16 * NT * 8 * 4;
}

// A candidate launch shape for contraction 1: `rt` 16-row tiles per CTA and
// `cs` CTAs splitting n_in; the largest chunk that fits in shared memory.
LatentPlan make_latent_plan(int rt, int cs, int M, int n_in, const int *ranks, int npaths, size_t smem_cap)
{
    LatentPlan lp{};
    const int NT = nt_of(M), warps = threads_of(M) / 32;
    lp.rt = rt;
    lp.cs = cs;
    lp.quads = quads_of(n_in);
    lp.groups0 = (ranks[0] + 16 * rt - 1) / (16 * rt);
    lp.groups = lp.groups0 + (npaths > 1 ? (ranks[1] + 16 * rt - 1) / (16 * rt) : 0);
    lp.nq_max = (lp.quads + cs - 1) / cs;
    lp.S = bit_row_stride(lp.nq_max);
    for (int cq = lp.nq_max; cq >= 1; --cq) {
        const size_t s = latent_smem(rt, lp.S, cq, M, NT, warps);
        if (s <= smem_cap) {
            lp.cq = cq;
            lp.smem = s;
            return lp;
        }
    }
    lp.smem = 0;
    return lp;
}

// Pick the launch shape for contraction 1.  Cost model: the busiest SM runs
// ceil(CTAs / SMs) CTAs (all resident), each costing its sign bits, its share
// of the activation staging, a fixed cost per chunk and per CTA; splitting
// n_in adds the partial-latent traffic of contraction 2.
LatentPlan plan_latent(int M, int n_in, const int *ranks, int npaths, const DeviceInfo &dev)
{
    LatentPlan best{};
    double best_cost = 1e300;
    const int R = ranks[0] + (npaths > 1 ? ranks[1] : 0);
    const int quads = quads_of(n_in);
    const int warps = threads_of(M) / 32;
    for (int rt : {1, 2, 4, 8, 16}) {
        if (rt > warps) continue;
        for (int cs : {1, 2, 3, 4, 6, 8, 12, 16}) {
            if (cs > quads) continue;
            if (cs > 1 && (size_t)cs * R * M * 4 > kMaxPartialBytes) continue;
            const LatentPlan lp = make_latent_plan(rt, cs, M, n_in, ranks, npaths, (size_t)dev.max_smem_optin);
            if (lp.smem == 0) continue;
            const int by_smem = (int)std::min<size_t>(228 * 1024 / (lp.smem + 1024), 8);
            const int per_sm = std::max(1, std::min(by_smem, 2048 / threads_of(M)));
            const long ctas = (long)lp.groups * cs;
            const long slots = (long)dev.sm_count * per_sm;
            const long waves = (ctas + slots - 1) / slots;
            const long per_sm_ctas = (ctas + dev.sm_count - 1) / dev.sm_count;
            const int chunks = (lp.nq_max + lp.cq - 1) / lp.cq;
            const double work = 16.0 * rt * lp.nq_max * 128 + 6.0 * M * lp.nq_max * 128 + 3000.0 * chunks + 4000.0;
            const double cost = (double)per_sm_ctas * work * (double)waves + (cs > 1 ? 2.0 * cs * R * M : 0.0);
            if (cost < best_cost) {
                best_cost = cost;
                best = lp;
            }
        }
    }
    return best;
}

size_t expand_smem(int tiles, const int *S, const int *kq, int npaths, int M, int NT, int warps, int zmode,
                   int cs, int R)
{
    size_t b = 0;
    for (int pp = 0; pp < npaths; ++pp)
        b += (size_t)16 * tiles * S[pp] * 4 + 16 + (size_t)32 * tiles + (size_t)16 * kq[pp] * M * 16;
    b += (size_t)warps * 16 * NT * 8 * 4;
    if (zmode == 1) b += (size_t)2 * R + (size_t)cs * R * M * 4;
    return b;
}

// A candidate launch shape for contraction 2: `ks` warps split the latent, so
// kWarps / ks tiles run at once, `nb` times per CTA.
ExpandPlan make_expand_plan(int ks, int nb, int M, int n_out, const int *ranks, const int64_t *u_ld, int npaths,
                            int zmode, int cs)
{
    ExpandPlan ep{};
    const int NT = nt_of(M), warps = threads_of(M) / 32;
    int kq[2] = {quads_of(ranks[0]), npaths > 1 ? quads_of(ranks[1]) : 0};
    for (int pp = 0; pp < 2; ++pp) {
        ep.flat[pp] = pp < npaths && (u_ld[pp] & 3) != 0;
        ep.S[pp] = pp >= npaths ? 4 : (ep.flat[pp] ? (int)u_ld[pp] : bit_row_stride(kq[pp]));
    }
    ep.ks = ks;
    ep.tiles_per_cta = (warps / ks) * nb;
    ep.ctas = (n_out / 16 + ep.tiles_per_cta - 1) / ep.tiles_per_cta;
    ep.smem = expand_smem(ep.tiles_per_cta, ep.S, kq, npaths, M, NT, warps, zmode, cs,
                          ranks[0] + (npaths > 1 ? ranks[1] : 0));
    return ep;
}

ExpandPlan plan_expand(int M, int n_out, const int *ranks, const int64_t *u_ld, int npaths, int zmode, int cs,
                       const DeviceInfo &dev)
{
    const int KQ = quads_of(ranks[0]) + (npaths > 1 ? quads_of(ranks[1]) : 0);
    const int warps = threads_of(M) / 32;
    ExpandPlan best{};
    double best_cost = 1e300;
    for (int ks : {16, 8, 4, 2, 1}) {
        if (ks > warps) continue;
        const double batch = (double)((KQ + ks - 1) / ks);
        for (int nb = 1; nb <= 256; ++nb) {
            const ExpandPlan ep = make_expand_plan(ks, nb, M, n_out, ranks, u_ld, npaths, zmode, cs);
            if (ep.smem > (size_t)dev.max_smem_optin) break;
            const int by_smem = (int)std::min<size_t>(228 * 1024 / (ep.smem + 1024), 8);
            const int per_sm = std::max(1, std::min(by_smem, 2048 / threads_of(M)));
            const long slots = (long)dev.sm_count * per_sm;
            const long waves = (ep.ctas + slots - 1) / slots;
            const long per_sm_ctas = (ep.ctas + dev.sm_count - 1) / dev.sm_count;
            const double cost =
                (double)per_sm_ctas * (nb * (batch * 512.0 + 1500.0) + 16.0 * KQ * M + 3000.0) * (double)waves;
            if (cost < best_cost) {
                best_cost = cost;
                best = ep;
            }
            if (ep.ctas <= dev.sm_count) break;  // more tiles per CTA only adds work
        }
    }
    return best;
}

// Workspace: the fp16 latent fragments (per path, quads_of(rank) * 4 words x
// M tokens x 4 lane positions x 16 bytes), or the fp32 partial latents of a
// split contraction 1 (at most kMaxPartialBytes).
size_t latent_frag_bytes(int M, const int *ranks, int npaths, int64_t *zoff)
{
    int64_t off = 0;
    for (int pp = 0; pp < npaths; ++pp) {
        if (zoff) zoff[pp] = off;
        off += (int64_t)16 * quads_of(ranks[pp]) * M;
    }
    return (size_t)off * 16;
}

template <int NT>
cudaError_t launch_decode(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    int ranks[2] = {a.path[0].rank, a.npaths > 1 ? a.path[1].rank : 0};
    const LatentPlan lp = plan_latent(M, a.n_in, ranks, a.npaths, dev);
    if (lp.smem == 0) return cudaErrorInvalidConfiguration;
    const int zmode = lp.cs > 1 ? 1 : 0;
    const int64_t u_ld[2] = {a.path[0].u_ld, a.npaths > 1 ? a.path[1].u_ld : 4};
    const ExpandPlan ep = plan_expand(M, a.n_out, ranks, u_ld, a.npaths, zmode, lp.cs, dev);
    if (ep.smem == 0) return cudaErrorInvalidConfiguration;

    LatentParams L{};
    L.x = a.x + (int64_t)m0 * a.ldx;
    L.ldx = a.ldx;
    L.M = M;
    L.n_in = a.n_in;
    L.vt0 = a.path[0].vt_bits;
    L.vt_ld0 = a.path[0].vt_ld;
    L.g0 = a.path[0].g;
    L.l0 = a.path[0].l;
    L.rank0 = a.path[0].rank;
    if (a.npaths > 1) {
        L.vt1 = a.path[1].vt_bits;
        L.vt_ld1 = a.path[1].vt_ld;
        L.g1 = a.path[1].g;
        L.l1 = a.path[1].l;
        L.rank1 = a.path[1].rank;
    }
    L.groups0 = lp.groups0;
    L.rt = lp.rt;
    L.cs = lp.cs;
    L.quads = lp.quads;
    L.cq = lp.cq;
    L.S = lp.S;
    int64_t zoff[2] = {0, 0};
    latent_frag_bytes(M, ranks, a.npaths, zoff);
    L.zf = static_cast<uint4 *>(a.workspace);
    L.zoff0 = zoff[0];
    L.zoff1 = zoff[1];
    L.part = static_cast<float *>(a.workspace);
    L.status = dev.status;

    ExpandParams E{};
    E.zmode = zmode;
    E.zf = static_cast<const uint4 *>(a.workspace);
    E.zoff0 = zoff[0];
    E.zoff1 = zoff[1];
    E.part = static_cast<const float *>(a.workspace);
    E.cs = lp.cs;
    E.l0 = a.path[0].l;
    E.l1 = a.npaths > 1 ? a.path[1].l : nullptr;
    E.M = M;
    E.n_out = a.n_out;
    E.npaths = a.npaths;
    E.u0 = a.path[0].u_bits;
    E.u_ld0 = a.path[0].u_ld;
    E.h0 = a.path[0].h;
    E.rank0 = a.path[0].rank;
    E.kq0 = quads_of(a.path[0].rank);
    E.S0 = ep.S[0];
    E.flat0 = ep.flat[0];
    if (a.npaths > 1) {
        E.u1 = a.path[1].u_bits;
        E.u_ld1 = a.path[1].u_ld;
        E.h1 = a.path[1].h;
        E.rank1 = a.path[1].rank;
        E.kq1 = quads_of(a.path[1].rank);
        E.S1 = ep.S[1];
        E.flat1 = ep.flat[1];
    }
    E.ks = ep.ks;
    E.tiles_per_cta = ep.tiles_per_cta;
    E.y = a.y + (int64_t)m0 * a.ldy;
    E.ldy = a.ldy;
    E.status = dev.status;

    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(lp.groups * lp.cs));
    cfg.blockDim = dim3((unsigned)Shape<NT>::kThreads);
    cfg.dynamicSmemBytes = lp.smem;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, latent_kernel<NT>, L);
    if (err != cudaSuccess) return err;
    cfg.gridDim = dim3((unsigned)ep.ctas);
    cfg.dynamicSmemBytes = ep.smem;
    return cudaLaunchKernelEx(&cfg, expand_kernel<NT>, E);
}

template <int NT>
cudaError_t prepare_nt(const DeviceInfo &dev)
{
    cudaError_t e = cudaFuncSetAttribute(latent_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         dev.max_smem_optin);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(expand_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                dev.max_smem_optin);
}

}  // namespace

cudaError_t decode_prepare_device(const DeviceInfo &dev)
{
    cudaError_t e = small_prepare_device(dev);
    if (e == cudaSuccess) e = mid_prepare_device(dev);
    if (e == cudaSuccess) e = prepare_nt<1>(dev);
    if (e == cudaSuccess) e = prepare_nt<2>(dev);
    if (e == cudaSuccess) e = prepare_nt<4>(dev);
    return e;
}

size_t decode_workspace_bytes(int tokens, int n_in, int n_out, const int *ranks, int npaths)
{
    (void)n_in;
    (void)n_out;
    const int M = std::min(tokens, kDecodeMaxTokens);
    const size_t mma = std::max(latent_frag_bytes(M, ranks, npaths, nullptr), kMaxPartialBytes);
    return std::max(std::max(mma, mid_workspace_bytes(M, ranks, npaths)),
                    small_workspace_bytes(std::min(M, kSmallMaxTokens), ranks, npaths));
}

cudaError_t decode_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    for (int m0 = 0; m0 < a.tokens; m0 += kDecodeMaxTokens) {
        const int M = std::min(kDecodeMaxTokens, a.tokens - m0);
        cudaError_t e;
        const int ranks[2] = {a.path[0].rank, a.npaths > 1 ? a.path[1].rank : 0};
        if (M <= kSmallMaxTokens && small_fits(M, a.n_in, a.n_out, ranks, a.npaths, dev))
            e = small_forward(a, dev, stream, m0, M);
        else if (M <= kMidMaxTokens) e = mid_forward(a, dev, stream, m0, M);
        else if (M <= 8) e = launch_decode<1>(a, dev, stream, m0, M);
        else if (M <= 16) e = launch_decode<2>(a, dev, stream, m0, M);
        else e = launch_decode<4>(a, dev, stream, m0, M);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lb
