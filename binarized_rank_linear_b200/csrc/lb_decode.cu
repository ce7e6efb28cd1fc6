// lb_decode.cu - the forward pass for 1..32 tokens.
//
// The layer (sesamedisk.com, "Samsung LittleBit 13B Model", section "What the
// method actually computes", Proposition 1), per path p:
//     z_p = l_p (.) (sign(V_p)^T (g_p (.) x))         contraction 1 (latent)
//     y   = sum_p h_p (.) (sign(U_p) z_p)             contraction 2 (expand)
// Both paths of residual compensation run in the same two launches.
//
// Design.  At batch 1 the layer is a stream of packed sign bits (2-3 MB for
// the Llama-2 shapes), so the kernels are built around moving those bits once
// and spending as few instructions per bit as possible:
//
//  * Every factor entry is +-1 times a scale that the pages give in FP16.  A
//    sign bit is turned into an fp16 operand +-s with two integer ops (shift
//    the bit pair into the fp16 sign positions, XOR it onto the packed scale
//    pair), and the products run on the register tensor cores
//    (mma.m16n8k16, fp16 x fp16 -> fp32).  In contraction 1 the A operand is
//    +-g_i and the B operand is x in fp16; in contraction 2 it is +-h_o and
//    z in fp16.  Both scale operands are exact, the products are exact in
//    fp32, so the only roundings are the fp32 sums, z -> fp16 and y -> bf16.
//    Activations in fp16 follow the page ("activations X stay in FP16").
//  * The packed layout is plain (column 32w + j at bit j of word w).  The
//    MMA's k index is mapped to columns so that a lane's two k values of one
//    A register are columns c and c + 16 of a word: one shift puts both bits
//    at the fp16 sign positions (bits 15 and 31).  The B operand is stored in
//    shared memory in the same column order.  The contraction is invariant to
//    this permutation of k, so nothing else changes.
//  * Contraction 1 splits n_in across the CTAs of a thread-block cluster and
//    sums their partial latents through distributed shared memory in a fixed
//    order (deterministic, no atomics).  The latent (<= 256 KB at 32 tokens)
//    goes to the workspace in the exact fragment order contraction 2 loads,
//    so it stays in L2 between the kernels.
//  * The two kernels are chained with programmatic dependent launch: each
//    starts by issuing the asynchronous copies of its own sign bits (which do
//    not depend on the previous kernel), then waits on the dependency, so the
//    weight stream of one kernel overlaps the tail of the one before it.
#include <algorithm>
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"

namespace lb {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// A 16-byte fragment holds 8 fp16 values of 32 consecutive columns for the
// lane quad position tg: halves 0..7 are columns tg, tg+16, tg+4, tg+20,
// tg+8, tg+24, tg+12, tg+28.  Register j (halves 2j, 2j+1) is one MMA B
// register: j = 0, 1 for the k-step over columns {0..7, 16..23}, j = 2, 3 for
// the k-step over {8..15, 24..31}.
__device__ __forceinline__ int frag_half_of_col(int c) { return 2 * ((c >> 2) & 3) + (c >> 4); }

// +-scale pair from a packed scale pair and the two sign bits at positions
// (15 - sh, 31 - sh) of w: shift them to the fp16 sign bits and flip.
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
    const uint32_t *vt[2];
    int64_t vt_ld[2];
    const uint16_t *g[2];
    const uint16_t *l[2];
    int rank[2];
    int groups0;  // row groups of path 0 (path 1's follow)
    int rt;       // 16-row tiles per group (1, 2, 4 or 8); 8 / rt warps per tile
    int quads;    // quads of n_in
    int nq_max;   // largest quad count of one CTA
    int S;        // smem stride of a bit row, words
    uint4 *zf;    // latent fragments (workspace)
    int64_t zoff[2];
    int *status;
};

template <int NT>
__global__ void __launch_bounds__(kThreads) latent_kernel(const LatentParams p)
{
    constexpr int N8 = NT * 8;
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gr = lane >> 2, tg = lane & 3;
    const int cs = (int)cluster_nctarank(), crank = (int)cluster_ctarank();
    const int group = blockIdx.x / cs;
    const int path = group < p.groups0 ? 0 : 1;
    const int row0 = (group - (path ? p.groups0 : 0)) * 16 * p.rt;
    const int rows = min(16 * p.rt, p.rank[path] - row0);
    const int q0 = (int)((int64_t)crank * p.quads / cs);
    const int q1 = (int)((int64_t)(crank + 1) * p.quads / cs);
    const int nq = q1 - q0;
    const int W = p.n_in >> 5;
    const int w0 = 4 * q0;
    const int nw = min(4 * q1, W) - w0;
    const int M = p.M;

    uint32_t *sbits = reinterpret_cast<uint32_t *>(smem);                 // [16 rt][S]
    uint4 *sg = reinterpret_cast<uint4 *>(sbits + 16 * p.rt * p.S);       // [4 nq][4]
    uint4 *sx = sg + 16 * p.nq_max;                                       // [4 nq][M][4]
    float *sred = reinterpret_cast<float *>(sx + 16 * p.nq_max * M);      // [warps][16][N8]
    float *scta = sred + kWarps * 16 * N8;                                // [16 rt][N8]

    pdl_launch_dependents();

    // (1) this CTA's sign bits -> shared memory, asynchronously
    {
        const uint32_t *vt = p.vt[path] + (int64_t)row0 * p.vt_ld[path] + w0;
        const int64_t ld = p.vt_ld[path];
        if ((ld & 3) == 0) {
            const int nqr = (nw + 3) >> 2;
            for (int e = tid; e < rows * nqr; e += kThreads) {
                const int r = e / nqr, qq = e - r * nqr;
                cp_async16(sbits + r * p.S + 4 * qq, vt + r * ld + 4 * qq);
            }
        } else {
            for (int e = tid; e < rows * nw; e += kThreads) {
                const int r = e / nw, w = e - r * nw;
                cp_async4(sbits + r * p.S + w, vt + r * ld + w);
            }
        }
        cp_async_commit();
    }

    // (2) packed g pairs in fragment order (weights: before the dependency)
    {
        const uint16_t *g = p.g[path];
        for (int e = tid; e < 16 * nq; e += kThreads) {
            const int wl = e >> 2, t = e & 3, w = w0 + wl;
            uint32_t v[4] = {0u, 0u, 0u, 0u};
            if (w < W) {
                const uint16_t *gw = g + 32 * w;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    v[j] = (uint32_t)gw[t + 4 * j] | ((uint32_t)gw[t + 4 * j + 16] << 16);
            }
            sg[e] = make_uint4(v[0], v[1], v[2], v[3]);
        }
    }

    // (3) x is produced by the previous kernel on the stream
    pdl_wait();

    // (4) x -> fp16 fragments
    {
        bool overflow = false;
        for (int e = tid; e < 4 * nq * M; e += kThreads) {
            const int wl = e / M, m = e - wl * M, w = w0 + wl;
            uint4 out[4] = {};
            if (w < W) {
                const uint4 *xr = reinterpret_cast<const uint4 *>(p.x + (int64_t)m * p.ldx + 32 * w);
                uint32_t raw[16];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 q = __ldcg(xr + v);  // written by the previous kernel: L2, not L1
                    raw[4 * v + 0] = q.x; raw[4 * v + 1] = q.y; raw[4 * v + 2] = q.z; raw[4 * v + 3] = q.w;
                }
                float f[32];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    f[2 * c] = __uint_as_float(raw[c] << 16);
                    f[2 * c + 1] = __uint_as_float(raw[c] & 0xffff0000u);
                }
#pragma unroll
                for (int c = 0; c < 32; ++c) overflow |= beyond_f16(f[c]);
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    out[t] = make_uint4(pack_half2(f[t], f[t + 16]), pack_half2(f[t + 4], f[t + 20]),
                                        pack_half2(f[t + 8], f[t + 24]), pack_half2(f[t + 12], f[t + 28]));
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) sx[(wl * M + m) * 4 + t] = out[t];
        }
        if (overflow) set_status(p.status, LB_ERR_RANGE);
    }
    cp_async_wait_all();
    __syncthreads();

    // (5) tensor-core contraction over this CTA's columns
    const int ws = kWarps / p.rt;
    const int tile = warp / ws, split = warp - tile * ws;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    if (16 * tile < rows) {
        const int qa = split * nq / ws, qb = (split + 1) * nq / ws;
        const uint32_t *b0 = sbits + (16 * tile + gr) * p.S;
        const uint32_t *b1 = b0 + 8 * p.S;
        for (int qq = qa; qq < qb; ++qq) {
            const uint4 W0 = *reinterpret_cast<const uint4 *>(b0 + 4 * qq);
            const uint4 W1 = *reinterpret_cast<const uint4 *>(b1 + 4 * qq);
            const uint32_t wa[4] = {W0.x, W0.y, W0.z, W0.w};
            const uint32_t wb[4] = {W1.x, W1.y, W1.z, W1.w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                const int wl = 4 * qq + wi;
                const uint4 G = sg[wl * 4 + tg];
                uint4 X[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int m = gr + 8 * nt;
                    X[nt] = m < M ? sx[(wl * M + m) * 4 + tg] : make_uint4(0u, 0u, 0u, 0u);
                }
                uint32_t a0 = signed_pair(G.x, wa[wi], 15 - tg), a1 = signed_pair(G.x, wb[wi], 15 - tg);
                uint32_t a2 = signed_pair(G.y, wa[wi], 11 - tg), a3 = signed_pair(G.y, wb[wi], 11 - tg);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_f16_16816(acc[nt], a0, a1, a2, a3, X[nt].x, X[nt].y);
                a0 = signed_pair(G.z, wa[wi], 7 - tg);
                a1 = signed_pair(G.z, wb[wi], 7 - tg);
                a2 = signed_pair(G.w, wa[wi], 3 - tg);
                a3 = signed_pair(G.w, wb[wi], 3 - tg);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_f16_16816(acc[nt], a0, a1, a2, a3, X[nt].z, X[nt].w);
            }
        }
    }

    // (6) sum the warps of each tile (fixed order)
    {
        float *mine = sred + warp * 16 * N8;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int c = 8 * nt + 2 * tg;
            mine[gr * N8 + c] = acc[nt][0];
            mine[gr * N8 + c + 1] = acc[nt][1];
            mine[(gr + 8) * N8 + c] = acc[nt][2];
            mine[(gr + 8) * N8 + c + 1] = acc[nt][3];
        }
    }
    __syncthreads();
    for (int e = tid; e < rows * M; e += kThreads) {
        const int r = e / M, m = e - r * M;
        const int t = r >> 4, rr = r & 15;
        float s = 0.f;
        for (int j = 0; j < ws; ++j) s += sred[((t * ws + j) * 16 + rr) * N8 + m];
        scta[r * N8 + m] = s;
    }
    cluster_sync();

    // (7) sum the cluster's CTAs (fixed order), scale by l, store the latent
    {
        const int E = rows * M;
        const int ea = (int)((int64_t)crank * E / cs), eb = (int)((int64_t)(crank + 1) * E / cs);
        const uint16_t *lp = p.l[path];
        bool overflow = false;
        for (int e = ea + tid; e < eb; e += kThreads) {
            const int r = e / M, m = e - r * M;
            float s = 0.f;
            for (int c = 0; c < cs; ++c) s += ld_shared_cluster_f32(map_shared_rank(scta + r * N8 + m, c));
            const int k = row0 + r;
            const float z = s * __half2float(__ushort_as_half(lp[k]));
            overflow |= beyond_f16(z);
            const int kw = k >> 5, cc = k & 31;
            uint16_t *dst = reinterpret_cast<uint16_t *>(p.zf + p.zoff[path] + ((int64_t)kw * M + m) * 4 + (cc & 3));
            dst[frag_half_of_col(cc)] = __half_as_ushort(__float2half_rn(z));
        }
        if (overflow) set_status(p.status, LB_ERR_RANGE);
    }
    cluster_sync();
}

// ============================================================ contraction 2
struct ExpandParams {
    const uint4 *zf;
    int64_t zoff[2];
    int M, n_out;
    const uint32_t *u[2];
    int64_t u_ld[2];
    const uint16_t *h[2];
    int rank[2];
    int npaths;
    int kq[2];  // latent quads per path
    int S[2];   // smem stride of a bit row per path, words
    int ks;     // warps splitting the latent; 8 / ks tiles in flight
    int tiles_per_cta;
    uint16_t *y;
    int64_t ldy;
    int *status;
};

template <int NT>
__global__ void __launch_bounds__(kThreads) expand_kernel(const ExpandParams p)
{
    constexpr int N8 = NT * 8;
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gr = lane >> 2, tg = lane & 3;
    const int M = p.M;
    const int tile0 = blockIdx.x * p.tiles_per_cta;
    const int ntiles = min(p.tiles_per_cta, p.n_out / 16 - tile0);
    const int o0 = 16 * tile0;
    const int npaths = p.npaths;

    uint32_t *const sb0 = reinterpret_cast<uint32_t *>(smem);
    uint32_t *const sb1 = sb0 + 16 * p.tiles_per_cta * p.S[0];
    uint4 *const sz = reinterpret_cast<uint4 *>(sb1 + (npaths > 1 ? 16 * p.tiles_per_cta * p.S[1] : 0));
    uint4 *const sz1 = sz + 16 * p.kq[0] * M;
    float *const sred = reinterpret_cast<float *>(sz1 + (npaths > 1 ? 16 * p.kq[1] * M : 0));

    pdl_launch_dependents();

    // (1) this CTA's sign bits of U -> shared memory, asynchronously
    for (int pp = 0; pp < npaths; ++pp) {
        const int64_t ld = p.u_ld[pp];
        const uint32_t *u = p.u[pp] + (int64_t)o0 * ld;
        const int rows = 16 * ntiles;
        const int W = p.rank[pp] >> 5;
        if ((ld & 3) == 0) {
            const int nqr = p.kq[pp];
            for (int e = tid; e < rows * nqr; e += kThreads) {
                const int r = e / nqr, qq = e - r * nqr;
                cp_async16((pp ? sb1 : sb0) + r * p.S[pp] + 4 * qq, u + r * ld + 4 * qq);
            }
        } else {
            for (int e = tid; e < rows * W; e += kThreads) {
                const int r = e / W, w = e - r * W;
                cp_async4((pp ? sb1 : sb0) + r * p.S[pp] + w, u + r * ld + w);
            }
        }
    }
    cp_async_commit();

    // (2) the latent is produced by the previous kernel
    pdl_wait();

    // (3) latent fragments -> shared memory; padding words past the rank are zero
    for (int pp = 0; pp < npaths; ++pp) {
        const int n = 16 * p.kq[pp] * M;
        const int W = p.rank[pp] >> 5;
        const uint4 *src = p.zf + p.zoff[pp];
        for (int e = tid; e < n; e += kThreads) {
            const int kw = e / (4 * M);
            const bool real = kw < W;
            cp_async16((pp ? sz1 : sz) + e, real ? src + e : src, real ? 16u : 0u);
        }
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();

    // (4) tensor-core contraction, 8 / ks tiles at a time
    const int rt_par = kWarps / p.ks;
    const int tw = warp / p.ks, split = warp - tw * p.ks;
    const int KQ = p.kq[0] + (npaths > 1 ? p.kq[1] : 0);
    const int qa = split * KQ / p.ks, qb = (split + 1) * KQ / p.ks;
    for (int tb = 0; tb < ntiles; tb += rt_par) {
        const int t = tb + tw;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        if (t < ntiles) {
            const int o = o0 + 16 * t + gr;
            uint32_t hlo0, hhi0, hlo1 = 0u, hhi1 = 0u;
            {
                const uint32_t a = p.h[0][o], b = p.h[0][o + 8];
                hlo0 = a | (a << 16);
                hhi0 = b | (b << 16);
            }
            if (npaths > 1) {
                const uint32_t a = p.h[1][o], b = p.h[1][o + 8];
                hlo1 = a | (a << 16);
                hhi1 = b | (b << 16);
            }
            const int kq0 = p.kq[0], S0 = p.S[0], S1 = p.S[1];
            for (int qf = qa; qf < qb; ++qf) {
                const bool second = qf >= kq0;
                const int qq = second ? qf - kq0 : qf;
                const int S = second ? S1 : S0;
                const uint32_t *b0 = (second ? sb1 : sb0) + (16 * t + gr) * S + 4 * qq;
                const uint4 W0 = *reinterpret_cast<const uint4 *>(b0);
                const uint4 W1 = *reinterpret_cast<const uint4 *>(b0 + 8 * S);
                const uint32_t wa[4] = {W0.x, W0.y, W0.z, W0.w};
                const uint32_t wb[4] = {W1.x, W1.y, W1.z, W1.w};
                const uint32_t hl = second ? hlo1 : hlo0, hh = second ? hhi1 : hhi0;
                const uint4 *zp = second ? sz1 : sz;
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    const int kw = 4 * qq + wi;
                    uint4 Z[NT];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int m = gr + 8 * nt;
                        Z[nt] = m < M ? zp[(kw * M + m) * 4 + tg] : make_uint4(0u, 0u, 0u, 0u);
                    }
                    uint32_t a0 = signed_pair(hl, wa[wi], 15 - tg), a1 = signed_pair(hh, wb[wi], 15 - tg);
                    uint32_t a2 = signed_pair(hl, wa[wi], 11 - tg), a3 = signed_pair(hh, wb[wi], 11 - tg);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16_16816(acc[nt], a0, a1, a2, a3, Z[nt].x, Z[nt].y);
                    a0 = signed_pair(hl, wa[wi], 7 - tg);
                    a1 = signed_pair(hh, wb[wi], 7 - tg);
                    a2 = signed_pair(hl, wa[wi], 3 - tg);
                    a3 = signed_pair(hh, wb[wi], 3 - tg);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16_16816(acc[nt], a0, a1, a2, a3, Z[nt].z, Z[nt].w);
                }
            }
        }
        float *mine = sred + warp * 16 * N8;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int c = 8 * nt + 2 * tg;
            mine[gr * N8 + c] = acc[nt][0];
            mine[gr * N8 + c + 1] = acc[nt][1];
            mine[(gr + 8) * N8 + c] = acc[nt][2];
            mine[(gr + 8) * N8 + c + 1] = acc[nt][3];
        }
        __syncthreads();
        // (5) sum the ks warps of each tile (fixed order) and store bf16 y
        for (int e = tid; e < rt_par * 16 * M; e += kThreads) {
            const int r = e & 15, m = (e >> 4) % M, tl = (e >> 4) / M;
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
    int rt, cs, groups0, groups, quads, nq_max, S;
    size_t smem;
};
struct ExpandPlan {
    int ks, tiles_per_cta, ctas, S[2];
    size_t smem;
};

size_t latent_smem(int rt, int nq, int S, int M, int NT)
{
    return (size_t)16 * rt * S * 4 + (size_t)16 * nq * 16 + (size_t)16 * nq * M * 16 +
           (size_t)kWarps * 16 * NT * 8 * 4 + (size_t)16 * rt * NT * 8 * 4;
}

int nt_of(int M) { return M <= 8 ? 1 : (M <= 16 ? 2 : 4); }

// Pick (tiles per CTA, cluster size) for contraction 1.  Cost model: the
// busiest SM runs ceil(CTAs / SMs) CTAs (all CTAs must be resident at once,
// one wave), each costing its sign bits plus its share of the x conversion
// plus a fixed overhead for the reductions.
LatentPlan plan_latent(int M, int n_in, const int *ranks, int npaths, const DeviceInfo &dev)
{
    const int NT = nt_of(M);
    const int quads = quads_of(n_in);
    LatentPlan best{};
    double best_cost = 1e300;
    const int rts[4] = {1, 2, 4, 8}, css[4] = {1, 2, 4, 8};
    for (int rt : rts) {
        int groups0 = (ranks[0] + 16 * rt - 1) / (16 * rt);
        int groups = groups0 + (npaths > 1 ? (ranks[1] + 16 * rt - 1) / (16 * rt) : 0);
        for (int cs : css) {
            if (cs > quads) continue;
            const int nq_max = (quads + cs - 1) / cs;
            const int S = bit_row_stride(nq_max);
            const size_t smem = latent_smem(rt, nq_max, S, M, NT);
            if (smem > (size_t)dev.max_smem_optin) continue;
            int per_sm = (int)std::min<size_t>(227 * 1024 / (smem + 1024), 4);
            if (per_sm < 1) continue;
            const long ctas = (long)groups * cs;
            const long waves = (ctas + (long)dev.sm_count * per_sm - 1) / ((long)dev.sm_count * per_sm);
            const long per_sm_ctas = (ctas + dev.sm_count - 1) / dev.sm_count;
            const double work = 16.0 * rt * nq_max * 128 + 3.0 * M * nq_max * 128 + 4000.0 + 1500.0 * cs;
            const double cost = (double)per_sm_ctas * work * (waves > 1 ? 2.0 : 1.0);
            if (cost < best_cost) {
                best_cost = cost;
                best = LatentPlan{rt, cs, groups0, groups, quads, nq_max, S, smem};
            }
        }
    }
    return best;
}

size_t expand_smem(int tiles, const int *S, const int *kq, int npaths, int M, int NT)
{
    size_t b = 0;
    for (int pp = 0; pp < npaths; ++pp) b += (size_t)16 * tiles * S[pp] * 4 + (size_t)16 * kq[pp] * M * 16;
    return b + (size_t)kWarps * 16 * NT * 8 * 4;
}

ExpandPlan plan_expand(int M, int n_out, const int *ranks, int npaths, const DeviceInfo &dev)
{
    const int NT = nt_of(M);
    int kq[2] = {quads_of(ranks[0]), npaths > 1 ? quads_of(ranks[1]) : 0};
    int S[2] = {bit_row_stride(kq[0]), npaths > 1 ? bit_row_stride(kq[1]) : 4};
    const int KQ = kq[0] + kq[1];
    const int T = n_out / 16;
    ExpandPlan best{};
    double best_cost = 1e300;
    const int kss[4] = {8, 4, 2, 1};
    for (int ks : kss) {
        const int rt_par = kWarps / ks;
        const double batch = (double)((KQ + ks - 1) / ks);
        for (int nb = 1; nb <= 256; ++nb) {
            const int tpc = rt_par * nb;
            const size_t smem = expand_smem(tpc, S, kq, npaths, M, NT);
            if (smem > (size_t)dev.max_smem_optin) break;
            const int per_sm = (int)std::min<size_t>(227 * 1024 / (smem + 1024), 4);
            if (per_sm < 1) break;
            const long ctas = (T + tpc - 1) / tpc;
            const long slots = (long)dev.sm_count * per_sm;
            const long waves = (ctas + slots - 1) / slots;
            const long per_sm_ctas = (ctas + dev.sm_count - 1) / dev.sm_count;
            const double cost = (double)per_sm_ctas * (nb * batch * 512.0 + 16.0 * KQ * M + 3000.0) *
                                (waves > 1 ? 2.0 : 1.0);
            if (cost < best_cost) {
                best_cost = cost;
                best = ExpandPlan{ks, tpc, (int)ctas, {S[0], S[1]}, smem};
            }
            if (ctas <= dev.sm_count) break;  // more tiles per CTA only adds work
        }
    }
    return best;
}

// Workspace layout: per path, quads_of(rank) * 4 latent words x M tokens x 4
// lane positions x 16 bytes.
size_t latent_bytes(int M, const int *ranks, int npaths, int64_t *zoff)
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
    const ExpandPlan ep = plan_expand(M, a.n_out, ranks, a.npaths, dev);
    if (lp.smem == 0 || ep.smem == 0) return cudaErrorInvalidConfiguration;

    LatentParams L{};
    L.x = a.x + (int64_t)m0 * a.ldx;
    L.ldx = a.ldx;
    L.M = M;
    L.n_in = a.n_in;
    for (int pp = 0; pp < a.npaths; ++pp) {
        L.vt[pp] = a.path[pp].vt_bits;
        L.vt_ld[pp] = a.path[pp].vt_ld;
        L.g[pp] = a.path[pp].g;
        L.l[pp] = a.path[pp].l;
        L.rank[pp] = a.path[pp].rank;
    }
    L.groups0 = lp.groups0;
    L.rt = lp.rt;
    L.quads = lp.quads;
    L.nq_max = lp.nq_max;
    L.S = lp.S;
    L.zf = static_cast<uint4 *>(a.workspace);
    latent_bytes(M, ranks, a.npaths, L.zoff);
    L.status = dev.status;

    ExpandParams E{};
    E.zf = static_cast<const uint4 *>(a.workspace);
    E.zoff[0] = L.zoff[0];
    E.zoff[1] = L.zoff[1];
    E.M = M;
    E.n_out = a.n_out;
    E.npaths = a.npaths;
    for (int pp = 0; pp < a.npaths; ++pp) {
        E.u[pp] = a.path[pp].u_bits;
        E.u_ld[pp] = a.path[pp].u_ld;
        E.h[pp] = a.path[pp].h;
        E.rank[pp] = a.path[pp].rank;
        E.kq[pp] = quads_of(a.path[pp].rank);
        E.S[pp] = ep.S[pp];
    }
    E.ks = ep.ks;
    E.tiles_per_cta = ep.tiles_per_cta;
    E.y = a.y + (int64_t)m0 * a.ldy;
    E.ldy = a.ldy;
    E.status = dev.status;

    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = (unsigned)lp.cs;
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = 1;

    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(lp.groups * lp.cs));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = lp.smem;
    cfg.stream = stream;
    cfg.attrs = attrs;
    cfg.numAttrs = 2;
    cudaError_t err = cudaLaunchKernelEx(&cfg, latent_kernel<NT>, L);
    if (err != cudaSuccess) return err;

    cfg.gridDim = dim3((unsigned)ep.ctas);
    cfg.dynamicSmemBytes = ep.smem;
    cfg.numAttrs = 1;
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
    cudaError_t e = prepare_nt<1>(dev);
    if (e == cudaSuccess) e = prepare_nt<2>(dev);
    if (e == cudaSuccess) e = prepare_nt<4>(dev);
    return e;
}

size_t decode_workspace_bytes(int tokens, int n_in, int n_out, const int *ranks, int npaths)
{
    (void)n_in;
    (void)n_out;
    const int M = std::min(tokens, kDecodeMaxTokens);
    return latent_bytes(M, ranks, npaths, nullptr);
}

cudaError_t decode_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    for (int m0 = 0; m0 < a.tokens; m0 += kDecodeMaxTokens) {
        const int M = std::min(kDecodeMaxTokens, a.tokens - m0);
        cudaError_t e;
        if (M <= 8) e = launch_decode<1>(a, dev, stream, m0, M);
        else if (M <= 16) e = launch_decode<2>(a, dev, stream, m0, M);
        else e = launch_decode<4>(a, dev, stream, m0, M);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lb
