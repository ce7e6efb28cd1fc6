// lb_gemv.cu - the forward pass for 1..4 tokens, on CUDA cores.
//
// The layer (sesamedisk.com, "Samsung LittleBit 13B Model", section "What the
// method actually computes", Proposition 1), per path p:
//     z_p = l_p (.) (sign(V_p)^T (g_p (.) x))         contraction 1 (latent)
//     y   = sum_p h_p (.) (sign(U_p) z_p)             contraction 2 (expand)
//
// With a handful of tokens both contractions are sign-matrix x vector
// products.  Each 4-bit group (a nibble) of a packed row selects one of 16
// precomputed signed sums:
//     for columns c .. c+3 with values v_c .. v_c+3 (v = g (.) x, or v = z),
//     T[nibble][p] = sum_j (bit j of p ? -v_{c+j} : +v_{c+j}),  p = 0..15,
// so a row costs one shared-memory lookup and one fp32 add per 4 sign bits.
// A CTA builds the tables of its columns once; the 32 lanes of a warp are 32
// rows reading the same 16-entry table, so a lookup is one wavefront.
//
// Work split (both kernels): lane = one row of the sign matrix, warp = up to
// 8 consecutive sign words (256 columns) of those 32 rows, held in registers.
// The words are loaded at kernel entry, before the wait for the previous
// kernel's output, so their DRAM latency overlaps the launch, the dependency
// wait and the table build.  Contraction 1 splits n_in across the CTAs of a
// cluster when that gives more CTAs (their fp32 partial latents are summed in
// cluster-rank order through distributed shared memory); contraction 2 gives
// each CTA whole rows of U.  Everything is fp32 until y is rounded to bf16;
// every sum runs in a fixed order.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"

namespace lb {
namespace {

constexpr int kWW = 8;          // sign words per lane at most (256 columns or latent entries)
constexpr int kMaxWarps = 16;   // warps per CTA at most
constexpr size_t kMaxPartialBytes = 96 * 1024;
constexpr int kMaxCluster = 8;  // CTAs splitting n_in: a portable cluster
// A nibble table is 16 floats, stored 20 floats (80 bytes) apart: the 16-byte
// stores of consecutive threads building consecutive tables then start in 8
// different bank groups, and a lookup still reads one 64-byte table.
constexpr int kTab = 20;

// 16 signed sums of 4 values: entry p = sum_j (p >> j & 1 ? -v_j : v_j).
// Complementary patterns get exactly negated values (every step is a sum or
// difference, and IEEE rounding is symmetric), so flipping the sign of a
// latent pair (u_k, v_k) leaves the output bit-identical.
__device__ __forceinline__ void nibble_table(float v0, float v1, float v2, float v3, float4 *dst)
{
    const float a = v0 + v1, b = v0 - v1, c = v2 + v3, d = v2 - v3;
    // bits 1,0 of p pick +a, -b, +b, -a (p & 3 = 0, 1, 2, 3); bits 3,2 pick +c, -d, +d, -c
    dst[0] = make_float4(a + c, c - b, b + c, c - a);
    dst[1] = make_float4(a - d, -b - d, b - d, -a - d);
    dst[2] = make_float4(a + d, d - b, b + d, d - a);
    dst[3] = make_float4(a - c, -b - c, b - c, -a - c);
}

// Words [0, n) of a packed row into registers (n <= kWW); the rest are zero.
__device__ __forceinline__ void load_words(uint32_t (&w)[kWW], const uint32_t *src, int n)
{
    if (n == kWW && (reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
        const uint4 a = ldg_early_v4(src);
        const uint4 b = ldg_early_v4(src + 4);
        w[0] = a.x, w[1] = a.y, w[2] = a.z, w[3] = a.w, w[4] = b.x, w[5] = b.y, w[6] = b.z, w[7] = b.w;
    } else {
#pragma unroll
        for (int j = 0; j < kWW; ++j) w[j] = j < n ? ldg_early_u32(src + j) : 0u;
    }
}

// ============================================================ contraction 1
// One path of the group (all paths read the same x): its 32-row latent
// blocks are blocks blk0 .. of the grid's block sequence, and its latents are
// rows koff .. of z.
struct S1Path {
    const uint32_t *vt;
    int64_t vt_ld;
    const uint16_t *g, *l;
    int blk0, koff;
};
template <int NP>  // path slots: 2 for one layer, 2 kMaxSiblings for a group
struct Small1Params {
    const uint16_t *x;
    int64_t ldx;
    int M, W;  // tokens; words of n_in
    int npaths;
    S1Path path[NP];  // in block order
    int cs;     // CTAs across n_in: one cluster, whose first CTA sums the partials
    int ww;     // words per warp (<= kWW)
    int early;  // release the dependent launch at entry instead of after the lookups
    float *z;   // z [R][M] over all paths, l applied
};

// CTA = 32 latent rows (one path) x (warps * ww) words of n_in.  When n_in is
// split (cs > 1) the cs CTAs of a row block form one thread-block cluster:
// each stores its partial sums into the first CTA's shared memory (distributed
// shared memory), and after one cluster barrier the first CTA adds them in
// cluster-rank order.
template <int MT, int NP>
__global__ void __launch_bounds__(kMaxWarps * 32) small1_kernel(const __grid_constant__ Small1Params<NP> p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nthr = blockDim.x, nwarps = nthr >> 5;
    const int M = p.M;
    const int blk = blockIdx.x / p.cs, split = blockIdx.x - blk * p.cs;
    // the path of this row block, selected field by field from fixed
    // parameter offsets: every load is independent of the block index, so
    // none waits for another before the weight loads can start
    S1Path P = p.path[0];
#pragma unroll
    for (int q = 1; q < NP; ++q)
        if (q < p.npaths && blk >= p.path[q].blk0) P = p.path[q];
    const int row0 = (blk - P.blk0) * 32;  // within the path
    const int cww = nwarps * p.ww;                           // words per CTA
    const int c0 = split * cww, c1 = min(p.W, c0 + cww);
    const int wa = c0 + warp * p.ww;
    const int nwd = max(0, min(c1, wa + p.ww) - wa);

    if (p.cs > 1) cluster_arrive_relaxed();  // waited for before the partials go to the first CTA

    // (1) weights, before the dependency wait: this lane's sign words (row
    // row0 + lane, words wa ..) into registers; the CTA's slice of g and l of
    // its rows into shared memory with asynchronous copies
    uint32_t bw[kWW];
    load_words(bw, P.vt + (int64_t)(row0 + lane) * P.vt_ld + wa, nwd);
    const int ntab = 8 * (c1 - c0);
    float4 *tab = reinterpret_cast<float4 *>(smem);  // [M][cww * 8][kTab / 4]
    float *red = reinterpret_cast<float *>(smem) + (size_t)M * cww * 8 * kTab;  // [warps][32][MT]
    float *part = red + nwarps * 32 * MT;                                       // [cs][32][MT] (first CTA)
    uint16_t *gsm = reinterpret_cast<uint16_t *>(part + kMaxCluster * 32 * MT);  // [cww * 32]
    uint16_t *lsm = gsm + cww * 32;                                              // [32]
    {
        const uint16_t *g = P.g + 32 * c0;
        for (int e = tid; e < 4 * (c1 - c0); e += nthr) cp_async16(gsm + 8 * e, g + 8 * e);
        if (tid < 4) cp_async16(lsm + 8 * tid, P.l + row0 + 8 * tid);
        cp_async_commit();
    }
    if (p.early) pdl_launch_dependents();

    // (2) x comes from the previous kernel: tables of v = g (.) x for the
    // CTA's columns, token-major
    pdl_wait();
    cp_async_wait_all();
    __syncthreads();
    // two tables per thread and pass, with every x load of the pass issued
    // before any of them is used (one L2 round trip per pass)
    for (int t = tid; t < ntab; t += 2 * nthr) {
        const int tt[2] = {t, t + nthr};
        uint2 xq[2][MT];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < M && tt[h] < ntab)
                    xq[h][m] = __ldg(reinterpret_cast<const uint2 *>(p.x + (int64_t)m * p.ldx + 32 * c0 + 4 * tt[h]));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (tt[h] >= ntab) continue;
            const uint2 gw = *reinterpret_cast<const uint2 *>(gsm + 4 * tt[h]);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= M) continue;
                const uint2 xv = xq[h][m];
                const float v0 = f16_bits_to_float(gw.x & 0xffff) * bf16_bits_to_float(xv.x & 0xffff);
                const float v1 = f16_bits_to_float(gw.x >> 16) * bf16_bits_to_float(xv.x >> 16);
                const float v2 = f16_bits_to_float(gw.y & 0xffff) * bf16_bits_to_float(xv.y & 0xffff);
                const float v3 = f16_bits_to_float(gw.y >> 16) * bf16_bits_to_float(xv.y >> 16);
                nibble_table(v0, v1, v2, v3, tab + (kTab / 4) * (m * cww * 8 + tt[h]));
            }
        }
    }
    __syncthreads();

    // (3) one lookup per 4 sign bits; two chains per token
    float acc[MT], acc2[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = acc2[m] = 0.f;
    const float *tb = reinterpret_cast<const float *>(smem) + (size_t)(wa - c0) * 8 * kTab;
#pragma unroll
    for (int j = 0; j < kWW; ++j) {
        if (j < nwd) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int nib = (bw[j] >> (4 * i)) & 15;
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m < M) {
                        const float v = tb[((size_t)m * cww * 8 + j * 8 + i) * kTab + nib];
                        if (i & 1) acc2[m] += v;
                        else acc[m] += v;
                    }
                }
            }
        }
    }
    if (!p.early) pdl_launch_dependents();

    // (4) sum the warps (fixed order), then the CTAs of the cluster (rank
    // order), scale by l
#pragma unroll
    for (int m = 0; m < MT; ++m) red[(warp * 32 + lane) * MT + m] = acc[m] + acc2[m];
    __syncthreads();
    const int kg0 = P.koff + row0;
    if (p.cs > 1) cluster_wait();  // every CTA of the cluster is running
    for (int e = tid; e < 32 * M; e += nthr) {
        const int r = e / M, m = e - r * M;
        float s = 0.f;
        for (int w = 0; w < nwarps; ++w) s += red[(w * 32 + r) * MT + m];
        if (p.cs == 1) p.z[(int64_t)(kg0 + r) * M + m] = s * f16_bits_to_float(lsm[r]);
        else st_shared_cluster_f32(map_shared_rank(part + (split * 32 + r) * MT + m, 0), s);
    }
    if (p.cs > 1) {
        cluster_sync();  // every CTA's partials have reached the first CTA
        if (split == 0) {
            for (int e = tid; e < 32 * M; e += nthr) {
                const int r = e / M, m = e - r * M;
                float s = 0.f;
                for (int c = 0; c < p.cs; ++c) s += part[(c * 32 + r) * MT + m];
                p.z[(int64_t)(kg0 + r) * M + m] = s * f16_bits_to_float(lsm[r]);
            }
        }
    }
}

// ============================================================ contraction 2
// One projection of the group: its rows, its paths' U and h, where its
// latents sit in z, the first CTA of its share of the grid, and its output.
struct S2Proj {
    const uint32_t *u0, *u1;
    int64_t u_ld0, u_ld1;
    const uint16_t *h0, *h1;  // h1 null without a residual path
    int n_out;
    int W0, WT;  // latent words of path 0; of both paths
    int koff;    // first latent row of the projection in z
    int cta0;    // first CTA of the projection
    uint16_t *y;
    int64_t ldy;
};
template <int NQ>  // projection slots: 1 for one layer, kMaxSiblings for a group
struct Small2Params {
    const float *z;  // [R][M] over all paths, l applied
    int M;
    int nproj;
    S2Proj proj[NQ];  // in CTA order
    int ks;     // warps per 32-row block (each takes ww words of the latent)
    int ww;     // latent words per warp (<= kWW)
    int early;  // release the dependent launch at entry instead of after the lookups
};

// CTA = (warps / ks) blocks of 32 output rows of one projection; the ks warps
// of a block split the latent words of the projection's paths (path 0 first).
// Warps past the projection's latent words (a sibling may have fewer) idle.
template <int MT, int NQ>
__global__ void __launch_bounds__(kMaxWarps * 32) small2_kernel(const __grid_constant__ Small2Params<NQ> p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nthr = blockDim.x, nwarps = nthr >> 5;
    const int M = p.M;
    // the projection of this CTA (selected as in contraction 1)
    S2Proj P = p.proj[0];
#pragma unroll
    for (int q = 1; q < NQ; ++q)
        if (q < p.nproj && (int)blockIdx.x >= p.proj[q].cta0) P = p.proj[q];
    const int lc = blockIdx.x - P.cta0;  // CTA within the projection
    const int rb = nwarps / p.ks, rbi = warp / p.ks, kw = warp - rbi * p.ks;
    const int o = (lc * rb + rbi) * 32 + lane;  // output row
    const bool rowok = o < P.n_out;             // whole warps: n_out is a multiple of 32
    const int WT = P.WT, W0 = P.W0;
    const int wa = kw * p.ww;
    const int nwd = rowok ? max(0, min(WT, wa + p.ww) - wa) : 0;

    // (1) this lane's sign words of U (row o, latent words wa ..) and its h
    uint32_t bw[kWW];
    if (wa >= W0 || wa + nwd <= W0) {  // one path
        const bool sec = wa >= W0;
        const uint32_t *src = sec ? P.u1 + (int64_t)o * P.u_ld1 + (wa - W0) : P.u0 + (int64_t)o * P.u_ld0 + wa;
        load_words(bw, nwd > 0 ? src : P.u0, nwd);
    } else {
#pragma unroll
        for (int j = 0; j < kWW; ++j) {
            const int w = wa + j;
            bw[j] = j < nwd ? ldg_early_u32(w < W0 ? P.u0 + (int64_t)o * P.u_ld0 + w
                                                   : P.u1 + (int64_t)o * P.u_ld1 + (w - W0))
                            : 0u;
        }
    }
    float h0 = 0.f, h1 = 0.f;
    if (rowok && kw == 0) {
        h0 = f16_bits_to_float(ldg_early_u16(P.h0 + o));
        if (P.h1) h1 = f16_bits_to_float(ldg_early_u16(P.h1 + o));
    }
    if (p.early) pdl_launch_dependents();

    // (2) the latent comes from the previous kernel: tables of the
    // projection's z over both its paths (path 0 first)
    pdl_wait();
    const int ntab = 8 * WT;
    float4 *tab = reinterpret_cast<float4 *>(smem);  // [M][WT * 8][kTab / 4]
    const float *zp = p.z + (int64_t)P.koff * M;
    // two tables per thread and pass, every z load of the pass issued before
    // any is used; one token reads its 4 latents as one 16-byte load
    for (int e = tid; e < ntab * M; e += 2 * nthr) {
        const int ee[2] = {e, e + nthr};
        float v[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (ee[h] >= ntab * M) continue;
            const int m = ee[h] / ntab, k = 4 * (ee[h] - m * ntab);
            if (MT == 1) {
                const float4 q = __ldg(reinterpret_cast<const float4 *>(zp + k));
                v[h][0] = q.x, v[h][1] = q.y, v[h][2] = q.z, v[h][3] = q.w;
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) v[h][j] = __ldg(zp + (int64_t)(k + j) * M + m);
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (ee[h] >= ntab * M) continue;
            const int m = ee[h] / ntab, t = ee[h] - m * ntab;
            nibble_table(v[h][0], v[h][1], v[h][2], v[h][3], tab + (kTab / 4) * (m * ntab + t));
        }
    }
    __syncthreads();

    // (3) one lookup per 4 sign bits; the paths accumulate apart (their h differ)
    float a0[MT], a1[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) a0[m] = a1[m] = 0.f;
    const float *tb = reinterpret_cast<const float *>(smem) + (size_t)wa * 8 * kTab;
#pragma unroll
    for (int j = 0; j < kWW; ++j) {
        if (j < nwd) {
            float s[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) s[m] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int nib = (bw[j] >> (4 * i)) & 15;
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    if (m < M) s[m] += tb[((size_t)m * ntab + j * 8 + i) * kTab + nib];
            }
            const bool sec = wa + j >= W0;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (sec) a1[m] += s[m];
                else a0[m] += s[m];
            }
        }
    }
    if (!p.early) pdl_launch_dependents();

    // (4) sum the ks warps of each row block (fixed order), apply h, round once
    float *red = reinterpret_cast<float *>(smem) + (size_t)M * ntab * kTab;  // [warps][32][2][MT]
    float *hs = red + (size_t)nwarps * 32 * 2 * MT;                         // [rb][32][2]
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        red[((warp * 32 + lane) * 2 + 0) * MT + m] = a0[m];
        red[((warp * 32 + lane) * 2 + 1) * MT + m] = a1[m];
    }
    if (kw == 0) {
        hs[(rbi * 32 + lane) * 2 + 0] = h0;
        hs[(rbi * 32 + lane) * 2 + 1] = h1;
    }
    __syncthreads();
    for (int e = tid; e < rb * 32 * M; e += nthr) {
        const int r = e & 31, rm = e >> 5, b = rm / M, m = rm - b * M;
        const int oo = (lc * rb + b) * 32 + r;
        if (oo >= P.n_out) continue;
        float s0 = 0.f, s1 = 0.f;
        for (int w = 0; w < p.ks; ++w) {
            const int ww_ = b * p.ks + w;
            s0 += red[((ww_ * 32 + r) * 2 + 0) * MT + m];
            s1 += red[((ww_ * 32 + r) * 2 + 1) * MT + m];
        }
        const float yv = hs[(b * 32 + r) * 2 + 0] * s0 + hs[(b * 32 + r) * 2 + 1] * s1;
        P.y[(int64_t)m * P.ldy + oo] = float_to_bf16_bits(yv);
    }
}

// ============================================================ planning
struct Small1Plan {
    int warps = 0, ww = 0, cs = 0, ctas = 0;
    size_t smem = 0;
};
struct Small2Plan {
    int warps = 0, ks = 0, ww = 0, ctas = 0;
    size_t smem = 0;
};

size_t small1_smem(int warps, int ww, int M, int MT)
{
    return (size_t)M * warps * ww * 8 * kTab * 4 + (size_t)(warps + kMaxCluster) * 32 * MT * 4 +
           (size_t)warps * ww * 32 * 2 + 64;
}
size_t small2_smem(int warps, int WT, int M, int MT)
{
    return (size_t)M * WT * 8 * kTab * 4 + (size_t)warps * 32 * 2 * MT * 4 + (size_t)warps * 32 * 2 * 4;
}

// Contraction 1: the most warps per CTA (fewest CTAs per cluster, at most 8)
// that still gives at least one CTA per SM; 8 words per warp unless that
// leaves SMs idle.
Small1Plan plan_small1(int M, int MT, int n_in, int R, const DeviceInfo &dev)
{
    const int W = n_in / 32, blocks = R / 32;
    Small1Plan best;
    for (int ww : {8, 4, 2}) {
        for (int warps : {16, 8, 4, 2, 1}) {
            Small1Plan pl;
            pl.warps = warps;
            pl.ww = ww;
            pl.cs = (W + warps * ww - 1) / (warps * ww);
            if (warps * ww >= W + ww) continue;  // every CTA would have an idle warp
            if (pl.cs > kMaxCluster) continue;
            pl.smem = small1_smem(warps, ww, M, MT);
            if (pl.smem > (size_t)dev.max_smem_optin) continue;
            pl.ctas = blocks * pl.cs;
            if (pl.ctas >= dev.sm_count) return pl;
            if (pl.ctas > best.ctas) best = pl;
        }
    }
    return best;
}

// Contraction 2: ks warps cover a row's latent words (8 per warp, fewer if
// the row's words would need more than kMaxWarps warps; sized for the
// projection with the widest latent).  Row blocks per CTA: at one token, as
// many as fit in kMaxWarps warps while the grid keeps at least 64 CTAs (or
// one per row block): fewer, fuller CTAs build the tables of z fewer times,
// measured 6.0 us per call against 6.7 at Llama-2-7B q_proj (64 CTAs of 16
// warps against 128 of 8) and 6.7 against 7.2 at 70B down_proj, and the same
// choice as before at the gate/up shapes.  At 2-4 tokens (tables per token),
// as many as keep one CTA per SM.  A CTA's row blocks belong to one projection.
Small2Plan plan_small2(int M, int MT, const GroupArgs &g, const DeviceInfo &dev)
{
    int WT = 0, blocks = 0;
    for (int j = 0; j < g.nproj; ++j) {
        WT = std::max(WT, (g.proj[j].path[0].rank + (g.proj[j].npaths > 1 ? g.proj[j].path[1].rank : 0)) / 32);
        blocks += g.proj[j].n_out / 32;
    }
    const int min_ctas = M == 1 ? std::min(64, blocks) : dev.sm_count;
    Small2Plan best;
    for (int ww : {8, 4, 2}) {
        const int ks = (WT + ww - 1) / ww;
        if (ks > kMaxWarps) continue;
        for (int rb : {8, 4, 2, 1}) {
            if (ks * rb > kMaxWarps) continue;
            Small2Plan pl;
            pl.warps = ks * rb;
            pl.ks = ks;
            pl.ww = ww;
            pl.ctas = 0;
            for (int j = 0; j < g.nproj; ++j) pl.ctas += (g.proj[j].n_out / 32 + rb - 1) / rb;
            pl.smem = small2_smem(pl.warps, WT, M, MT);
            if (pl.smem > (size_t)dev.max_smem_optin) continue;
            if (pl.ctas >= min_ctas) return pl;
            if (pl.ctas > best.ctas) best = pl;
        }
    }
    return best;
}

int group_rank(const GroupArgs &g)
{
    int R = 0;
    for (int j = 0; j < g.nproj; ++j)
        for (int q = 0; q < g.proj[j].npaths; ++q) R += g.proj[j].path[q].rank;
    return R;
}

// NP / NQ: path and projection slots of the kernels (a single layer takes the
// kernels with 2 and 1, whose parameter blocks and selection code are the
// smallest; a group takes 2 kMaxSiblings and kMaxSiblings).
template <int MT, int NP, int NQ>
cudaError_t launch_small(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    const int R = group_rank(g);
    const Small1Plan p1 = plan_small1(M, MT, g.n_in, R, dev);
    if (p1.ctas == 0) return cudaErrorInvalidConfiguration;
    const Small2Plan p2 = plan_small2(M, MT, g, dev);
    if (p2.ctas == 0) return cudaErrorInvalidConfiguration;

    // the latent of every path of every projection, in projection order
    Small1Params<NP> L{};
    L.x = g.x + (int64_t)m0 * g.ldx;
    L.ldx = g.ldx;
    L.M = M;
    L.W = g.n_in / 32;
    Small2Params<NQ> E{};
    E.z = static_cast<const float *>(g.workspace);
    E.M = M;
    E.nproj = g.nproj;
    int koff = 0, cta0 = 0;
    const int rb = p2.warps / p2.ks;
    for (int j = 0; j < g.nproj; ++j) {
        const ProjDesc &pj = g.proj[j];
        S2Proj &e = E.proj[j];
        e.u0 = pj.path[0].u_bits;
        e.u_ld0 = pj.path[0].u_ld;
        e.h0 = pj.path[0].h;
        if (pj.npaths > 1) {
            e.u1 = pj.path[1].u_bits;
            e.u_ld1 = pj.path[1].u_ld;
            e.h1 = pj.path[1].h;
        }
        e.n_out = pj.n_out;
        e.W0 = pj.path[0].rank / 32;
        e.WT = e.W0 + (pj.npaths > 1 ? pj.path[1].rank / 32 : 0);
        e.koff = koff;
        e.cta0 = cta0;
        e.y = pj.y + (int64_t)m0 * pj.ldy;
        e.ldy = pj.ldy;
        cta0 += (pj.n_out / 32 + rb - 1) / rb;
        for (int q = 0; q < pj.npaths; ++q) {
            S1Path &v = L.path[L.npaths++];
            v.vt = pj.path[q].vt_bits;
            v.vt_ld = pj.path[q].vt_ld;
            v.g = pj.path[q].g;
            v.l = pj.path[q].l;
            v.blk0 = koff / 32;
            v.koff = koff;
            koff += pj.path[q].rank;
        }
    }
    L.cs = p1.cs;
    L.ww = p1.ww;
    L.early = 0;
    L.z = static_cast<float *>(g.workspace);
    E.ks = p2.ks;
    E.ww = p2.ww;
    // Releasing the next kernel on the stream (the next layer's contraction
    // 1) at entry overlaps its weight loads with this kernel, but its CTAs
    // then compete for SMs: measured faster when this grid is light (at most
    // 8 warps per SM), slower when it is not.
    E.early = (int64_t)p2.ctas * p2.warps <= 8 * (int64_t)dev.sm_count ? 1 : 0;

    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)p1.cs;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)p1.ctas);
    cfg.blockDim = dim3((unsigned)(32 * p1.warps));
    cfg.dynamicSmemBytes = p1.smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = p1.cs > 1 ? 2 : 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, small1_kernel<MT, NP>, L);
    if (err != cudaSuccess) return err;
    cfg.gridDim = dim3((unsigned)p2.ctas);
    cfg.blockDim = dim3((unsigned)(32 * p2.warps));
    cfg.dynamicSmemBytes = p2.smem;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, small2_kernel<MT, NQ>, E);
}

template <int MT>
cudaError_t prepare_mt(const DeviceInfo &dev)
{
    const int sm = dev.max_smem_optin;
    cudaError_t e = cudaFuncSetAttribute(small1_kernel<MT, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(small1_kernel<MT, 2 * kMaxSiblings>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(small2_kernel<MT, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(small2_kernel<MT, kMaxSiblings>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    return e;
}

template <int MT>
cudaError_t launch_small_mt(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    return g.nproj == 1 ? launch_small<MT, 2, 1>(g, dev, stream, m0, M)
                        : launch_small<MT, 2 * kMaxSiblings, kMaxSiblings>(g, dev, stream, m0, M);
}

}  // namespace

cudaError_t small_prepare_device(const DeviceInfo &dev)
{
    cudaError_t e = prepare_mt<1>(dev);
    if (e == cudaSuccess) e = prepare_mt<2>(dev);
    if (e == cudaSuccess) e = prepare_mt<4>(dev);
    return e;
}

size_t small_workspace_bytes(int M, const GroupArgs &g)
{
    return std::max((size_t)group_rank(g) * (size_t)M * 4, kMaxPartialBytes);
}

bool small_fits(int M, const GroupArgs &g, const DeviceInfo &dev)
{
    const int MT = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
    const Small1Plan p1 = plan_small1(M, MT, g.n_in, group_rank(g), dev);
    return p1.ctas > 0 && plan_small2(M, MT, g, dev).ctas > 0;
}

cudaError_t small_forward(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    if (M <= 1) return launch_small_mt<1>(g, dev, stream, m0, M);
    if (M <= 2) return launch_small_mt<2>(g, dev, stream, m0, M);
    return launch_small_mt<4>(g, dev, stream, m0, M);
}

}  // namespace lb
