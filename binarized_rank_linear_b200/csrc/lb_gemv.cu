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
struct Small1Params {
    const uint16_t *x;
    int64_t ldx;
    int M, W;  // tokens; words of n_in
    const uint32_t *vt0, *vt1;
    int64_t vt_ld0, vt_ld1;
    const uint16_t *g0, *g1, *l0, *l1;
    int rank0, rank1;
    int blocks0;  // 32-row blocks of path 0 (path 1's follow)
    int cs;       // CTAs across n_in: one cluster, whose first CTA sums the partials
    int ww;       // words per warp (<= kWW)
    int early;    // release the dependent launch at entry instead of after the lookups
    float *z;     // z [R][M], l applied
};

// CTA = 32 latent rows (one path) x (warps * ww) words of n_in.  When n_in is
// split (cs > 1) the cs CTAs of a row block form one thread-block cluster:
// each stores its partial sums into the first CTA's shared memory (distributed
// shared memory), and after one cluster barrier the first CTA adds them in
// cluster-rank order.
template <int MT>
__global__ void __launch_bounds__(kMaxWarps * 32) small1_kernel(const Small1Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nthr = blockDim.x, nwarps = nthr >> 5;
    const int M = p.M;
    const int blk = blockIdx.x / p.cs, split = blockIdx.x - blk * p.cs;
    const bool second = blk >= p.blocks0;
    const int row0 = (second ? blk - p.blocks0 : blk) * 32;  // within the path
    const int cww = nwarps * p.ww;                           // words per CTA
    const int c0 = split * cww, c1 = min(p.W, c0 + cww);
    const int wa = c0 + warp * p.ww;
    const int nwd = max(0, min(c1, wa + p.ww) - wa);

    if (p.cs > 1) cluster_arrive_relaxed();  // waited for before the partials go to the first CTA

    // (1) weights, before the dependency wait: this lane's sign words (row
    // row0 + lane, words wa ..) into registers; the CTA's slice of g and l of
    // its rows into shared memory with asynchronous copies
    uint32_t bw[kWW];
    {
        const int64_t ld = second ? p.vt_ld1 : p.vt_ld0;
        load_words(bw, (second ? p.vt1 : p.vt0) + (int64_t)(row0 + lane) * ld + wa, nwd);
    }
    const int ntab = 8 * (c1 - c0);
    float4 *tab = reinterpret_cast<float4 *>(smem);  // [M][cww * 8][kTab / 4]
    float *red = reinterpret_cast<float *>(smem) + (size_t)M * cww * 8 * kTab;  // [warps][32][MT]
    float *part = red + nwarps * 32 * MT;                                       // [cs][32][MT] (first CTA)
    uint16_t *gsm = reinterpret_cast<uint16_t *>(part + kMaxCluster * 32 * MT);  // [cww * 32]
    uint16_t *lsm = gsm + cww * 32;                                              // [32]
    {
        const uint16_t *g = (second ? p.g1 : p.g0) + 32 * c0;
        for (int e = tid; e < 4 * (c1 - c0); e += nthr) cp_async16(gsm + 8 * e, g + 8 * e);
        if (tid < 4) cp_async16(lsm + 8 * tid, (second ? p.l1 : p.l0) + row0 + 8 * tid);
        cp_async_commit();
    }
    if (p.early) pdl_launch_dependents();

    // (2) x comes from the previous kernel: tables of v = g (.) x for the
    // CTA's columns, token-major
    pdl_wait();
    cp_async_wait_all();
    __syncthreads();
    for (int t = tid; t < ntab; t += nthr) {
        const uint2 gw = *reinterpret_cast<const uint2 *>(gsm + 4 * t);
        for (int m = 0; m < M; ++m) {
            const uint2 xq = __ldg(reinterpret_cast<const uint2 *>(p.x + (int64_t)m * p.ldx + 32 * c0 + 4 * t));
            const float v0 = f16_bits_to_float(gw.x & 0xffff) * bf16_bits_to_float(xq.x & 0xffff);
            const float v1 = f16_bits_to_float(gw.x >> 16) * bf16_bits_to_float(xq.x >> 16);
            const float v2 = f16_bits_to_float(gw.y & 0xffff) * bf16_bits_to_float(xq.y & 0xffff);
            const float v3 = f16_bits_to_float(gw.y >> 16) * bf16_bits_to_float(xq.y >> 16);
            nibble_table(v0, v1, v2, v3, tab + (kTab / 4) * (m * cww * 8 + t));
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
    const int kg0 = (second ? p.rank0 : 0) + row0;
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
struct Small2Params {
    const float *z;  // [R][M], l applied
    int M, n_out;
    const uint32_t *u0, *u1;
    int64_t u_ld0, u_ld1;
    const uint16_t *h0, *h1;
    int rank0, rank1;
    int ks;     // warps per 32-row block (each takes ww words of the latent)
    int ww;     // latent words per warp (<= kWW)
    int early;  // release the dependent launch at entry instead of after the lookups
    uint16_t *y;
    int64_t ldy;
};

// CTA = (warps / ks) blocks of 32 output rows; the ks warps of a block split
// the latent words of both paths (path 0 first).
template <int MT>
__global__ void __launch_bounds__(kMaxWarps * 32) small2_kernel(const Small2Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nthr = blockDim.x, nwarps = nthr >> 5;
    const int M = p.M;
    const int rb = nwarps / p.ks, rbi = warp / p.ks, kw = warp - rbi * p.ks;
    const int o = (blockIdx.x * rb + rbi) * 32 + lane;  // output row
    const bool rowok = o < p.n_out;                     // whole warps: n_out is a multiple of 32
    const int R = p.rank0 + p.rank1, WT = R >> 5, W0 = p.rank0 >> 5;
    const int wa = kw * p.ww;
    const int nwd = rowok ? max(0, min(WT, wa + p.ww) - wa) : 0;

    // (1) this lane's sign words of U (row o, latent words wa ..) and its h
    uint32_t bw[kWW];
    if (wa >= W0 || wa + nwd <= W0) {  // one path
        const bool sec = wa >= W0;
        const uint32_t *src = sec ? p.u1 + (int64_t)o * p.u_ld1 + (wa - W0) : p.u0 + (int64_t)o * p.u_ld0 + wa;
        load_words(bw, nwd > 0 ? src : p.u0, nwd);
    } else {
#pragma unroll
        for (int j = 0; j < kWW; ++j) {
            const int w = wa + j;
            bw[j] = j < nwd ? ldg_early_u32(w < W0 ? p.u0 + (int64_t)o * p.u_ld0 + w
                                                   : p.u1 + (int64_t)o * p.u_ld1 + (w - W0))
                            : 0u;
        }
    }
    float h0 = 0.f, h1 = 0.f;
    if (rowok && kw == 0) {
        h0 = f16_bits_to_float(ldg_early_u16(p.h0 + o));
        if (p.h1) h1 = f16_bits_to_float(ldg_early_u16(p.h1 + o));
    }
    if (p.early) pdl_launch_dependents();

    // (2) the latent comes from the previous kernel: tables of z over both
    // paths (path 0 first)
    pdl_wait();
    const int ntab = 8 * WT;
    float4 *tab = reinterpret_cast<float4 *>(smem);  // [M][WT * 8][kTab / 4]
    for (int e = tid; e < ntab * M; e += nthr) {
        const int m = e / ntab, t = e - m * ntab;
        const int k = 4 * t;
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = __ldg(p.z + (int64_t)(k + j) * M + m);
        nibble_table(v[0], v[1], v[2], v[3], tab + (kTab / 4) * (m * ntab + t));
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
        const int oo = (blockIdx.x * rb + b) * 32 + r;
        if (oo >= p.n_out) continue;
        float s0 = 0.f, s1 = 0.f;
        for (int w = 0; w < p.ks; ++w) {
            const int ww_ = b * p.ks + w;
            s0 += red[((ww_ * 32 + r) * 2 + 0) * MT + m];
            s1 += red[((ww_ * 32 + r) * 2 + 1) * MT + m];
        }
        const float yv = hs[(b * 32 + r) * 2 + 0] * s0 + hs[(b * 32 + r) * 2 + 1] * s1;
        p.y[(int64_t)m * p.ldy + oo] = float_to_bf16_bits(yv);
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

// Contraction 2: ks warps cover a row's latent words (8 per warp, 4 if that
// leaves SMs idle); as many row blocks per CTA as keep one CTA per SM.
Small2Plan plan_small2(int M, int MT, int n_out, int R, const DeviceInfo &dev)
{
    const int WT = R / 32, blocks = n_out / 32;
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
            pl.ctas = (blocks + rb - 1) / rb;
            pl.smem = small2_smem(pl.warps, WT, M, MT);
            if (pl.smem > (size_t)dev.max_smem_optin) continue;
            if (pl.ctas >= dev.sm_count) return pl;
            if (pl.ctas > best.ctas) best = pl;
        }
    }
    return best;
}

template <int MT>
cudaError_t launch_small(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    const int R = a.path[0].rank + (a.npaths > 1 ? a.path[1].rank : 0);
    const Small1Plan p1 = plan_small1(M, MT, a.n_in, R, dev);
    if (p1.ctas == 0) return cudaErrorInvalidConfiguration;
    const Small2Plan p2 = plan_small2(M, MT, a.n_out, R, dev);
    if (p2.ctas == 0) return cudaErrorInvalidConfiguration;

    Small1Params L{};
    L.x = a.x + (int64_t)m0 * a.ldx;
    L.ldx = a.ldx;
    L.M = M;
    L.W = a.n_in / 32;
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
    L.blocks0 = a.path[0].rank / 32;
    L.cs = p1.cs;
    L.ww = p1.ww;
    L.early = 0;
    L.z = static_cast<float *>(a.workspace);

    Small2Params E{};
    E.z = static_cast<const float *>(a.workspace);
    E.M = M;
    E.n_out = a.n_out;
    E.u0 = a.path[0].u_bits;
    E.u_ld0 = a.path[0].u_ld;
    E.h0 = a.path[0].h;
    E.rank0 = a.path[0].rank;
    if (a.npaths > 1) {
        E.u1 = a.path[1].u_bits;
        E.u_ld1 = a.path[1].u_ld;
        E.h1 = a.path[1].h;
        E.rank1 = a.path[1].rank;
    }
    E.ks = p2.ks;
    E.ww = p2.ww;
    // Releasing the next kernel on the stream (the next layer's contraction
    // 1) at entry overlaps its weight loads with this kernel, but its CTAs
    // then compete for SMs: measured faster when this grid is light (at most
    // 8 warps per SM), slower when it is not.
    E.early = (int64_t)p2.ctas * p2.warps <= 8 * (int64_t)dev.sm_count ? 1 : 0;
    E.y = a.y + (int64_t)m0 * a.ldy;
    E.ldy = a.ldy;

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
    cudaError_t err = cudaLaunchKernelEx(&cfg, small1_kernel<MT>, L);
    if (err != cudaSuccess) return err;
    cfg.gridDim = dim3((unsigned)p2.ctas);
    cfg.blockDim = dim3((unsigned)(32 * p2.warps));
    cfg.dynamicSmemBytes = p2.smem;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, small2_kernel<MT>, E);
}

template <int MT>
cudaError_t prepare_mt(const DeviceInfo &dev)
{
    cudaError_t e =
        cudaFuncSetAttribute(small1_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, dev.max_smem_optin);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(small2_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, dev.max_smem_optin);
}

}  // namespace

cudaError_t small_prepare_device(const DeviceInfo &dev)
{
    cudaError_t e = prepare_mt<1>(dev);
    if (e == cudaSuccess) e = prepare_mt<2>(dev);
    if (e == cudaSuccess) e = prepare_mt<4>(dev);
    return e;
}

size_t small_workspace_bytes(int M, const int *ranks, int npaths)
{
    const size_t R = (size_t)ranks[0] + (npaths > 1 ? ranks[1] : 0);
    return std::max(R * (size_t)M * 4, kMaxPartialBytes);
}

bool small_fits(int M, int n_in, int n_out, const int *ranks, int npaths, const DeviceInfo &dev)
{
    const int R = ranks[0] + (npaths > 1 ? ranks[1] : 0);
    const int MT = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
    const Small1Plan p1 = plan_small1(M, MT, n_in, R, dev);
    return p1.ctas > 0 && plan_small2(M, MT, n_out, R, dev).ctas > 0;
}

cudaError_t small_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    if (M <= 1) return launch_small<1>(a, dev, stream, m0, M);
    if (M <= 2) return launch_small<2>(a, dev, stream, m0, M);
    return launch_small<4>(a, dev, stream, m0, M);
}

}  // namespace lb
