// lb_gemv.cu - the forward pass for 1..4 tokens, on CUDA cores.
//
// The layer (sesamedisk.com, "Samsung LittleBit 13B Model", section "What the
// method actually computes", Proposition 1), per path p:
//     z_p = l_p (.) (sign(V_p)^T (g_p (.) x))         contraction 1 (latent)
//     y   = sum_p h_p (.) (sign(U_p) z_p)             contraction 2 (expand)
//
// With a handful of tokens both contractions are sign-matrix x vector
// products, and the register tensor-core path spends most of its time
// rebuilding MMA operands from bits.  Here each 4-bit group (a nibble) of a
// packed row selects one of 16 precomputed signed sums:
//     for columns c .. c+3 with values v_c .. v_c+3 (v = g (.) x, or v = z),
//     T[nibble][p] = sum_j (bit j of p ? -v_{c+j} : +v_{c+j}),  p = 0..15.
// A table row is built once per CTA and shared by every row of the factor the
// CTA handles, so a row costs one shared-memory lookup and one fp32 add per 4
// sign bits.  Tables hold 64 bytes per nibble: the 32 lanes of a warp (32
// different rows) read at most 16 distinct words of 16 distinct banks, so a
// lookup is one wavefront.  Everything stays fp32 until y is rounded to bf16.
//
// Launch structure, data movement and the dependent-launch protocol are the
// same as the tensor-core kernels (lb_decode.cu): weights are copied
// asynchronously at entry, activations after the dependency wait, and the
// dependent kernel is released after the main loop.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"

namespace lb {
namespace {

constexpr int kT = 512;           // threads per CTA
constexpr int kNW = kT / 32;      // warps per CTA
constexpr int kMaxChunkWords = 64;
constexpr size_t kMaxPartialBytes = 96 * 1024;
// A nibble table is 16 floats, stored 20 floats (80 bytes) apart: the 16-byte
// stores of consecutive threads building consecutive tables then start in 8
// different bank groups, and a lookup still reads one 64-byte table.
constexpr int kTab = 20;

__host__ __device__ __forceinline__ int quads_of_words(int w) { return (w + 3) / 4; }
// Row stride in words for bit rows that 16-byte copies fill: a multiple of 4
// whose quad count is odd (lanes reading 32 consecutive rows then hit 8
// different bank groups).
__host__ __device__ __forceinline__ int row_stride(int words) { return 4 * (quads_of_words(words) | 1); }

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

// ============================================================ contraction 1
struct SmallLatentParams {
    const uint16_t *x;
    int64_t ldx;
    int M, n_in;
    const uint32_t *vt0, *vt1;
    int64_t vt_ld0, vt_ld1;
    const uint16_t *g0, *g1, *l0, *l1;
    int rank0, rank1;
    int groups0;  // row groups of path 0 (path 1's follow)
    int rg;       // 32-row groups per CTA
    int cs;       // CTAs splitting n_in (> 1: fp32 partials, l applied later)
    int quads;    // quads (4 words) of n_in
    int cw;       // words per chunk
    int S;        // smem stride of a bit row, words
    float *z;     // cs == 1: z [rank0 + rank1][M]; cs > 1: partials [cs][rank0 + rank1][M]
};

template <int MT>
__global__ void __launch_bounds__(kT) small_latent_kernel(const SmallLatentParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cs = p.cs;
    const int group = blockIdx.x / cs, split_c = blockIdx.x - group * cs;
    const bool second = group >= p.groups0;
    const int row0 = (second ? group - p.groups0 : group) * 32 * p.rg;
    const int rank = second ? p.rank1 : p.rank0;
    const int rows = min(32 * p.rg, rank - row0);
    const int q0 = split_c * p.quads / cs, q1 = (split_c + 1) * p.quads / cs;
    const int W = p.n_in >> 5;
    const int w0 = 4 * q0;
    const int nw = min(4 * q1, W) - w0;
    const int M = p.M, cw = p.cw;
    const int nch = (nw + cw - 1) / cw;
    const int64_t ld = second ? p.vt_ld1 : p.vt_ld0;
    const uint32_t *vt = (second ? p.vt1 : p.vt0) + (int64_t)row0 * ld + w0;
    const uint16_t *g = (second ? p.g1 : p.g0) + 32 * w0;
    const uint16_t *lsrc = (second ? p.l1 : p.l0) + row0;
    const uint16_t *xb = p.x + 32 * w0;
    const int ccols = 32 * cw;  // columns per chunk

    uint32_t *sbits = reinterpret_cast<uint32_t *>(smem);                    // [32 rg][S]
    uint16_t *lraw = reinterpret_cast<uint16_t *>(sbits + 32 * p.rg * p.S);  // [32 rg]
    uint16_t *graw = lraw + 32 * p.rg;                                       // [2][ccols]
    uint16_t *xraw = graw + 2 * ccols;                                       // [2][M][ccols]
    float4 *tab = reinterpret_cast<float4 *>(xraw + 2 * ccols * M);          // [M][cw][8][kTab / 4]
    float *red = reinterpret_cast<float *>(tab + 8 * cw * M * (kTab / 4));   // [kNW][32][MT]

    // (1) weights, all asynchronous: sign bits, l slice, g of the first chunk
    if ((ld & 3) == 0) {
        const int nqr = (nw + 3) >> 2;
        for (int r = warp; r < rows; r += kNW)
            for (int qq = lane; qq < nqr; qq += 32) cp_async16(sbits + r * p.S + 4 * qq, vt + r * ld + 4 * qq);
    } else {
        for (int r = warp; r < rows; r += kNW)
            for (int w = lane; w < nw; w += 32) cp_async4(sbits + r * p.S + w, vt + r * ld + w);
    }
    if (tid < rows / 8) cp_async16(lraw + 8 * tid, lsrc + 8 * tid);
    auto stage_g = [&](int ch) {
        const int wa = ch * cw, n16 = 4 * (min(nw, wa + cw) - wa);
        uint16_t *dst = graw + (ch & 1) * ccols;
        for (int e = tid; e < n16; e += kT) cp_async16(dst + 8 * e, g + 32 * wa + 8 * e);
    };
    auto stage_x = [&](int ch) {
        const int wa = ch * cw, n16 = 4 * (min(nw, wa + cw) - wa);
        uint16_t *dst = xraw + (ch & 1) * ccols * M;
        for (int m = 0; m < M; ++m)
            for (int e = tid; e < n16; e += kT)
                cp_async16(dst + m * ccols + 8 * e, xb + (int64_t)m * p.ldx + 32 * wa + 8 * e);
    };
    stage_g(0);
    cp_async_commit();

    // (2) x comes from the previous kernel on the stream
    pdl_wait();
    stage_x(0);
    cp_async_commit();

    const int ks_n = kNW / p.rg;  // warps per row group
    const int rgi = warp / ks_n, ks = warp - rgi * ks_n;
    const int row = 32 * rgi + lane;
    const bool active = row < rows;
    const uint32_t *brow = sbits + row * p.S;
    float acc[MT], acc2[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = acc2[m] = 0.f;

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
        // (3) nibble tables of this chunk: v = g (.) x in fp32 (exact: an
        // fp16 times a bf16 fits in 24 bits)
        const int cwn = min(cw, nw - ch * cw);
        const uint16_t *gbuf = graw + (ch & 1) * ccols;
        const uint16_t *xbuf = xraw + (ch & 1) * ccols * M;
        for (int e = tid; e < 8 * cwn * M; e += kT) {
            const int m = e / (8 * cwn), wi = e - m * 8 * cwn;  // wi = 8 * word + nibble
            const int c = 4 * wi;
            const uint2 gq = *reinterpret_cast<const uint2 *>(gbuf + c);
            const uint2 xq = *reinterpret_cast<const uint2 *>(xbuf + m * ccols + c);
            const float v0 = f16_bits_to_float(gq.x & 0xffff) * bf16_bits_to_float(xq.x & 0xffff);
            const float v1 = f16_bits_to_float(gq.x >> 16) * bf16_bits_to_float(xq.x >> 16);
            const float v2 = f16_bits_to_float(gq.y & 0xffff) * bf16_bits_to_float(xq.y & 0xffff);
            const float v3 = f16_bits_to_float(gq.y >> 16) * bf16_bits_to_float(xq.y >> 16);
            nibble_table(v0, v1, v2, v3, tab + (kTab / 4) * (m * 8 * cw + wi));
        }
        __syncthreads();
        // (4) one lookup per 4 sign bits of the row
        if (active) {
            const int wa = ks * cwn / ks_n, wb = (ks + 1) * cwn / ks_n;
            const float *tb = reinterpret_cast<const float *>(tab);
            for (int wl = wa; wl < wb; ++wl) {
                const uint32_t bits = brow[ch * cw + wl];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int nib = (bits >> (4 * i)) & 15;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        const float v = tb[((m * cw + wl) * 8 + i) * kTab + nib];
                        if (i & 1) acc2[m] += v;
                        else acc[m] += v;
                    }
                }
            }
        }
    }
    pdl_launch_dependents();

    // (5) sum the warps of each row group (fixed order); scale by l or keep partial
#pragma unroll
    for (int m = 0; m < MT; ++m) red[(warp * 32 + lane) * MT + m] = acc[m] + acc2[m];
    __syncthreads();
    const int R = p.rank0 + p.rank1;
    for (int e = tid; e < rows * M; e += kT) {
        const int r = e / M, m = e - r * M;
        const int rgr = r >> 5, ln = r & 31;
        float s = 0.f;
        for (int j = 0; j < ks_n; ++j) s += red[((rgr * ks_n + j) * 32 + ln) * MT + m];
        const int kg = (second ? p.rank0 : 0) + row0 + r;
        if (cs == 1) p.z[(int64_t)kg * M + m] = s * f16_bits_to_float(lraw[r]);
        else p.z[((int64_t)split_c * R + kg) * M + m] = s;
    }
}

// ============================================================ contraction 2
struct SmallExpandParams {
    const float *z;  // zmode 0: [R][M] (l applied); 1: partials [cs][R][M]
    int zmode, cs;
    const uint16_t *l0, *l1;
    int M, n_out;
    const uint32_t *u0, *u1;
    int64_t u_ld0, u_ld1;
    const uint16_t *h0, *h1;
    int rank0, rank1, npaths;
    int rg;        // 32-row groups per CTA
    int S0, S1;    // smem stride of a bit row per path, words
    int flat0, flat1;
    uint16_t *y;
    int64_t ldy;
};

template <int MT>
__global__ void __launch_bounds__(kT) small_expand_kernel(const SmallExpandParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int M = p.M;
    const bool two = p.npaths > 1;
    const int R = p.rank0 + p.rank1;
    const int W0 = p.rank0 >> 5, WT = R >> 5;
    const int o0 = blockIdx.x * 32 * p.rg;
    const int rows = min(32 * p.rg, p.n_out - o0);

    uint32_t *const sb0 = reinterpret_cast<uint32_t *>(smem);
    uint32_t *const sb1 = sb0 + 32 * p.rg * p.S0 + 4;
    uint16_t *const sh0 = reinterpret_cast<uint16_t *>(sb1 + (two ? 32 * p.rg * p.S1 + 4 : 0));
    uint16_t *const sh1 = sh0 + 32 * p.rg;
    uint16_t *const sl = sh1 + (two ? 32 * p.rg : 0);                        // [R] (zmode 1)
    float *const zr = reinterpret_cast<float *>(sl + (p.zmode ? R : 0));     // [cs or 1][R][M]
    float4 *const tab = reinterpret_cast<float4 *>(zr + (p.zmode ? p.cs : 1) * R * M);  // [M][WT][8][kTab / 4]
    float *const red = reinterpret_cast<float *>(tab + 8 * WT * M * (kTab / 4));        // [kNW][32][MT]

    // (1) weights: this CTA's rows of U, h and (zmode 1) l, asynchronously
    for (int pp = 0; pp < p.npaths; ++pp) {
        const int64_t ld = pp ? p.u_ld1 : p.u_ld0;
        const uint32_t *u = (pp ? p.u1 : p.u0) + (int64_t)o0 * ld;
        uint32_t *sb = pp ? sb1 : sb0;
        const int S = pp ? p.S1 : p.S0;
        if (!(pp ? p.flat1 : p.flat0)) {
            const int nqr = quads_of_words((pp ? p.rank1 : p.rank0) >> 5);
            for (int r = warp; r < rows; r += kNW)
                for (int qq = lane; qq < nqr; qq += 32) cp_async16(sb + r * S + 4 * qq, u + r * ld + 4 * qq);
        } else {
            const int n16 = rows * (int)ld / 4;  // contiguous block of rows
            for (int e = tid; e < n16; e += kT) cp_async16(sb + 4 * e, u + 4 * e);
        }
        const uint16_t *h = (pp ? p.h1 : p.h0) + o0;
        if (tid < rows / 8) cp_async16((pp ? sh1 : sh0) + 8 * tid, h + 8 * tid);
    }
    if (p.zmode) {
        for (int e = tid; e < p.rank0 / 8; e += kT) cp_async16(sl + 8 * e, p.l0 + 8 * e);
        for (int e = tid; e < p.rank1 / 8; e += kT) cp_async16(sl + p.rank0 + 8 * e, p.l1 + 8 * e);
    }
    cp_async_commit();

    // (2) the latent comes from the previous kernel
    pdl_wait();
    {
        const int n16 = (p.zmode ? p.cs : 1) * R * M / 4;
        for (int e = tid; e < n16; e += kT) cp_async16(zr + 4 * e, p.z + 4 * e);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();

    // (3) nibble tables of the whole latent (both paths); a split contraction
    // 1 left partial sums: add them (fixed order) and scale by l here
    for (int e = tid; e < 8 * WT * M; e += kT) {
        const int m = e / (8 * WT), wi = e - m * 8 * WT;
        const int k = 4 * wi;  // latent index over both paths
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float s = zr[(int64_t)(k + j) * M + m];
            if (p.zmode) {
                for (int c = 1; c < p.cs; ++c) s += zr[((int64_t)c * R + k + j) * M + m];
                s *= f16_bits_to_float(sl[k + j]);
            }
            v[j] = s;
        }
        nibble_table(v[0], v[1], v[2], v[3], tab + (kTab / 4) * (m * 8 * WT + wi));
    }
    __syncthreads();

    // (4) one lookup per 4 sign bits; the two paths accumulate apart (their h differ)
    const int ks_n = kNW / p.rg;
    const int rgi = warp / ks_n, ks = warp - rgi * ks_n;
    const int row = 32 * rgi + lane;
    const bool active = row < rows;
    float a0[MT], a1[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) a0[m] = a1[m] = 0.f;
    if (active) {
        const int wa = ks * WT / ks_n, wb = (ks + 1) * WT / ks_n;
        const float *tb = reinterpret_cast<const float *>(tab);
        for (int w = wa; w < wb; ++w) {
            const bool sec = w >= W0;
            const uint32_t bits = sec ? sb1[row * p.S1 + (w - W0)] : sb0[row * p.S0 + w];
            float s[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) s[m] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int nib = (bits >> (4 * i)) & 15;
#pragma unroll
                for (int m = 0; m < MT; ++m) s[m] += tb[((m * WT + w) * 8 + i) * kTab + nib];
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (sec) a1[m] += s[m];
                else a0[m] += s[m];
            }
        }
    }
    pdl_launch_dependents();
    if (active) {
        const float h0 = f16_bits_to_float(sh0[row]);
        const float h1 = two ? f16_bits_to_float(sh1[row]) : 0.f;
#pragma unroll
        for (int m = 0; m < MT; ++m) red[(warp * 32 + lane) * MT + m] = h0 * a0[m] + h1 * a1[m];
    }
    __syncthreads();
    // (5) sum the warps of each row group (fixed order), store bf16 y
    for (int e = tid; e < rows * M; e += kT) {
        const int m = e / rows, r = e - m * rows;
        const int rgr = r >> 5, ln = r & 31;
        float s = 0.f;
        for (int j = 0; j < ks_n; ++j) s += red[((rgr * ks_n + j) * 32 + ln) * MT + m];
        p.y[(int64_t)m * p.ldy + o0 + r] = float_to_bf16_bits(s);
    }
}

// ============================================================ planning
struct SmallLatentPlan {
    int rg, cs, groups0, groups, quads, cw, S;
    size_t smem;
};
struct SmallExpandPlan {
    int rg, ctas, S[2], flat[2];
    size_t smem;
};

size_t small_latent_smem(int rg, int S, int cw, int M)
{
    const int MT = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
    return (size_t)32 * rg * S * 4 + (size_t)64 * rg + (size_t)128 * cw + (size_t)128 * cw * M +
           (size_t)32 * kTab * cw * M + (size_t)kNW * 32 * MT * 4;
}

SmallLatentPlan make_small_latent_plan(int rg, int cs, int M, int n_in, const int *ranks, int npaths,
                                       size_t smem_cap)
{
    SmallLatentPlan lp{};
    lp.rg = rg;
    lp.cs = cs;
    lp.quads = quads_of_words(n_in / 32);
    lp.groups0 = (ranks[0] + 32 * rg - 1) / (32 * rg);
    lp.groups = lp.groups0 + (npaths > 1 ? (ranks[1] + 32 * rg - 1) / (32 * rg) : 0);
    const int nq_max = (lp.quads + cs - 1) / cs;
    lp.S = row_stride(4 * nq_max);
    for (int cw = std::min(kMaxChunkWords, 4 * nq_max); cw >= 1; --cw) {
        const size_t s = small_latent_smem(rg, lp.S, cw, M);
        if (s <= smem_cap) {
            lp.cw = cw;
            lp.smem = s;
            return lp;
        }
    }
    lp.smem = 0;
    return lp;
}

// Cost model: the busiest SM runs ceil(CTAs / SMs) CTAs; a CTA costs its
// lookups (rows x words x 8), its table builds (words x 8 x M) and a fixed
// amount; splitting n_in adds the partial-latent reads of contraction 2.
SmallLatentPlan plan_small_latent(int M, int n_in, const int *ranks, int npaths, const DeviceInfo &dev)
{
    SmallLatentPlan best{};
    double best_cost = 1e300;
    const int R = ranks[0] + (npaths > 1 ? ranks[1] : 0);
    const int quads = quads_of_words(n_in / 32);
    for (int rg : {1, 2, 4, 8, 16}) {
        for (int cs : {1, 2, 3, 4, 6, 8, 12, 16}) {
            if (cs > quads) continue;
            if (cs > 1 && (size_t)cs * R * M * 4 > kMaxPartialBytes) continue;
            const SmallLatentPlan lp = make_small_latent_plan(rg, cs, M, n_in, ranks, npaths,
                                                              (size_t)dev.max_smem_optin);
            if (lp.smem == 0) continue;
            const long ctas = (long)lp.groups * cs;
            const int per_sm = std::max(1, std::min<int>(228 * 1024 / (int)(lp.smem + 1024), 4));
            const long slots = (long)dev.sm_count * per_sm;
            const long waves = (ctas + slots - 1) / slots;
            const long per_sm_ctas = (ctas + dev.sm_count - 1) / dev.sm_count;
            const double words = 4.0 * ((lp.quads + cs - 1) / cs);
            const double work = 32.0 * rg * words * 8 * M / 16 + words * 8 * M * 2 + 1500.0;
            const double cost = (double)per_sm_ctas * work * (double)waves + (cs > 1 ? 0.5 * cs * R * M : 0.0);
            if (cost < best_cost) {
                best_cost = cost;
                best = lp;
            }
        }
    }
    return best;
}

size_t small_expand_smem(int rg, const int *S, int npaths, int M, int zmode, int cs, int R)
{
    const int MT = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
    size_t b = 0;
    for (int pp = 0; pp < npaths; ++pp) b += (size_t)32 * rg * S[pp] * 4 + 16 + (size_t)64 * rg;
    if (zmode) b += (size_t)2 * R;
    b += (size_t)(zmode ? cs : 1) * R * M * 4;
    b += (size_t)(R / 32) * 8 * 4 * kTab * M;
    b += (size_t)kNW * 32 * MT * 4;
    return b;
}

SmallExpandPlan make_small_expand_plan(int rg, int M, int n_out, const int *ranks, const int64_t *u_ld,
                                       int npaths, int zmode, int cs)
{
    SmallExpandPlan ep{};
    ep.rg = rg;
    ep.ctas = (n_out + 32 * rg - 1) / (32 * rg);
    for (int pp = 0; pp < 2; ++pp) {
        ep.flat[pp] = pp < npaths && (u_ld[pp] & 3) != 0;
        ep.S[pp] = pp >= npaths ? 4 : (ep.flat[pp] ? (int)u_ld[pp] : row_stride(ranks[pp] / 32));
    }
    ep.smem = small_expand_smem(rg, ep.S, npaths, M, zmode, cs, ranks[0] + (npaths > 1 ? ranks[1] : 0));
    return ep;
}

SmallExpandPlan plan_small_expand(int M, int n_out, const int *ranks, const int64_t *u_ld, int npaths, int zmode,
                                  int cs, const DeviceInfo &dev)
{
    SmallExpandPlan best{};
    double best_cost = 1e300;
    const int WT = (ranks[0] + (npaths > 1 ? ranks[1] : 0)) / 32;
    for (int rg : {1, 2, 4, 8, 16}) {
        const SmallExpandPlan ep = make_small_expand_plan(rg, M, n_out, ranks, u_ld, npaths, zmode, cs);
        if (ep.smem > (size_t)dev.max_smem_optin) continue;
        const int per_sm = std::max(1, std::min<int>(228 * 1024 / (int)(ep.smem + 1024), 4));
        const long slots = (long)dev.sm_count * per_sm;
        const long waves = (ep.ctas + slots - 1) / slots;
        const long per_sm_ctas = (ep.ctas + dev.sm_count - 1) / dev.sm_count;
        const double work = 32.0 * rg * WT * 8 * M / 16 + WT * 8.0 * M * 2 + 1500.0;
        const double cost = (double)per_sm_ctas * work * (double)waves;
        if (cost < best_cost) {
            best_cost = cost;
            best = ep;
        }
    }
    return best;
}

template <int MT>
cudaError_t launch_small(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    int ranks[2] = {a.path[0].rank, a.npaths > 1 ? a.path[1].rank : 0};
    const SmallLatentPlan lp = plan_small_latent(M, a.n_in, ranks, a.npaths, dev);
    if (lp.smem == 0) return cudaErrorInvalidConfiguration;
    const int zmode = lp.cs > 1 ? 1 : 0;
    const int64_t u_ld[2] = {a.path[0].u_ld, a.npaths > 1 ? a.path[1].u_ld : 4};
    const SmallExpandPlan ep = plan_small_expand(M, a.n_out, ranks, u_ld, a.npaths, zmode, lp.cs, dev);
    if (ep.smem == 0) return cudaErrorInvalidConfiguration;

    SmallLatentParams L{};
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
    L.rg = lp.rg;
    L.cs = lp.cs;
    L.quads = lp.quads;
    L.cw = lp.cw;
    L.S = lp.S;
    L.z = static_cast<float *>(a.workspace);

    SmallExpandParams E{};
    E.z = static_cast<const float *>(a.workspace);
    E.zmode = zmode;
    E.cs = lp.cs;
    E.l0 = a.path[0].l;
    E.l1 = a.npaths > 1 ? a.path[1].l : nullptr;
    E.M = M;
    E.n_out = a.n_out;
    E.u0 = a.path[0].u_bits;
    E.u_ld0 = a.path[0].u_ld;
    E.h0 = a.path[0].h;
    E.rank0 = a.path[0].rank;
    E.npaths = a.npaths;
    if (a.npaths > 1) {
        E.u1 = a.path[1].u_bits;
        E.u_ld1 = a.path[1].u_ld;
        E.h1 = a.path[1].h;
        E.rank1 = a.path[1].rank;
    }
    E.rg = ep.rg;
    E.S0 = ep.S[0];
    E.S1 = ep.S[1];
    E.flat0 = ep.flat[0];
    E.flat1 = ep.flat[1];
    E.y = a.y + (int64_t)m0 * a.ldy;
    E.ldy = a.ldy;

    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(lp.groups * lp.cs));
    cfg.blockDim = dim3(kT);
    cfg.dynamicSmemBytes = lp.smem;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, small_latent_kernel<MT>, L);
    if (err != cudaSuccess) return err;
    cfg.gridDim = dim3((unsigned)ep.ctas);
    cfg.dynamicSmemBytes = ep.smem;
    return cudaLaunchKernelEx(&cfg, small_expand_kernel<MT>, E);
}

template <int MT>
cudaError_t prepare_mt(const DeviceInfo &dev)
{
    cudaError_t e = cudaFuncSetAttribute(small_latent_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         dev.max_smem_optin);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(small_expand_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                dev.max_smem_optin);
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

cudaError_t small_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    if (M <= 1) return launch_small<1>(a, dev, stream, m0, M);
    if (M <= 2) return launch_small<2>(a, dev, stream, m0, M);
    return launch_small<4>(a, dev, stream, m0, M);
}

}  // namespace lb
