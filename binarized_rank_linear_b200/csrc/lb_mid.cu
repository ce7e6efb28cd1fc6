// lb_mid.cu - the forward pass for 5..128 tokens, on tcgen05 tensor cores.
//
// The layer (sesamedisk.com, "Samsung LittleBit 13B Model", section "What the
// method actually computes", Proposition 1) as two skinny products in which
// the sign matrix is the 128-row MMA operand and the tokens are the N
// dimension (16, 32, 64 or 128):
//
//   contraction 1:  C1[k, m] = sum_i W1[k, i] x[m, i],  W1[k, i] = sign(V_p[i, k]) g_p[i]   (bf16)
//                   z[m, k]  = l_k C1[k, m], rounded to fp16 (the operand of contraction 2)
//   contraction 2:  C2[o, m] = sum_k W2[o, k] z[m, k],  W2[o, k] = sign(U_p[o, k]) h_p[o]   (fp16)
//                   y[m, o]  = C2[o, m], rounded to bf16
//
// with both paths of residual compensation concatenated (rows of W1, columns
// of W2).  Every sign bit is expanded into shared memory exactly once per
// call, whatever the number of tokens.
//
// A CTA takes one 128-row tile of W and a range of its K-blocks.  The `cs`
// CTAs that split the K-blocks of a tile form a thread-block cluster: each
// sends the rows of its partial accumulator that CTA r finalises to CTA r
// (distributed shared memory), and every CTA adds what it received in
// cluster-rank order, so results do not depend on timing.
//   warp 0      allocates tensor memory, waits for the previous kernel, then
//               streams the token tiles (x or z) with TMA (no multicast)
//   warp 1      one thread issues tcgen05.mma (M = 128, N = 16 .. 128, K = 16)
//   warps 2..9  two groups of 4 taking alternate K-blocks, one W row per
//               thread: expand the row's packed signs into +-scale values in
//               128-byte-swizzled shared memory; warps 2..5 then read the
//               accumulator and finish the tile
// Every wait on an mbarrier is bounded in time; a wait that gives up sets
// LB_ERR_DEVICE_TIMEOUT and the CTA winds down.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"
#include "lb_tc.cuh"

namespace lb {
namespace {

using namespace tc;

constexpr int TM = 128, BK = 64, STAGES = 4;
constexpr int kGroupWarps = 4;                  // one W row per thread: 128 rows
constexpr int kProducerWarps = 2 * kGroupWarps;  // two groups take alternate K-blocks
constexpr int kThreads = 32 * (2 + kProducerWarps);
constexpr int kMaxCluster = 8;
constexpr uint32_t A_BYTES = TM * BK * 2;  // expanded W tile, 16 KB
constexpr uint32_t G_BYTES = 2 * BK * 2;   // a K-block of g for both paths

// NT = token columns of the MMA (16, 32, 64 or 128); the accumulator is read
// out in chunks of CH columns.
template <int NT>
struct MidShape {
    static constexpr int CH = NT < 32 ? NT : 32;
    static constexpr uint32_t kTmemCols = NT < 32 ? 32 : NT;
    static constexpr uint32_t kBBytes = (uint32_t)NT * BK * 2;  // token tile
    // partials received, [cs][128 / cs][kRedStride] fp32: rows padded by 4
    // floats so that 16-byte accesses of consecutive rows cover every bank
    static constexpr int kRedStride = NT + 4;
    static constexpr uint32_t kRedBytes = (uint32_t)TM * kRedStride * 4;
    // per producer warp: two g slots; per producer thread: two 8-byte slots
    // of sign words
    static constexpr size_t kSmem = 1024 + (size_t)STAGES * (A_BYTES + kBBytes) + kRedBytes +
                                    (size_t)kProducerWarps * (2 * G_BYTES + 32 * 8 * 2) + 256;
    static constexpr int kCtasPerSm = 2 * kSmem <= 227 * 1024 ? 2 : 1;
};

// One layer of the call (a group of sibling layers that share x has up to
// kMaxSiblings).  Mode 1 rows are the layer's latents (path 0, then path 1),
// which sit at rows first .. of the group's latent z; mode 2 rows are its
// outputs, in tiles first .. of the grid, reading z columns koff ..
struct MidParams {
    int M;       // tokens (at most NT)
    int rows;    // rows of W: mode 1 R (both paths), mode 2 n_out
    int K;       // mode 1 n_in, mode 2 R
    int r0;      // mode 1: rows [0, r0) are path 0; mode 2: K columns [0, r0) are path 0
    int bits8;   // every K-block's two words of a row can be fetched as one aligned 8-byte load
    const uint32_t *bits0, *bits1;
    int64_t bld0, bld1;       // words per packed row
    const uint16_t *s0, *s1;  // mode 1: g (length K); mode 2: h (length rows)
    const uint16_t *l0, *l1;  // mode 1: latent scale
    int cs;                   // CTAs per tile (cluster size), splitting the K-blocks
    int kpc;                  // K-blocks per CTA
    void *out;                // mode 1: z fp16 [M][ldo]; mode 2: y bf16 [M][ldo]
    int64_t ldo;
    int *status;
    int first;  // mode 1: first row of the layer's latents in z; mode 2: first tile of the layer
    int koff;   // mode 2: first column of the layer's latents in z
};

template <int NQ>  // layer slots: 1 for one layer, kMaxSiblings for a group
struct MidGroup {
    int nlayers;
    // Bounded waits give up after wait_ns.  skip_arrival (a fault-injection
    // hook for tests, lb_debug_inject_stall): the first producer warp of CTA 0
    // does not arrive on its first K-block's stage barrier, so the MMA
    // thread's wait on it runs out and the CTA winds down.
    unsigned long long wait_ns;
    int skip_arrival;
    MidParams layer[NQ];  // in row (mode 1) or tile (mode 2) order
};

// The layer that row nn (mode 1) or tile t (mode 2) belongs to, selected field
// by field from fixed parameter offsets.
template <int NQ>
__device__ __forceinline__ MidParams mid_layer(const MidGroup<NQ> &g, int at)
{
    MidParams p = g.layer[0];
#pragma unroll
    for (int q = 1; q < NQ; ++q)
        if (q < g.nlayers && at >= g.layer[q].first) p = g.layer[q];
    return p;
}

// Finished values of row nn of the tile for the tokens c0 .. c0 + CH - 1:
// mode 1 z[m][nn] = l_nn c (fp16; returns true if a value does not fit),
// mode 2 y[m][nn] (bf16).  A warp's lanes take consecutive rows, so each
// token's stores are contiguous.
template <int MODE, int CH>
__device__ __forceinline__ bool finish_chunk(const MidParams &p, int col, int nn, int c0, const float (&c)[CH])
{
    // col: the output column (mode 1: the latent's row in the group's z; mode
    // 2: nn); nn: the row within the layer
    uint16_t *out = static_cast<uint16_t *>(p.out) + col;
    bool overflow = false;
    if (MODE == 1) {
        const float lv = f16_bits_to_float(nn < p.r0 ? p.l0[nn] : p.l1[nn - p.r0]);
#pragma unroll
        for (int j = 0; j < CH; ++j) {
            if (c0 + j < p.M) {
                const float z = c[j] * lv;
                out[(int64_t)(c0 + j) * p.ldo] = (uint16_t)(pack_half2(z, 0.f) & 0xffffu);
                overflow |= beyond_f16(z);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < CH; ++j)
            if (c0 + j < p.M) out[(int64_t)(c0 + j) * p.ldo] = float_to_bf16_bits(c[j]);
    }
    return overflow;
}

// CH accumulator columns c0 .. of this warp's 32 lanes (zero when the
// accumulator was never written); warp-collective.
template <int CH>
__device__ __forceinline__ void acc_chunk(uint32_t taddr, bool valid, float (&c)[CH])
{
    if (valid) {
        uint32_t v[CH];
        if constexpr (CH == 16) tmem_ld16(taddr, v);
        else tmem_ld32(taddr, v);
#pragma unroll
        for (int j = 0; j < CH; ++j) c[j] = __uint_as_float(v[j]);
    } else {
#pragma unroll
        for (int j = 0; j < CH; ++j) c[j] = 0.f;
    }
}

template <int MODE, int NT, int NQ>
__global__ void __launch_bounds__(kThreads, 2)
    mid_gemm_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ MidGroup<NQ> g)
{
    using S = MidShape<NT>;
    constexpr uint32_t B_BYTES = S::kBBytes;
    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // SW128 tiles need 1024-byte alignment
    const uint32_t sA = base, sB = base + STAGES * A_BYTES;
    const uint32_t sRed = sB + STAGES * B_BYTES;  // partials received from the cluster, [cs][rpr][NT] fp32
    const uint32_t sGbf = sRed + S::kRedBytes;    // mode 1, per producer warp: g in bf16, [warp][2][path][64]
    const uint32_t sRing = sGbf + kProducerWarps * 2 * G_BYTES;  // per producer thread: two sign-word slots
    const uint32_t bars = sRing + kProducerWarps * 32 * 8 * 2;
    // full[STAGES], empty[STAGES], acc_full, drain, then the tmem address
    const uint32_t full0 = bars, empty0 = bars + 8 * STAGES, accf = bars + 16 * STAGES, drain = accf + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + (drain + 8 - raw));
    __shared__ int abort_shared;
    volatile int &abort_flag = abort_shared;

    const int cs = g.layer[0].cs;
    const int tile = blockIdx.x / cs, split = blockIdx.x - tile * cs;  // split = rank in the cluster
    // Mode 2: the CTA's layer and its tile within the layer.  Mode 1: the
    // layer of the tile's first row; only the fields all layers share (M, K,
    // kpc, z) are read from it, as a tile's rows may belong to several layers.
    const MidParams p = mid_layer<NQ>(g, MODE == 1 ? tile * TM : tile);
    const int ltile = MODE == 1 ? tile : tile - p.first;
    const int nk = (p.K + BK - 1) / BK;
    const int kb0 = split * p.kpc, nkb = max(0, min(nk, kb0 + p.kpc) - kb0);
    if (cs > 1) cluster_arrive_relaxed();  // waited for before partials go to other CTAs

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(full0 + 8 * s, 1 + kGroupWarps);  // TMA arrive.expect_tx + one group's warps
                mbar_init(empty0 + 8 * s, 1);               // one tcgen05.commit
            }
            mbar_init(accf, 1);
            mbar_init(drain, 1);
            abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool acc_ok = false;  // warps 2..5: the accumulator is complete and holds this CTA's K-blocks

    if (warp == 0) {
        // ---------------- token tiles (TMA); the tokens come from the previous kernel
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
            pdl_wait();
            int issued = 0;
            for (int j = 0; j < nkb; ++j) {
                const int s = j % STAGES;
                const uint32_t ph = (uint32_t)(j / STAGES) & 1u;
                if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, g.wait_ns) || abort_flag) {
                    abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(full0 + 8 * s, B_BYTES);
                tma_load_2d(sB + s * B_BYTES, &tmB, (MODE == 2 ? p.koff : 0) + (kb0 + j) * BK, 0, full0 + 8 * s);
                ++issued;
            }
            if (abort_flag) {
                for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
                    mbar_wait(full0 + 8 * (j % STAGES), (uint32_t)(j / STAGES) & 1u, g.wait_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = instr_desc(MODE == 1 ? 1u : 0u, TM, NT);
            for (int j = 0; j < nkb; ++j) {
                const int s = j % STAGES;
                const uint32_t ph = (uint32_t)(j / STAGES) & 1u;
                if (!mbar_wait(full0 + 8 * s, ph, g.wait_ns) || abort_flag) {
                    abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = smem_desc(sA + s * A_BYTES), bd = smem_desc(sB + s * B_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)  // +32 bytes along K per step of 16
                    umma(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (j | kk) != 0);
                umma_commit(empty0 + 8 * s);
            }
            umma_commit(accf);
            // every MMA issued has finished before the CTA frees tensor memory
            umma_commit(drain);
            if (!mbar_wait(drain, 0, g.wait_ns)) abort_flag = 1;
        }
    } else {
        // ---------------- producers: group grp expands blocks j = grp, grp + 2, ...
        // of this CTA's K range, one W row per thread; what a block needs from
        // memory (the row's sign words; g in mode 1) comes in by cp.async two
        // of the group's blocks ahead (below)
        const int pw = warp - 2;  // producer warp 0 .. 7
        const int grp = pw >> 2;
        const int row = ((pw & 3) << 5) | lane;  // W row within the tile
        // the layer of this warp's 32 rows (a layer's rows start at a
        // multiple of 32, so they are all in one) and the row within it
        const MidParams w = MODE == 1 ? mid_layer<NQ>(g, tile * TM + 32 * (pw & 3)) : p;
        const int nn = (MODE == 1 ? tile * TM - w.first : ltile * TM) + row;
        const uint32_t x7 = (uint32_t)(row & 7);  // the row's 128-byte swizzle
        const bool row_in = nn < w.rows;
        const bool sec_row = MODE == 1 && nn >= w.r0;  // mode 1: the row's path
        const int kwords = w.K >> 5, r0w = w.r0 >> 5;
        const uint32_t gbfw = sGbf + (uint32_t)pw * 2 * G_BYTES;  // this warp's two bf16 g slots
        const uint32_t *rb0 = nullptr, *rb1 = nullptr;
        uint32_t hs0 = 0u, hs1 = 0u;  // mode 2: h of the row, both paths, both halves
        if (row_in) {
            if (MODE == 1) {
                rb0 = sec_row ? w.bits1 + (int64_t)(nn - w.r0) * w.bld1 : w.bits0 + (int64_t)nn * w.bld0;
            } else {
                rb0 = w.bits0 + (int64_t)nn * w.bld0;
                if (w.bits1) rb1 = w.bits1 + (int64_t)nn * w.bld1;
                const uint32_t h0 = ldg_early_u16(w.s0 + nn), h1 = w.s1 ? ldg_early_u16(w.s1 + nn) : 0u;
                hs0 = h0 | (h0 << 16);
                hs1 = h1 | (h1 << 16);
            }
        }
        auto wp = [&](int w) { return (MODE == 1 || w < r0w) ? rb0 + w : rb1 + (w - r0w); };
        // A block's sign words (and, mode 1, lanes 0..15, its g in fp16) come
        // in by cp.async into slot `slot` of the thread's two-slot ring (and
        // of the warp's two g slots), two of the group's blocks ahead, and are
        // waited for just before use: no register holds a load in flight
        // across blocks (copying one would wait for it).
        constexpr uint32_t RING_STRIDE = (uint32_t)kProducerWarps * 32 * 8;
        const uint32_t ring = sRing + (uint32_t)(pw * 32 + lane) * 8;
        auto copy_block = [&](int j, int slot) {
            if (j < nkb) {
                const int kb = kb0 + j, wd = 2 * kb;
                const uint32_t dst = ring + (uint32_t)slot * RING_STRIDE;
                if (row_in && wd < kwords) {
                    if (w.bits8 && wd + 1 < kwords) {
                        cp_async8(dst, wp(wd));
                    } else {
                        cp_async4(dst, wp(wd));
                        if (wd + 1 < kwords)
                            cp_async4(dst + 4, wp(wd + 1));
                        else
                            asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst + 4), "r"(0u) : "memory");
                    }
                } else {
                    asm volatile("st.shared.v2.u32 [%0], {%1, %1};" ::"r"(dst), "r"(0u) : "memory");
                }
                if (MODE == 1 && lane < 16) {
                    const int pp = lane >> 3, k0 = kb * BK + 8 * (lane & 7);
                    const uint16_t *gs = pp ? w.s1 : w.s0;
                    const uint32_t gdst = gbfw + (uint32_t)slot * G_BYTES + (uint32_t)lane * 16;
                    if (gs != nullptr && k0 < w.K)
                        cp_async16s(gdst, gs + k0);
                    else
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(gdst), "r"(0u) : "memory");
                }
            }
            cp_async_commit();  // one group per block (empty past the end), so the waits count blocks
        };
        copy_block(grp, 0);
        copy_block(grp + 2, 1);
        for (int j = grp, it = 0; j < nkb; j += 2, ++it) {
            const int kb = kb0 + j;
            const int s = j % STAGES;
            const uint32_t ph = (uint32_t)(j / STAGES) & 1u;
            bool ok = mbar_wait(empty0 + 8 * s, ph ^ 1u, g.wait_ns) && !abort_flag;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                abort_flag = 1;
                break;
            }
            // this block's copies have landed (at most one younger group pending)
            cp_async_wait_group<1>();
            const int slot = it & 1;
            uint4 sc[8];  // per chunk: the four packed scale words
            if (MODE == 1) {
                // lanes 0..15 round their 8 values of g to bf16 in place
                const uint32_t gsl = gbfw + (uint32_t)slot * G_BYTES;
                if (lane < 16) {
                    uint32_t w[4];
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                                 : "r"(gsl + (uint32_t)lane * 16)
                                 : "memory");
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        w[q] = pack_bf162(f16_bits_to_float((uint16_t)(w[q] & 0xffffu)), f16_bits_to_float((uint16_t)(w[q] >> 16)));
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(gsl + (uint32_t)lane * 16), "r"(w[0]),
                                 "r"(w[1]), "r"(w[2]), "r"(w[3])
                                 : "memory");
                }
                __syncwarp();
                const uint8_t *gb = smem_raw + (gsl + (sec_row ? BK * 2 : 0) - raw);
#pragma unroll
                for (int q = 0; q < 8; ++q) sc[q] = *reinterpret_cast<const uint4 *>(gb + 16 * q);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int k0 = kb * BK + 8 * q;  // first column of the chunk
                    const uint32_t h = k0 < w.K ? (k0 >= w.r0 ? hs1 : hs0) : 0u;
                    sc[q] = make_uint4(h, h, h, h);
                }
            }
            uint2 bits;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                         : "=r"(bits.x), "=r"(bits.y)
                         : "r"(ring + (uint32_t)slot * RING_STRIDE)
                         : "memory");
            const uint32_t rowx = (sA + s * A_BYTES + row * 128) | (x7 << 4);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                store_sign_chunk(rowx ^ (16u * q), __byte_perm(q < 4 ? bits.x : bits.y, 0u, 0x4440u | (uint32_t)(q & 3)),
                                 sc[q]);
            fence_async_shared();
            __syncwarp();
            if (lane == 0 && !(g.skip_arrival && blockIdx.x == 0 && pw == 0 && j == 0)) mbar_arrive(full0 + 8 * s);
            // refill the slots (used above; every lane is past its reads after
            // the __syncwarp) with the group's block two ahead
            copy_block(j + 4, slot);
        }
        cp_async_wait_all();  // no copy may land after the CTA is gone
        // warps 2..5: this thread's row 32 (warp % 4) + lane of the accumulator
        if (pw < 4) {
            bool ok = !abort_flag && mbar_wait(accf, 0, g.wait_ns);
            ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
            if (!ok) abort_flag = 1;
            tc_fence_after();
            acc_ok = ok && nkb > 0;
        }
    }

    // ---------------- finish: every partial of the tile added in rank order
    pdl_launch_dependents();
    __syncwarp();
    constexpr int CH = S::CH;
    const bool holder = warp >= 2 && warp < 6;  // these warps read accumulator rows 32 (warp % 4) ..
    const uint32_t ta = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    bool overflow = false;
    if (cs == 1) {
        if (holder) {
            pdl_wait();  // y / z may still be in use by the previous kernel
            const int gr = tile * TM + 32 * (warp & 3) + lane;  // the row in the grid (mode 1: in z)
            const MidParams L = MODE == 1 ? mid_layer<NQ>(g, gr) : p;
            const int nn = MODE == 1 ? gr - L.first : ltile * TM + 32 * (warp & 3) + lane;  // within the layer
            for (int c0 = 0; c0 < NT; c0 += CH) {
                float c[CH];
                acc_chunk<CH>(ta + (uint32_t)c0, acc_ok, c);
                if (nn < L.rows) overflow |= finish_chunk<MODE, CH>(L, MODE == 1 ? gr : nn, nn, c0, c);
            }
        }
    } else {
        // CTA r finalises rows r * rpr .. of the tile: every CTA sends it its
        // partials of those rows, then adds what it received
        const int rpr = TM / cs;
        cluster_wait();  // every CTA of the cluster is running
        if (holder) {
            const int rho = 32 * (warp & 3) + lane;
            const int dst = rho / rpr, q = rho - dst * rpr;
            const uint32_t ra = map_shared_addr(sRed + (uint32_t)((split * rpr + q) * S::kRedStride) * 4u, (uint32_t)dst);
            for (int c0 = 0; c0 < NT; c0 += CH) {
                float c[CH];
                acc_chunk<CH>(ta + (uint32_t)c0, acc_ok, c);
#pragma unroll
                for (int j = 0; j < CH; j += 4)
                    st_shared_cluster_v4(ra + 4u * (c0 + j), __float_as_uint(c[j]), __float_as_uint(c[j + 1]),
                                         __float_as_uint(c[j + 2]), __float_as_uint(c[j + 3]));
            }
        }
        cluster_sync();  // every partial has arrived
        pdl_wait();
        const float *red = reinterpret_cast<const float *>(smem_raw + (sRed - raw));
        for (int q = tid; q < rpr; q += kThreads) {  // one row per thread, every token
            const int gr = tile * TM + split * rpr + q;  // the row in the grid (mode 1: in z)
            const MidParams L = MODE == 1 ? mid_layer<NQ>(g, gr) : p;
            const int nn = MODE == 1 ? gr - L.first : ltile * TM + split * rpr + q;  // within the layer
            for (int c0 = 0; c0 < NT; c0 += CH) {
                float c[CH];
#pragma unroll
                for (int j = 0; j < CH; ++j) c[j] = 0.f;
                for (int r = 0; r < cs; ++r) {
                    const float4 *src = reinterpret_cast<const float4 *>(red + (r * rpr + q) * S::kRedStride + c0);
#pragma unroll
                    for (int j4 = 0; j4 < CH / 4; ++j4) {
                        const float4 v = src[j4];
                        c[4 * j4] += v.x;
                        c[4 * j4 + 1] += v.y;
                        c[4 * j4 + 2] += v.z;
                        c[4 * j4 + 3] += v.w;
                    }
                }
                if (nn < L.rows) overflow |= finish_chunk<MODE, CH>(L, MODE == 1 ? gr : nn, nn, c0, c);
            }
        }
    }
    if (overflow) set_status(p.status, LB_ERR_RANGE);

    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) set_status(p.status, LB_ERR_DEVICE_TIMEOUT);
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, S::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
// CTAs per tile: a power of two (each finalises 128 / cs rows of the tile),
// at most a portable cluster, enough to fill the CTA slots (one or two per
// SM, as shared memory allows), and never a CTA without a K-block.
int pick_split(int tiles, int nk, int slots)
{
    const int want = std::max(1, std::min(kMaxCluster, slots / std::max(1, tiles)));
    int cs = 1;
    while (2 * cs <= want && 2 * cs <= nk) cs *= 2;
    while (cs > 1 && (cs - 1) * ((nk + cs - 1) / cs) >= nk) cs /= 2;
    return cs;
}

int layer_rank(const ProjDesc &pj) { return pj.path[0].rank + (pj.npaths > 1 ? pj.path[1].rank : 0); }

// Contraction MODE for the layers of a group, tokens m0 .. m0 + M, the
// latent z fp16 [M][ldz] (token-major, every layer's latents side by side in
// layer order, path 0 first).  Mode 1 covers the latent rows of all layers
// with one grid of 128-row tiles (the K range, n_in, is shared); mode 2 gives
// each layer its own tiles of output rows, reading its columns of z.  One
// split of the K-blocks across a cluster serves every layer; it is chosen
// for the layer with the fewest K-blocks, and a CTA past a longer layer's
// blocks contributes zeros.
template <int MODE, int NT, int NQ>
cudaError_t launch_mid(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream, int m0, int M, const uint16_t *z,
                       int64_t ldz)
{
    MidGroup<NQ> G{};
    G.nlayers = g.nproj;
    G.wait_ns = debug_wait_ns();
    G.skip_arrival = debug_skip_arrival();
    int tiles = 0, nk = 0, koff = 0;
    if (MODE == 1) {
        int R = 0;
        for (int j = 0; j < g.nproj; ++j) R += layer_rank(g.proj[j]);
        tiles = (R + TM - 1) / TM;
        nk = (g.n_in + BK - 1) / BK;
    } else {
        nk = 1 << 30;
        for (int j = 0; j < g.nproj; ++j) {
            tiles += (g.proj[j].n_out + TM - 1) / TM;
            nk = std::min(nk, (layer_rank(g.proj[j]) + BK - 1) / BK);
        }
    }
    const int cs = pick_split(tiles, nk, MidShape<NT>::kCtasPerSm * dev.sm_count);
    int tile0 = 0;
    for (int j = 0; j < g.nproj; ++j) {
        const ProjDesc &pj = g.proj[j];
        const PathDesc &q0 = pj.path[0], &q1 = pj.path[1];
        const bool two = pj.npaths > 1;
        const int R = layer_rank(pj);
        MidParams &L = G.layer[j];
        L.M = M;
        L.r0 = q0.rank;
        L.cs = cs;
        L.status = dev.status;
        if (MODE == 1) {
            L.rows = R;
            L.K = g.n_in;
            L.bits8 = even8(q0.vt_bits, q0.vt_ld) && (!two || even8(q1.vt_bits, q1.vt_ld));
            L.bits0 = q0.vt_bits;
            L.bld0 = q0.vt_ld;
            L.s0 = q0.g;
            L.l0 = q0.l;
            if (two) {
                L.bits1 = q1.vt_bits;
                L.bld1 = q1.vt_ld;
                L.s1 = q1.g;
                L.l1 = q1.l;
            }
            L.kpc = (nk + cs - 1) / cs;
            L.out = const_cast<uint16_t *>(z);
            L.ldo = ldz;
            L.first = koff;
        } else {
            L.rows = pj.n_out;
            L.K = R;
            L.bits8 = even8(q0.u_bits, q0.u_ld) && (!two || (q0.rank % 64 == 0 && even8(q1.u_bits, q1.u_ld)));
            L.bits0 = q0.u_bits;
            L.bld0 = q0.u_ld;
            L.s0 = q0.h;
            if (two) {
                L.bits1 = q1.u_bits;
                L.bld1 = q1.u_ld;
                L.s1 = q1.h;
            }
            L.kpc = ((R + BK - 1) / BK + cs - 1) / cs;
            L.out = pj.y + (int64_t)m0 * pj.ldy;
            L.ldo = pj.ldy;
            L.first = tile0;
            L.koff = koff;
            tile0 += (pj.n_out + TM - 1) / TM;
        }
        koff += R;
    }
    // the token operand: x (mode 1) or z over every layer's latents (mode 2)
    CUtensorMap tm;
    const cudaError_t e = MODE == 1 ? encode_2d(&tm, g.x + (int64_t)m0 * g.ldx, M, g.n_in, g.ldx, true, NT)
                                    : encode_2d(&tm, z, M, koff, ldz, false, NT);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cs;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(tiles * cs));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = MidShape<NT>::kSmem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = cs > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, mid_gemm_kernel<MODE, NT, NQ>, tm, G);
}

// Dispatch on the token tile (NT) and the layer slots (a single layer takes
// the one-slot kernels, whose parameter block and selection are smallest).
template <int MODE>
cudaError_t launch_mid_any(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream, int m0, int M,
                           const uint16_t *z, int64_t ldz)
{
    const bool one = g.nproj == 1;
    if (M <= 16)
        return one ? launch_mid<MODE, 16, 1>(g, dev, stream, m0, M, z, ldz)
                   : launch_mid<MODE, 16, kMaxSiblings>(g, dev, stream, m0, M, z, ldz);
    if (M <= 32)
        return one ? launch_mid<MODE, 32, 1>(g, dev, stream, m0, M, z, ldz)
                   : launch_mid<MODE, 32, kMaxSiblings>(g, dev, stream, m0, M, z, ldz);
    if (M <= 64)
        return one ? launch_mid<MODE, 64, 1>(g, dev, stream, m0, M, z, ldz)
                   : launch_mid<MODE, 64, kMaxSiblings>(g, dev, stream, m0, M, z, ldz);
    return one ? launch_mid<MODE, 128, 1>(g, dev, stream, m0, M, z, ldz)
               : launch_mid<MODE, 128, kMaxSiblings>(g, dev, stream, m0, M, z, ldz);
}

template <int NT, int NQ>
cudaError_t prepare_slots(cudaError_t e)
{
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(mid_gemm_kernel<1, NT, NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)MidShape<NT>::kSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(mid_gemm_kernel<2, NT, NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)MidShape<NT>::kSmem);
    return e;
}

template <int NT>
cudaError_t prepare_nt(cudaError_t e)
{
    return prepare_slots<NT, kMaxSiblings>(prepare_slots<NT, 1>(e));
}

}  // namespace

cudaError_t mid_prepare_device(const DeviceInfo &dev)
{
    (void)dev;
    cudaError_t e = get_encoder();
    e = prepare_nt<16>(e);
    e = prepare_nt<32>(e);
    e = prepare_nt<64>(e);
    return prepare_nt<128>(e);
}

size_t mid_workspace_bytes(int tokens, const int *ranks, int npaths)
{
    const size_t R = (size_t)ranks[0] + (npaths > 1 ? ranks[1] : 0);
    return (size_t)std::min(tokens, kMidMaxTokens) * R * 2;
}

size_t mid_group_workspace_bytes(int tokens, const GroupArgs &g)
{
    size_t R = 0;
    for (int j = 0; j < g.nproj; ++j) R += (size_t)layer_rank(g.proj[j]);
    return (size_t)std::min(tokens, kMidMaxTokens) * R * 2;
}

cudaError_t mid_latent(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M, uint16_t *z,
                       int64_t ldz)
{
    return launch_mid_any<1>(group_of_one(a), dev, stream, m0, M, z, ldz);
}

cudaError_t mid_expand(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M,
                       const uint16_t *z, int64_t ldz)
{
    return launch_mid_any<2>(group_of_one(a), dev, stream, m0, M, z, ldz);
}

cudaError_t mid_group_forward(const GroupArgs &g, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    int R = 0;
    for (int j = 0; j < g.nproj; ++j) R += layer_rank(g.proj[j]);
    uint16_t *z = static_cast<uint16_t *>(g.workspace);  // [M][R] fp16, every layer's latents
    const cudaError_t e = launch_mid_any<1>(g, dev, stream, m0, M, z, R);
    return e != cudaSuccess ? e : launch_mid_any<2>(g, dev, stream, m0, M, z, R);
}

cudaError_t mid_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, int m0, int M)
{
    return mid_group_forward(group_of_one(a), dev, stream, m0, M);
}

}  // namespace lb
