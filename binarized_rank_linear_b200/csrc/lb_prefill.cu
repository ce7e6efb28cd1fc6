// lb_prefill.cu - the forward pass for more than 32 tokens, on tcgen05 tensor cores.
//
// The layer (sesamedisk.com, "Samsung LittleBit 13B Model", section "What the
// method actually computes", Proposition 1) is two dense contractions once
// there are many tokens, so each runs as one GEMM with a binary operand:
//
//   contraction 1:  Z[M x R]     = (X[M x n_in] . B1^T) (.) l,  B1[k, i] = sign(V_p[i, k]) g_p[i]
//   contraction 2:  Y[M x n_out] =  Z . B2^T,                   B2[o, k] = sign(U_p[o, k]) h_p[o]
//
// with both paths of residual compensation concatenated: along N in
// contraction 1 (R = r0 + r1 latent columns, path 0 first) and along K in
// contraction 2 (the latent columns of both paths, each row of B2 scaled by
// its own path's h).  Contraction 1 runs bf16 x bf16 (x as given; g rounded
// to bf16); contraction 2 runs fp16 x fp16 (z rounded to fp16; h exact).
// Accumulation is fp32 in tensor memory.
//
// One CTA computes a 128 x 256 tile of C = A . B^T:
//   warp 0      allocates tensor memory and streams A tiles with TMA (128-byte
//               swizzle, no multicast)
//   warp 1      one thread issues tcgen05.mma (M = 128, N = 256, K = 16) and
//               commits each stage back to its producers
//   warps 2..9  one B row per thread: expand the row's packed sign bits into
//               +-scale values in the same swizzled layout, then read the
//               accumulator out of tensor memory and store the tile
// Stages are handed over with mbarriers (4-deep ring).  Every wait is bounded
// in time: a wait that gives up sets LB_ERR_DEVICE_TIMEOUT on the status word
// and the CTA winds down (drains its copies, frees tensor memory) instead of
// hanging.
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"

namespace lb {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int kGroupWarps = 8;                   // producer warps per K-block: one B row per thread
constexpr int kProducerWarps = 2 * kGroupWarps;  // two groups take alternate K-blocks
constexpr int kThreads = 64 + 32 * kProducerWarps;
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;  // 32 KB
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t G_BYTES = 2 * BK * 2;  // a K-block of g for both paths
// per stage: A tile, B tile; per producer warp: two slots of g rounded to bf16
constexpr size_t kSmem = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + (size_t)kProducerWarps * 2 * G_BYTES + 256;
constexpr unsigned long long kWaitNs = 2000000000ull;  // give up on a wait after 2 s

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ unsigned long long globaltimer()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// Wait for the phase with the given parity to complete, for at most kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > kWaitNs) return false;
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *tm, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(tm), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor for kind::f16: fp32 accumulate, K-major A and B,
// M = 128, N = 256; `fmt` 0 = fp16 operands, 1 = bf16 operands.
__device__ __forceinline__ uint32_t instr_desc(uint32_t fmt)
{
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// Tiles are K-major with 128-byte swizzle: row `row` holds 64 two-byte
// elements in 128 bytes, and its 16-byte chunk j (elements 8j .. 8j + 7) is
// stored at chunk position j ^ (row % 8).

// ---------------------------------------------------------------- kernel
struct SignGemmParams {
    int M, N, K;
    int r0;  // mode 1: B rows [0, r0) are path 0; mode 2: K columns [0, r0) are path 0
    int bits8;  // every K-block's two words of a row can be fetched as one aligned 8-byte copy
    const uint32_t *bits0, *bits1;
    int64_t bld0, bld1;          // words per packed row
    const uint16_t *s0, *s1;     // mode 1: g (fp16, length K); mode 2: h (fp16, length N)
    const uint16_t *l0, *l1;     // mode 1: latent scale (epilogue)
    void *out;                   // mode 1: z fp16 [M x N]; mode 2: y bf16 [M x N]
    int64_t ldo;
    int *status;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    sign_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const SignGemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // SW128 tiles need 1024-byte alignment
    const uint32_t sA = base, sB = base + STAGES * A_BYTES;
    const uint32_t sGbf = sB + STAGES * B_BYTES;  // mode 1, per producer warp: g in bf16, [warp][2][path][64]
    const uint32_t bars = sGbf + kProducerWarps * 2 * G_BYTES;       // full[4], empty[4], accum, then the tmem address
    const uint32_t full0 = bars, empty0 = bars + 8 * STAGES, accum = bars + 16 * STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + (bars + 16 * STAGES + 8 - raw));
    __shared__ int abort_shared;
    volatile int &abort_flag = abort_shared;  // set by whichever role gives up; read by all

    const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;
    const int nk = (p.K + BK - 1) / BK;

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(full0 + 8 * s, 1 + kGroupWarps);  // TMA arrive.expect_tx + one group's warps
                mbar_init(empty0 + 8 * s, 1);     // one tcgen05.commit
            }
            mbar_init(accum, 1);
            abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- A producer (TMA)
        if (lane == 0) {
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % STAGES;
                const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
                if (!mbar_wait(empty0 + 8 * s, ph ^ 1u) || abort_flag) {
                    abort_flag = 1;
                    break;
                }
                mbar_arrive_expect_tx(full0 + 8 * s, A_BYTES);
                tma_load_2d(sA + s * A_BYTES, &tmA, kb * BK, m0, full0 + 8 * s);
                ++issued;
            }
            if (abort_flag) {
                // let copies already in flight land before the CTA goes away
                for (int kb = (issued > STAGES ? issued - STAGES : 0); kb < issued; ++kb)
                    mbar_wait(full0 + 8 * (kb % STAGES), (uint32_t)(kb / STAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = instr_desc(MODE == 1 ? 1u : 0u);
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % STAGES;
                const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
                if (!mbar_wait(full0 + 8 * s, ph) || abort_flag) {
                    abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = smem_desc(sA + s * A_BYTES), bd = smem_desc(sB + s * B_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)  // +32 bytes along K per step of 16
                    umma(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                umma_commit(empty0 + 8 * s);
            }
            umma_commit(accum);
        }
    } else {
        // ---------------- B producers: 16 warps in two groups.  Group q expands
        // the K-blocks kb = q, q + 2, ..., one B row per thread, so every warp
        // has two MMA periods for each of its blocks and its latency (barrier
        // wait, expansion, arrive) hides behind the other group's block.  The
        // row's sign words (and, in mode 1, a piece of g) are loaded into
        // registers four K-blocks ahead of use.
        const int pt = tid - 64;
        const int grp = pt >> 8;        // 0 or 1
        const int row = pt & (BN - 1);  // B row within the tile
        const int wl = warp - 2;        // producer warp 0 .. 15
        const int nn = n0 + row;        // row of B (mode 1: latent index; mode 2: output row)
        const uint32_t x7 = (uint32_t)(row & 7);  // the row's 128-byte swizzle: logical chunk j sits at chunk j ^ x7
        const bool row_in = nn < p.N;
        const bool sec_row = MODE == 1 && nn >= p.r0;  // mode 1: the row's path
        uint32_t hs0 = 0u, hs1 = 0u;                   // mode 2: h of the row, both halves
        if (MODE == 2 && row_in) {
            const uint32_t h0 = p.s0[nn], h1 = p.s1 ? p.s1[nn] : 0u;
            hs0 = h0 | (h0 << 16);
            hs1 = h1 | (h1 << 16);
        }
        const uint32_t *row_bits0 = nullptr;  // mode 1: the row's packed words; mode 2: path 0 row
        const uint32_t *row_bits1 = nullptr;  // mode 2: path 1 row
        if (row_in) {
            if (MODE == 1)
                row_bits0 = sec_row ? p.bits1 + (int64_t)(nn - p.r0) * p.bld1 : p.bits0 + (int64_t)nn * p.bld0;
            else {
                row_bits0 = p.bits0 + (int64_t)nn * p.bld0;
                if (p.bits1) row_bits1 = p.bits1 + (int64_t)nn * p.bld1;
            }
        }
        const int kwords = p.K >> 5, r0w = p.r0 >> 5;
        const uint32_t gbfw = sGbf + (uint32_t)wl * 2 * G_BYTES;  // this warp's two bf16 g slots
        auto word_ptr = [&](int w) { return (MODE == 1 || w < r0w) ? row_bits0 + w : row_bits1 + (w - r0w); };
        // The row's two words of K-block kb (zero past the end of the row).
        auto load_bits = [&](int kb) {
            uint2 v = make_uint2(0u, 0u);
            const int wd = 2 * kb;
            if (row_in && wd < kwords) {
                if (p.bits8 && wd + 1 < kwords) {
                    v = ldg_early_v2(word_ptr(wd));
                } else {
                    v.x = ldg_early_u32(word_ptr(wd));
                    if (wd + 1 < kwords) v.y = ldg_early_u32(word_ptr(wd + 1));
                }
            }
            return v;
        };
        // Mode 1: lanes 0..15 fetch one 16-byte piece of g of K-block kb (path
        // lane / 8, columns 8 (lane % 8) ..), as given (fp16).
        auto load_g = [&](int kb) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (MODE == 1 && lane < 16) {
                const int pp = lane >> 3, k0 = kb * BK + 8 * (lane & 7);
                const uint16_t *gs = pp ? p.s1 : p.s0;
                if (gs != nullptr && k0 < p.K) v = ldg_early_v4(gs + k0);
            }
            return v;
        };
        uint2 nb0 = load_bits(grp), nb1 = load_bits(grp + 2);
        uint4 ng0 = load_g(grp), ng1 = load_g(grp + 2);
        for (int kb = grp, j = 0; kb < nk; kb += 2, ++j) {
            const uint2 wb2 = nb0;
            const uint4 gcur = ng0;
            nb0 = nb1;
            ng0 = ng1;
            if (kb + 4 < nk) {
                nb1 = load_bits(kb + 4);
                ng1 = load_g(kb + 4);
            }
            const int s = kb % STAGES;
            const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
            // wait for the MMA to release stage s (it last held block kb - 4,
            // this group's previous use of it); the decision is per warp
            bool ok = mbar_wait(empty0 + 8 * s, ph ^ 1u) && !abort_flag;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                abort_flag = 1;
                break;
            }
            uint4 sc[8];  // per chunk: the four packed scale words
            if (MODE == 1) {
                // lanes 0..15 round this block's g to bf16 into the warp's slot
                // j % 2 (last read two iterations ago, before a __syncwarp)
                if (lane < 16) {
                    const uint32_t w[4] = {gcur.x, gcur.y, gcur.z, gcur.w};
                    uint32_t o[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        o[i] = (uint32_t)float_to_bf16_bits(f16_bits_to_float((uint16_t)(w[i] & 0xffffu))) |
                               ((uint32_t)float_to_bf16_bits(f16_bits_to_float((uint16_t)(w[i] >> 16))) << 16);
                    *reinterpret_cast<uint4 *>(smem_raw + (gbfw + (j & 1) * G_BYTES + lane * 16 - raw)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
                __syncwarp();
                const uint8_t *gb = smem_raw + (gbfw + (j & 1) * G_BYTES + (sec_row ? BK * 2 : 0) - raw);
#pragma unroll
                for (int q = 0; q < 8; ++q) sc[q] = *reinterpret_cast<const uint4 *>(gb + 16 * q);
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int k0 = kb * BK + 8 * q;  // first column of the chunk
                    const uint32_t h = k0 < p.K ? (k0 >= p.r0 ? hs1 : hs0) : 0u;
                    sc[q] = make_uint4(h, h, h, h);
                }
            }
            // chunk q of the row goes to chunk position q ^ x7 (the tile is
            // 1024-byte aligned, so the XOR acts on address bits 4..6 alone);
            // the 8 rows of a store phase then cover all 32 banks
            const uint32_t rowx = (sB + s * B_BYTES + row * 128) | (x7 << 4);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t b = __byte_perm(q < 4 ? wb2.x : wb2.y, 0u, 0x4440u | (uint32_t)(q & 3));
                // (b * K_i) puts sign bit 2i at bit 15 and bit 2i + 1 at bit 31
                // (the two shifted copies of the byte do not overlap: no carries)
                const uint32_t v0 = ((b * 0x40008000u) & 0x80008000u) ^ sc[q].x;
                const uint32_t v1 = ((b * 0x10002000u) & 0x80008000u) ^ sc[q].y;
                const uint32_t v2 = ((b * 0x04000800u) & 0x80008000u) ^ sc[q].z;
                const uint32_t v3 = ((b * 0x01000200u) & 0x80008000u) ^ sc[q].w;
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowx ^ (16u * q)), "r"(v0), "r"(v1),
                             "r"(v2), "r"(v3)
                             : "memory");
            }
            fence_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(full0 + 8 * s);
        }

        // ---------------- epilogue: tensor memory -> registers -> global
        bool ok = !abort_flag;
        if (ok) ok = mbar_wait(accum, 0);
        ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
        if (!ok) abort_flag = 1;
        tc_fence_after();
        const int quad = warp & 3;  // warp w reads tensor-memory lanes 32 (w % 4) ..
        const int m = m0 + 32 * quad + lane;
        const int cbeg = ((warp - 2) / 4) * (BN / 4);  // four warps per lane quadrant: column quarters
        bool overflow = false;
        for (int c0 = cbeg; c0 < cbeg + BN / 4; c0 += 16) {
            uint32_t v[16];
            if (ok) tmem_ld16(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)c0, v);
            const int nn = n0 + c0;
            if (!ok || m >= p.M || nn >= p.N) continue;
            uint32_t o[8];
            if (MODE == 1) {
                // z = l (.) c, rounded to fp16 (the operand of contraction 2)
                const bool sec = nn >= p.r0;
                const uint16_t *lp = sec ? p.l1 + (nn - p.r0) : p.l0 + nn;
                const uint4 la = __ldg(reinterpret_cast<const uint4 *>(lp));
                const uint4 lb = __ldg(reinterpret_cast<const uint4 *>(lp + 8));
                const uint32_t lw[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float z0 = __uint_as_float(v[2 * i]) * f16_bits_to_float((uint16_t)(lw[i] & 0xffffu));
                    const float z1 = __uint_as_float(v[2 * i + 1]) * f16_bits_to_float((uint16_t)(lw[i] >> 16));
                    overflow |= beyond_f16(z0) | beyond_f16(z1);
                    o[i] = pack_half2(z0, z1);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    o[i] = (uint32_t)float_to_bf16_bits(__uint_as_float(v[2 * i])) |
                           ((uint32_t)float_to_bf16_bits(__uint_as_float(v[2 * i + 1])) << 16);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + (int64_t)m * p.ldo + nn);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
        if (overflow) set_status(p.status, LB_ERR_RANGE);
    }

    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) set_status(p.status, LB_ERR_DEVICE_TIMEOUT);
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

cudaError_t get_encoder()
{
    if (g_encode) return cudaSuccess;
    cudaDriverEntryPointQueryResult q;
    void *fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return cudaSuccess;
}

// 2-D map over a row-major [rows x cols] matrix of 2-byte elements with row
// stride `ld` elements; boxes of 64 columns x 128 rows, 128-byte swizzle.
cudaError_t encode_a(CUtensorMap *tm, const void *ptr, int rows, int cols, int64_t ld, bool bf16)
{
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {BK, BM};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                                const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// True when every row of a packed matrix starts 8-byte aligned.
bool even8(const uint32_t *bits, int64_t ld) { return (reinterpret_cast<uintptr_t>(bits) & 7u) == 0 && ld % 2 == 0; }

}  // namespace

cudaError_t prefill_prepare_device(const DeviceInfo &dev)
{
    (void)dev;
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(sign_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(sign_gemm_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
}

size_t prefill_workspace_bytes(int tokens, const int *ranks, int npaths)
{
    const size_t R = (size_t)ranks[0] + (npaths > 1 ? ranks[1] : 0);
    return (size_t)tokens * R * 2 + 256;
}

cudaError_t prefill_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    const int M = a.tokens;
    const int r0 = a.path[0].rank, r1 = a.npaths > 1 ? a.path[1].rank : 0;
    const int R = r0 + r1;
    uint16_t *z = static_cast<uint16_t *>(a.workspace);  // [M x R] fp16
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;

    // contraction 1: Z = (X . B1^T) (.) l
    CUtensorMap tx;
    e = encode_a(&tx, a.x, M, a.n_in, a.ldx, true);
    if (e != cudaSuccess) return e;
    SignGemmParams p1{};
    p1.M = M;
    p1.N = R;
    p1.K = a.n_in;
    p1.r0 = r0;
    p1.bits8 = even8(a.path[0].vt_bits, a.path[0].vt_ld) && (a.npaths < 2 || even8(a.path[1].vt_bits, a.path[1].vt_ld));
    p1.bits0 = a.path[0].vt_bits;
    p1.bld0 = a.path[0].vt_ld;
    p1.s0 = a.path[0].g;
    p1.l0 = a.path[0].l;
    if (a.npaths > 1) {
        p1.bits1 = a.path[1].vt_bits;
        p1.bld1 = a.path[1].vt_ld;
        p1.s1 = a.path[1].g;
        p1.l1 = a.path[1].l;
    }
    p1.out = z;
    p1.ldo = R;
    p1.status = dev.status;
    dim3 grid1((unsigned)((M + BM - 1) / BM), (unsigned)((R + BN - 1) / BN));
    sign_gemm_kernel<1><<<grid1, kThreads, kSmem, stream>>>(tx, p1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // contraction 2: Y = Z . B2^T
    CUtensorMap tz;
    e = encode_a(&tz, z, M, R, R, false);
    if (e != cudaSuccess) return e;
    SignGemmParams p2{};
    p2.M = M;
    p2.N = a.n_out;
    p2.K = R;
    p2.r0 = r0;
    p2.bits8 = even8(a.path[0].u_bits, a.path[0].u_ld) && (a.npaths < 2 || (r0 % 64 == 0 && even8(a.path[1].u_bits, a.path[1].u_ld)));
    p2.bits0 = a.path[0].u_bits;
    p2.bld0 = a.path[0].u_ld;
    p2.s0 = a.path[0].h;
    if (a.npaths > 1) {
        p2.bits1 = a.path[1].u_bits;
        p2.bld1 = a.path[1].u_ld;
        p2.s1 = a.path[1].h;
    }
    p2.out = a.y;
    p2.ldo = a.ldy;
    p2.status = dev.status;
    dim3 grid2((unsigned)((M + BM - 1) / BM), (unsigned)((a.n_out + BN - 1) / BN));
    sign_gemm_kernel<2><<<grid2, kThreads, kSmem, stream>>>(tz, p2);
    return cudaGetLastError();
}

}  // namespace lb
