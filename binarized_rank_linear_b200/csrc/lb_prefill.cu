// lb_prefill.cu - the forward pass for more than 128 tokens, on tcgen05 tensor cores.
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
// A persistent grid (one CTA per SM, or one CTA pair per two SMs) walks the
// tiles of C = A . B^T, 128 or 256 rows per CTA by bn columns, bn a multiple
// of 32 up to 256, the shape chosen per call (see plan_tiles).  In each CTA
// (here for single-CTA tiles of 128 rows):
//   warp 0       allocates tensor memory (two 256-column accumulators) and
//                streams A tiles with TMA (128-byte swizzle, no multicast)
//   warp 1       one thread issues tcgen05.mma (M = 128, N = bn, K = 16)
//   warps 2..17  two groups of 8 taking alternate K-blocks, one B row per
//                thread (rows past bn idle): expand the row's packed sign
//                bits into +-scale values in the same swizzled layout
//   warps 18..21 read a finished accumulator out of tensor memory and store
//                the tile, while the MMA fills the other accumulator
// Stages are handed over with mbarriers (3- to 6-deep rings).  Every
// mbarrier wait is bounded in time: a wait that gives up sets
// LB_ERR_DEVICE_TIMEOUT on the status word and the CTA winds down (drains its
// copies, frees tensor memory) instead of hanging.  The other waits are the
// hardware's own (tensor-memory allocation, which the one CTA per SM always
// gets, and the pair's cluster barriers, which every thread of both CTAs
// reaches once its mbarrier waits have ended).
//
// Larger problems run on CTA pairs (clusters of two, cta_group::2): one MMA
// of M = 256 spans both SMs, each CTA stages its own 128 rows of A and half
// of the B tile, and the MMA reads each half of B once for both SMs.  Per
// flop, each CTA then expands half as many sign rows and its shared memory
// serves a third fewer operand bytes, which is what bounds the one-CTA tiles
// (MMA operand reads plus the producers' and TMA's writes come close to the
// shared-memory bandwidth).  CTA 0 issues the MMAs and its tcgen05.commit
// arrives on the barriers of both CTAs; the TMA loads and producer arrivals
// of CTA 1 count on CTA 0's stage barriers.
//
// One more mode serves the layer's backward pass (lb_backward.cu):
//   mode 3:  the contraction-1 shape (bf16 operands, B1 rows scaled along K)
//            with the latent scale optional (l0 null: unit), the output in
//            fp16 or bf16, and optionally a column dot in the epilogue: for
//            every output column n, part0[row block][n] = sum over the
//            block's 32 rows m of C[m, n] * aux[m, n] (the unscaled C; aux
//            fp16 or bf16 [M x N]);
// and mode 2 takes bf16 operands on request (bf16_ops: A bf16, the row
// scales rounded to bf16), for the backward's dx.
// Partial sums are per 32-row block of the output, so each is written once
// and the caller reduces them in a fixed order: the results do not depend on
// timing.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"
#include "lb_tc.cuh"

namespace lb {
namespace {

using namespace tc;

constexpr int BM = 128, BN = 256, BK = 64;  // one MMA: M = 128, N = bn <= 256; K-blocks of 64
constexpr int kRowWarps = 8;                  // warps for the 256 rows of a whole B tile, one row per thread
constexpr uint32_t B_BYTES = BN * BK * 2;     // 32 KB: a whole B tile
constexpr uint32_t TMEM_COLS = 2 * BN;        // two 256-column accumulators
constexpr uint32_t G_BYTES = 2 * BK * 2;      // a K-block of g for both paths
constexpr uint32_t OUT_BYTES = 32 * 64;       // an output box: 32 rows x 32 two-byte columns

// Two tile heights.  H = 1: a CTA holds 128 rows of a tile; the two
// accumulators double-buffer consecutive tiles, and (P = 1) two producer
// groups take alternate K-blocks.  H = 2: a CTA holds 256 rows, two M = 128
// halves that share each expanded B tile (half the sign expansion per flop);
// the two accumulators hold the halves of one tile, and (P = 1) one producer
// group has twice as long per K-block.
//
// P = 2: a CTA pair (cluster of two) shares each MMA (cta_group::2, M = 256):
// CTA r of the pair holds rows 128 H r .. of the pair's 256 H-row tile of A
// and expands B rows bn r / 2 .. of the tile's bn, so each CTA stages and
// expands half of B, and the MMA reads each half of B from shared memory once
// for both SMs.  Stages are then smaller and the ring deeper.
template <int H, int P, int MODE>
struct Shape {
    static constexpr int kStages = P == 1 ? (H == 1 ? 4 : 3) : (H == 1 ? 6 : 4);
    // producer groups: one B row per thread, a group per K-block in turn
    // (P = 2: a CTA's B rows take half a group's warps, so twice the groups)
    static constexpr int kGroupWarps = kRowWarps / P;
    static constexpr int kGroups = (H == 1 ? 2 : 1) * P;
    static constexpr int kProducerWarps = kGroupWarps * kGroups;  // 16 (H = 1) or 8 (H = 2)
    static constexpr int kEpiWarps = 4 * H;  // per accumulator in use, one per tensor-memory lane quadrant
    static constexpr int kThreads = 32 * (2 + kProducerWarps + kEpiWarps);
    static constexpr int kTileM = BM * H;
    static constexpr uint32_t kABytes = (uint32_t)kTileM * BK * 2;  // 16 or 32 KB
    static constexpr uint32_t kBBytes = B_BYTES / P;                 // this CTA's rows of a B tile
    static constexpr int kOutBufs = 1;  // output boxes per epilogue warp
    static constexpr int kRing = 2;     // sign-word slots per producer thread
    // per stage: A tile, B tile; per epilogue warp: its output boxes and the
    // tile's latent scale in fp32 (mode 1); per producer warp: two slots of g
    // rounded to bf16; per producer thread: kRing slots of sign words
    static constexpr size_t kSmem = 1024 + (size_t)kStages * (kABytes + kBBytes) +
                                    (size_t)kEpiWarps * (kOutBufs * OUT_BYTES + BN * 4) +
                                    (size_t)kProducerWarps * (2 * G_BYTES + 32 * 8 * kRing) + 256;
    static_assert(kSmem <= 232448, "shared memory per CTA");
};
// Tiles are K-major with 128-byte swizzle: row `row` holds 64 two-byte
// elements in 128 bytes, and its 16-byte chunk j (elements 8j .. 8j + 7) is
// stored at chunk position j ^ (row % 8).

// ---------------------------------------------------------------- column sums
// v[j] holds row `lane` of 16 columns; returns, in lanes l and l + 16, the sum
// of column l over the warp's 32 rows.  The first step adds row pairs (lanes
// l, l ^ 16) for every column; each later step halves the columns a lane
// keeps and doubles the rows it has summed: 31 shuffles for 16 columns, in a
// fixed order.
__device__ __forceinline__ float column_sum16(float (&v)[16], int lane)
{
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] += __shfl_xor_sync(0xffffffffu, v[j], 16);
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int j = 0; j < s; ++j) {
            const float give = upper ? v[j] : v[j + s];
            const float keep = upper ? v[j + s] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, give, s);
        }
    }
    return v[0];
}

// Two bf16 or fp16 values packed in a word, widened.
__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float lo_f16(uint32_t w) { return f16_bits_to_float((uint16_t)(w & 0xffffu)); }
__device__ __forceinline__ float hi_f16(uint32_t w) { return f16_bits_to_float((uint16_t)(w >> 16)); }

// ---------------------------------------------------------------- kernel
struct SignGemmParams {
    int M, N, K;
    int bn;  // tile width along N: a multiple of 32, at most BN
    int r0;  // mode 1: B rows [0, r0) are path 0; mode 2: K columns [0, r0) are path 0
    int bits8;  // every K-block's two words of a row can be fetched as one aligned 8-byte copy
    const uint32_t *bits0, *bits1;
    int64_t bld0, bld1;          // words per packed row
    const uint16_t *s0, *s1;     // mode 1: g (fp16, length K); mode 2: h (fp16, length N)
    const uint16_t *l0, *l1;     // mode 1: latent scale (epilogue)
    void *out;                   // mode 1: z fp16 [M x N]; mode 2: y bf16 [M x N]
    int64_t ldo;
    int *status;
    // backward modes (3, 4)
    const void *aux;             // mode 3: column-dot operand, fp16 or bf16 [M x N], row stride ldaux
    int64_t ldaux;
    float *part0;                // column-dot partials [ceil(M / 32) x N]
    int out_bf16, aux_bf16;      // mode 3: store C as bf16 (else fp16); aux is bf16 (else fp16)
    int bf16_ops;                // mode 2: A and the +-scale operand in bf16 (else fp16)
};

// Persistent: CTA c computes the tiles t = c, c + gridDim.x, ...
// (tile t is rows (t % tiles_m) * 128 H and columns (t / tiles_m) * bn, so the
// CTAs running at once share the same few columns of B).  Its K-blocks form
// one sequence over all its tiles, so stages, phases and the producer groups'
// alternation run on across tile boundaries.  Two accumulators in tensor
// memory let the epilogue warps drain tile i while the MMA runs tile i + 1.
template <int MODE, int H, int P>
__global__ void __launch_bounds__(Shape<H, P, MODE>::kThreads, 1)
    sign_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmOut,
                     const SignGemmParams p)
{
    using S = Shape<H, P, MODE>;
    // modes 1 and 3 have the contraction-1 shape (bf16 operands; a B row's
    // scale runs along K and depends on the row's path), modes 2 and 4 the
    // contraction-2 shape (fp16 operands; K runs over the paths' latents)
    constexpr bool C1 = MODE == 1 || MODE == 3;
    constexpr int STAGES = S::kStages;
    constexpr uint32_t A_BYTES = S::kABytes;
    constexpr uint32_t B_STAGE = S::kBBytes;
    constexpr int kProducerWarps = S::kProducerWarps;
    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // SW128 tiles need 1024-byte alignment
    const uint32_t sA = base, sB = base + STAGES * A_BYTES;
    const uint32_t sOut = sB + STAGES * B_STAGE;  // per epilogue warp: kOutBufs output boxes
    const uint32_t sGbf = sOut + S::kEpiWarps * S::kOutBufs * OUT_BYTES;  // mode 1, per producer warp: g in bf16, [warp][2][path][64]
    const uint32_t sLf = sGbf + kProducerWarps * 2 * G_BYTES;  // mode 1, per epilogue warp: l of the tile in fp32
    const uint32_t sRing = sLf + S::kEpiWarps * BN * 4;  // per producer thread: kRing 8-byte sign-word slots
    const uint32_t bars = sRing + kProducerWarps * 32 * 8 * S::kRing;
    // full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain, then the tmem address
    const uint32_t full0 = bars, empty0 = bars + 8 * STAGES, accf0 = bars + 16 * STAGES;
    const uint32_t acce0 = accf0 + 16, drain = acce0 + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + (drain + 8 - raw));
    __shared__ int abort_shared;
    volatile int &abort_flag = abort_shared;  // set by whichever role gives up; read by all

    // P = 2: this CTA's rank in its pair; the pair's tiles are 256 H x bn
    const int rank = P == 2 ? (int)cluster_rank() : 0;
    const int tiles_m = (p.M + P * S::kTileM - 1) / (P * S::kTileM);
    const int ntiles = tiles_m * ((p.N + p.bn - 1) / p.bn);
    const int rows_b = p.bn / P;                // B rows this CTA expands per tile
    const int busy_warps = (rows_b + 31) >> 5;  // producer warps per group with rows in the tile
    const int G = gridDim.x / P, c = blockIdx.x / P;  // persistent units: CTAs, or pairs
    const int my_tiles = c < ntiles ? (ntiles - c + G - 1) / G : 0;
    const int nk = (p.K + BK - 1) / BK;
    const int nblocks = my_tiles * nk;  // this CTA's K-blocks, all tiles

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                // TMA arrive.expect_tx + one group's busy warps (P = 2: of both
                // CTAs; only CTA 0's full barriers are used)
                mbar_init(full0 + 8 * s, 1 + P * busy_warps);
                mbar_init(empty0 + 8 * s, 1);               // one tcgen05.commit
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(accf0 + 8 * b, 1);          // one tcgen05.commit
                mbar_init(acce0 + 8 * b, P * S::kEpiWarps);  // every epilogue warp (of the pair)
            }
            mbar_init(drain, 1);
            abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        if constexpr (P == 2)
            tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
        else
            tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tc_fence_before();
    }
    if (P == 2)
        cluster_sync();  // both CTAs' barriers are initialised before either arrives on the other's
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // P = 2: CTA 0's full and acc-empty barriers, as this CTA reaches them
    const uint32_t full_lead = P == 2 ? map_shared_addr(full0, 0) : full0;
    const uint32_t acce_lead = P == 2 ? map_shared_addr(acce0, 0) : acce0;

    if (warp == 0) {
        // ---------------- A producer (TMA)
        if (lane == 0) {
            int issued = 0;
            for (int gb = 0; gb < nblocks; ++gb) {
                const int i = gb / nk, kb = gb - i * nk;
                const int t = c + i * G;
                const int s = gb % STAGES;
                const uint32_t ph = (uint32_t)(gb / STAGES) & 1u;
                if (!mbar_wait(empty0 + 8 * s, ph ^ 1u) || abort_flag) {
                    abort_flag = 1;
                    break;
                }
                const int row0 = (t % tiles_m) * (P * S::kTileM);  // the (pair's) tile
                if (P == 1) {
                    mbar_arrive_expect_tx(full0 + 8 * s, A_BYTES);
                    tma_load_2d(sA + s * A_BYTES, &tmA, kb * BK, row0, full0 + 8 * s);
                } else {
                    // both CTAs' A bytes complete on CTA 0's barrier, which CTA 0 arms
                    if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * s, 2 * A_BYTES);
                    tma_load_2d_pair(sA + s * A_BYTES, &tmA, kb * BK, row0 + rank * S::kTileM, full_lead + 8 * s);
                }
                ++issued;
            }
            if (abort_flag && P == 2 && rank == 1) {
                // this CTA cannot wait on CTA 0's barriers: give copies in
                // flight time to land (they take microseconds)
                const unsigned long long t0 = globaltimer();
                while (globaltimer() - t0 < 200000ull) {
                }
            } else if (abort_flag) {
                // let copies already in flight land before the CTA goes away
                for (int gb = (issued > STAGES ? issued - STAGES : 0); gb < issued; ++gb)
                    mbar_wait(full0 + 8 * (gb % STAGES), (uint32_t)(gb / STAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer.  H = 1: tile i accumulates in columns
        // 256 (i % 2) ..; H = 2: half h of every tile accumulates in columns 256 h ..
        // P = 2: CTA 0 issues the pair's MMAs and signals both CTAs; CTA 1
        // only waits for the last of them before it may free tensor memory.
        if (lane == 0 && P == 2 && rank == 1) {
            if (!mbar_wait(drain, 0)) abort_flag = 1;
        } else if (lane == 0) {
            const uint32_t idesc = instr_desc((C1 || p.bf16_ops) ? 1u : 0u, BM * P, p.bn);
            auto commit = [&](uint32_t bar) {
                if constexpr (P == 2)
                    umma_commit_pair(bar);
                else
                    umma_commit(bar);
            };
            int gb = 0;
            for (int i = 0; i < my_tiles && !abort_flag; ++i) {
                const int b = H == 1 ? (i & 1) : 0;  // hand-over barriers of the accumulator(s)
                const int use = H == 1 ? (i >> 1) : i;
                // the epilogue has drained the accumulator(s) (tile i - 2, or i - 1)
                if (!mbar_wait(acce0 + 8 * b, (uint32_t)(use & 1) ^ 1u)) {
                    abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(b * BN);
                for (int kb = 0; kb < nk; ++kb, ++gb) {
                    const int s = gb % STAGES;
                    const uint32_t ph = (uint32_t)(gb / STAGES) & 1u;
                    if (!mbar_wait(full0 + 8 * s, ph) || abort_flag) {
                        abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bd = smem_desc(sB + s * B_STAGE);
#pragma unroll
                    for (int h = 0; h < H; ++h) {
                        // half h: A rows 128 h .. (16 KB further on, a whole number of 8-row atoms)
                        const uint64_t ad = smem_desc(sA + s * A_BYTES + (uint32_t)h * (BM * BK * 2));
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {  // +32 bytes along K per step of 16
                            if constexpr (P == 2) {
                                umma_pair(acc + (uint32_t)(h * BN), ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                            } else {
                                umma(acc + (uint32_t)(h * BN), ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0);
                            }
                        }
                    }
                    commit(empty0 + 8 * s);
                }
                if (abort_flag) break;
                commit(accf0 + 8 * b);
            }
            // every MMA issued has finished before the CTA (and its pair) frees tensor memory
            commit(drain);
            if (!mbar_wait(drain, 0)) abort_flag = 1;
        }
    } else if (warp < 2 + kProducerWarps) {
        // ---------------- B producers: groups of kGroupWarps warps, one B row
        // per thread.  P = 1, H = 1: two groups of 8; group q expands the
        // blocks gb = q, q + 2, ... of the CTA's K-block sequence, so every
        // warp has two MMA periods for each of its blocks and its latency
        // (barrier wait, expansion, arrive) hides behind the other group's
        // block.  P = 1, H = 2: one group; a block feeds two MMA halves, so it
        // has two MMA periods as well.  P = 2: a CTA expands at most 128 rows
        // of a block, so groups of 4 warps and twice as many of them: four
        // (or two) MMA periods per block.
        // What a block needs from memory arrives without a register holding a
        // load in flight across blocks (copying such a register would wait
        // for the load):
        //   sign words  copied asynchronously (cp.async) into the thread's
        //               slot of a ring in shared memory, kRing of the group's
        //               blocks ahead, and waited for just before use;
        //   g (mode 1)  lanes 0..15 copy a block's 64 values of each path
        //               (fp16) into the warp's g slot the same way, and round
        //               them to bf16 in place just before use;
        //   h (mode 2)  depends on the row only, so it is loaded once per
        //               tile, a tile ahead.
        const int pt = tid - 64;
        constexpr int NG = S::kGroups;  // block stride of a group
        constexpr int RING = S::kRing;
        static_assert(RING == 2, "the warp's two g slots double as the g ring");
        constexpr uint32_t RING_STRIDE = (uint32_t)kProducerWarps * 32 * 8;  // bytes between ring slots
        constexpr int GT = S::kGroupWarps * 32;  // threads (rows) of a group
        const int grp = pt / GT;                // 0 .. NG - 1
        const int row = pt & (GT - 1);          // B row within this CTA's rows of the tile (valid below rows_b)
        const int nrow = rank * rows_b + row;  // ... within the tile
        const int wl = warp - 2;        // producer warp 0 .. 15
        const uint32_t x7 = (uint32_t)(row & 7);  // the row's 128-byte swizzle: logical chunk j sits at chunk j ^ x7
        const int kwords = p.K >> 5, r0w = p.r0 >> 5;
        const uint32_t gbfw = sGbf + (uint32_t)wl * 2 * G_BYTES;  // this warp's two bf16 g slots
        const uint32_t ring = sRing + (uint32_t)pt * 8;           // this thread's slot 0 (8 bytes)
        // a warp whose rows all lie past bn takes no part (the stage barriers
        // count only the busy warps)
        const int my_blocks = (wl & (S::kGroupWarps - 1)) < busy_warps ? nblocks : 0;
        // Position of a block in the sequence, advanced without divisions:
        // tile iteration, K-block, and this thread's B row in that tile.
        struct Cursor {
            int gb, i, kb, nn;
        };
        auto cursor_at = [&](int gb) {
            Cursor u;
            u.gb = gb;
            u.i = gb / nk;
            u.kb = gb - u.i * nk;
            u.nn = ((c + u.i * G) / tiles_m) * p.bn + nrow;
            return u;
        };
        auto advance = [&](Cursor &u) {
            u.gb += NG;
            u.kb += NG;
            if (u.kb >= nk) {
                while (u.kb >= nk) {
                    u.kb -= nk;
                    ++u.i;
                }
                u.nn = ((c + u.i * G) / tiles_m) * p.bn + nrow;
            }
        };
        // Start the copies of block u's two sign words into ring slot `slot`
        // (zeros outside the matrix) and, mode 1, lanes 0..15, of its g into
        // the warp's g slot `slot`: one cp.async group.
        auto copy_block = [&](const Cursor &u, int slot) {
            if (C1 && u.gb < my_blocks && lane < 16) {
                // lane: path lane / 8, columns 8 (lane % 8) .. 8 (lane % 8) + 7 of the block
                const int pp = lane >> 3, k0 = u.kb * BK + 8 * (lane & 7);
                const uint16_t *gs = pp ? p.s1 : p.s0;
                const uint32_t gdst = gbfw + (uint32_t)slot * G_BYTES + (uint32_t)lane * 16;
                if (gs != nullptr && k0 < p.K)
                    cp_async16s(gdst, gs + k0);
                else
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(gdst), "r"(0u) : "memory");
            }
            const uint32_t dst = ring + (uint32_t)slot * RING_STRIDE;
            const int wd = 2 * u.kb;  // first word of the block in the (concatenated) row
            if (u.gb < my_blocks && row < rows_b && u.nn < p.N && wd < kwords) {
                const int nn = u.nn;
                const uint32_t *rb0, *rb1 = nullptr;
                if (C1) {
                    const bool sec = nn >= p.r0;
                    rb0 = sec ? p.bits1 + (int64_t)(nn - p.r0) * p.bld1 : p.bits0 + (int64_t)nn * p.bld0;
                } else {
                    rb0 = p.bits0 + (int64_t)nn * p.bld0;
                    if (p.bits1) rb1 = p.bits1 + (int64_t)nn * p.bld1;
                }
                auto wp = [&](int w) { return (C1 || w < r0w) ? rb0 + w : rb1 + (w - r0w); };
                if (p.bits8 && wd + 1 < kwords) {
                    cp_async8(dst, wp(wd));
                } else {
                    cp_async4(dst, wp(wd));
                    if (wd + 1 < kwords)
                        cp_async4(dst + 4, wp(wd + 1));
                    else
                        asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst + 4), "r"(0u) : "memory");
                }
            } else if (u.gb < my_blocks) {
                asm volatile("st.shared.v2.u32 [%0], {%1, %1};" ::"r"(dst), "r"(0u) : "memory");
            }
            cp_async_commit();  // one group per block (empty past the end), so the waits count blocks
        };
        // mode 2: h of this thread's row in tile iteration i, both paths (fp16 pair)
        auto fetch_h = [&](int i) {
            uint32_t hv = 0u;
            const int nn = ((c + i * G) / tiles_m) * p.bn + nrow;
            if (MODE == 2 && i < my_tiles && row < rows_b && nn < p.N) {
                hv = ldg_early_u16(p.s0 + nn);
                if (p.s1) hv |= (uint32_t)ldg_early_u16(p.s1 + nn) << 16;
            }
            return hv;
        };
        Cursor u = cursor_at(grp), ua = cursor_at(grp + RING * NG);  // this block, and the group's block RING ahead
        {
            Cursor w = u;
            for (int d = 0; d < RING; ++d, advance(w)) copy_block(w, d);
        }
        int hi = -2;                  // tile iteration whose h is in hcur (none yet; hnext is for hi + 1)
        uint32_t hcur = 0u, hnext = 0u;
        for (int j = 0; u.gb < my_blocks; ++j, advance(u), advance(ua)) {
            const int gb = u.gb, kb = u.kb, nn = u.nn;
            if (MODE == 2 && u.i != hi) {  // first block of a tile for this group
                hcur = u.i == hi + 1 ? hnext : fetch_h(u.i);
                if (p.bf16_ops)  // the row's scales rounded to bf16, the operand type
                    hcur = pack_bf162(f16_bits_to_float((uint16_t)(hcur & 0xffffu)), f16_bits_to_float((uint16_t)(hcur >> 16)));
                hnext = fetch_h(u.i + 1);
                hi = u.i;
            }
            const int s = gb % STAGES;
            const uint32_t ph = (uint32_t)(gb / STAGES) & 1u;
            // wait for the MMA to release stage s (it last held block
            // gb - STAGES); the decision is per warp
            bool ok = mbar_wait(empty0 + 8 * s, ph ^ 1u) && !abort_flag;
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                abort_flag = 1;
                break;
            }
            // this block's copies have landed (at most RING - 1 younger
            // groups still pending)
            cp_async_wait_group<RING - 1>();
            const int slot = j % RING;
            uint4 sc[8];  // per chunk: the four packed scale words
            if (C1) {
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
                const bool sec_row = nn >= p.r0;  // the row's path
                const uint8_t *gb_ = smem_raw + (gsl + (sec_row ? BK * 2 : 0) - raw);
#pragma unroll
                for (int q = 0; q < 8; ++q) sc[q] = *reinterpret_cast<const uint4 *>(gb_ + 16 * q);
            } else {
                const uint32_t hs0 = (hcur & 0xffffu) * 0x10001u, hs1 = (hcur >> 16) * 0x10001u;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int k0 = kb * BK + 8 * q;  // first column of the chunk
                    const uint32_t h = k0 < p.K ? (k0 >= p.r0 ? hs1 : hs0) : 0u;
                    sc[q] = make_uint4(h, h, h, h);
                }
            }
            uint2 bits;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                         : "=r"(bits.x), "=r"(bits.y)
                         : "r"(ring + (uint32_t)slot * RING_STRIDE)
                         : "memory");
            // chunk q of the row goes to chunk position q ^ x7 (the tile is
            // 1024-byte aligned, so the XOR acts on address bits 4..6 alone);
            // the 8 rows of a store phase then cover all 32 banks
            const uint32_t rowx = (sB + s * B_STAGE + row * 128) | (x7 << 4);
            if (row < rows_b) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    store_sign_chunk(rowx ^ (16u * q), __byte_perm(q < 4 ? bits.x : bits.y, 0u, 0x4440u | (uint32_t)(q & 3)),
                                     sc[q]);
                }
            }
            fence_async_shared();
            __syncwarp();
            if (lane == 0) {
                if (P == 2 && rank == 1)
                    mbar_arrive_remote(full_lead + 8 * s);
                else
                    mbar_arrive(full0 + 8 * s);
            }
            // refill the slots (their contents are used above, and every lane
            // is past its reads after the __syncwarp) with the group's block
            // RING ahead
            copy_block(ua, slot);
        }
        cp_async_wait_all();  // no copy may land after the CTA is gone
    } else {
        // ---------------- epilogue: warp w drains tensor-memory lanes 32 (w % 4)
        // .. of a finished accumulator (H = 2: warps 4 e .. 4 e + 3 of the
        // epilogue drain half e), then hands the accumulator back.  Each
        // 32-column chunk of the warp's 32 rows goes out as one bulk tensor
        // store: the lanes (one row each) write the converted chunk into a
        // swizzled box in shared memory, and lane 0 issues the store.  Rows or
        // columns past the matrix are clipped by the store itself.
        const int quad = warp & 3;
        const int ew = warp - 2 - kProducerWarps;  // epilogue warp 0 .. kEpiWarps - 1
        const int eh = H == 1 ? 0 : ew >> 2;
        const uint32_t obox = sOut + (uint32_t)ew * S::kOutBufs * OUT_BYTES;  // the warp's boxes
        const uint32_t lsm = sLf + (uint32_t)ew * BN * 4;                        // the warp's fp32 l
        const uint32_t rsw = (uint32_t)((lane >> 1) & 3);  // the row's 64-byte swizzle
        int nst = 0;  // boxes this warp has stored
        bool overflow = false;
        for (int i = 0; i < my_tiles; ++i) {
            const int b = H == 1 ? (i & 1) : 0;
            const int use = H == 1 ? (i >> 1) : i;
            const int t = c + i * G;
            // the warp's first row (P = 2: this CTA's rows of the pair's tile)
            const int m0 = (t % tiles_m) * (P * S::kTileM) + rank * S::kTileM + eh * BM + 32 * quad;
            const bool row_in = m0 + lane < p.M;
            const int n0 = (t / tiles_m) * p.bn;
            if (C1) {
                // the tile's latent scale, widened to fp32 once (lane j takes
                // columns j, j + 32, ...) while the accumulator fills (mode 3
                // without one: 1)
                for (int cc = lane; cc < p.bn && n0 + cc < p.N; cc += 32) {
                    const int nn = n0 + cc;
                    const float lv = (MODE == 3 && p.l0 == nullptr)
                                         ? 1.0f
                                         : f16_bits_to_float(nn >= p.r0 ? p.l1[nn - p.r0] : p.l0[nn]);
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(lsm + 4u * (uint32_t)cc), "f"(lv) : "memory");
                }
                __syncwarp();
            }
            if (MODE == 3 && p.aux != nullptr && row_in) {
                // the column dot's operand for this lane's row of the tile into
                // L2 while the accumulator fills (128 bytes per prefetch)
                const uint16_t *ar = static_cast<const uint16_t *>(p.aux) + (int64_t)(m0 + lane) * p.ldaux;
                for (int cc = 0; cc < p.bn && n0 + cc < p.N; cc += 64)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(ar + n0 + cc));
            }
            bool ok = !abort_flag && mbar_wait(accf0 + 8 * b, (uint32_t)(use & 1));
            ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
            if (!ok) {
                abort_flag = 1;
                break;
            }
            tc_fence_after();
            for (int c32 = 0; c32 < p.bn && n0 + c32 < p.N; c32 += 32) {
                const int nn = n0 + c32;
                uint32_t o[16];
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)((b + eh) * BN + c32), v);
                if (C1) {
                    // z = l (.) c, rounded to fp16 (the operand of contraction 2);
                    // every lane reads the same l (a shared-memory broadcast)
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        float4 lq;
                        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                     : "=f"(lq.x), "=f"(lq.y), "=f"(lq.z), "=f"(lq.w)
                                     : "r"(lsm + 4u * (uint32_t)(c32 + 4 * q4)));
                        const float z0 = __uint_as_float(v[4 * q4]) * lq.x, z1 = __uint_as_float(v[4 * q4 + 1]) * lq.y;
                        const float z2 = __uint_as_float(v[4 * q4 + 2]) * lq.z, z3 = __uint_as_float(v[4 * q4 + 3]) * lq.w;
                        if (MODE == 3 && p.out_bf16) {
                            o[2 * q4] = pack_bf162(z0, z1);
                            o[2 * q4 + 1] = pack_bf162(z2, z3);
                        } else {
                            overflow |= row_in && (beyond_f16(z0) | beyond_f16(z1) | beyond_f16(z2) | beyond_f16(z3));
                            o[2 * q4] = pack_half2(z0, z1);
                            o[2 * q4 + 1] = pack_half2(z2, z3);
                        }
                    }
                    if (MODE == 3 && p.aux != nullptr) {
                        // the column dot of the unscaled accumulator with aux
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            uint4 ax[2] = {make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
                            if (row_in) {
                                const uint4 *src = reinterpret_cast<const uint4 *>(
                                    static_cast<const uint16_t *>(p.aux) + (int64_t)(m0 + lane) * p.ldaux + nn + 16 * hh);
                                ax[0] = __ldg(src);
                                ax[1] = __ldg(src + 1);
                            }
                            const uint32_t aw[8] = {ax[0].x, ax[0].y, ax[0].z, ax[0].w,
                                                    ax[1].x, ax[1].y, ax[1].z, ax[1].w};
                            float pr[16];
                            if (p.aux_bf16) {
#pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    pr[j] = ((j & 1) ? hi_bf16(aw[j >> 1]) : lo_bf16(aw[j >> 1])) *
                                            __uint_as_float(v[16 * hh + j]);
                            } else {
#pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    pr[j] = ((j & 1) ? hi_f16(aw[j >> 1]) : lo_f16(aw[j >> 1])) *
                                            __uint_as_float(v[16 * hh + j]);
                            }
                            const float r = column_sum16(pr, lane);
                            if (m0 < p.M && lane < 16) p.part0[(int64_t)(m0 >> 5) * p.N + nn + 16 * hh + lane] = r;
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) o[q] = pack_bf162(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1]));
                }
                if (m0 >= p.M) continue;  // the warp's rows all lie past the matrix
                const uint32_t box = obox + (uint32_t)(nst % S::kOutBufs) * OUT_BYTES;
                const uint32_t rowa = box + (uint32_t)lane * 64;  // this lane's row of the box
                // the store that last used this box has finished reading it
                if (lane == 0) bulk_wait_read<S::kOutBufs - 1>();
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowa + (((uint32_t)q ^ rsw) << 4)),
                                 "r"(o[4 * q]), "r"(o[4 * q + 1]), "r"(o[4 * q + 2]), "r"(o[4 * q + 3])
                                 : "memory");
                fence_async_shared();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmOut, nn, m0, box);
                    bulk_commit();
                }
                ++nst;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (P == 2 && rank == 1)
                    mbar_arrive_remote(acce_lead + 8 * b);
                else
                    mbar_arrive(acce0 + 8 * b);
            }
        }
        if (lane == 0) bulk_wait_all();
        if (overflow) set_status(p.status, LB_ERR_RANGE);
    }

    tc_fence_before();
    __syncthreads();
    // P = 2: neither CTA leaves (or frees its half of tensor memory) while
    // the other may still arrive on its barriers or read its shared memory
    if (P == 2) cluster_sync();
    if (abort_flag && tid == 0) set_status(p.status, LB_ERR_DEVICE_TIMEOUT);
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        if constexpr (P == 2)
            tmem_dealloc_pair(tmem, TMEM_COLS);
        else
            tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
// The tile shape of one contraction, from a makespan model fitted to timings
// of this kernel on B200 (Qwen3-14B and Llama-2-7B shapes, 129 to 8192
// tokens).  A CTA (or each CTA of a pair) spends per K-block of a tile, in
// tenths of a nanosecond,
//   P = 1, H = 1:  max(4800, 2000 + 20 bn)    (two producer groups alternate)
//   P = 1, H = 2:  max(8000, 5500 + 18 bn)    (one group feeds both halves)
//   P = 2, H = 1:  max(4300, 2000 + 11 bn)    (each CTA expands bn / 2 rows)
//   P = 2, H = 2:  max(5000, 24.5 bn)
// where the constant floors are the latency of a stage's round trip (shorter
// for a pair, whose four producer groups each have four MMA periods per
// block) and the slopes the sign expansion and MMA, plus per tile 500 ns (H = 1: its
// epilogue overlaps the next tile), 3000 ns (P = 1, H = 2: both accumulators
// hold the one tile, so the MMA waits for its epilogue) or 5600 ns (P = 2,
// H = 2: the same for a 512-row tile, whose stores leave all SMs at once).
// The makespan is ceil(tiles / units) tiles, units being SMs (P = 1) or the
// pairs resident at once (P = 2).  Of the widths giving each column-tile count only the narrowest
// (rounded up to 32, the output box width) is worth trying; ties (plans whose
// blocks all sit at a floor) go to more tiles, i.e. less work per unit.
struct TilePlan {
    int H, bn, tiles;
    int P;  // CTAs per MMA
};

TilePlan plan_tiles(int M, int N, int K, int sms, int pairs)
{
    const long nk = (K + BK - 1) / BK;
    TilePlan best{1, BN, 0, 1};
    long best_cost = -1;
    for (int P = 1; P <= 2; ++P) {
        const int units = P == 1 ? sms : pairs;
        if (units <= 0) continue;
        for (int H = 1; H <= 2; ++H) {
            const int tm = (M + BM * H * P - 1) / (BM * H * P);
            for (int tn = (N + BN - 1) / BN; tn <= (N + 31) / 32; ++tn) {
                const int bn = ((N + tn - 1) / tn + 31) & ~31;
                if ((N + bn - 1) / bn != tn) continue;
                const int tiles = tm * tn, waves = (tiles + units - 1) / units;
                long per_block, per_tile;
                if (P == 1) {
                    per_block = H == 1 ? std::max(4800, 2000 + 20 * bn) : std::max(8000, 5500 + 18 * bn);
                    per_tile = H == 1 ? 5000 : 30000;
                } else {
                    per_block = H == 1 ? std::max(4300, 2000 + 11 * bn) : std::max(5000, 49 * bn / 2);
                    per_tile = H == 1 ? 5000 : 56000;
                }
                const long cost = (long)waves * (nk * per_block + per_tile);
                if (best_cost < 0 || cost < best_cost || (cost == best_cost && tiles > best.tiles)) {
                    best_cost = cost;
                    best = TilePlan{H, bn, tiles, P};
                }
            }
        }
    }
    return best;
}

// A persistent grid of `units` CTAs (P = 1) or CTA pairs (P = 2, clusters of two).
template <int MODE, int H, int P>
cudaError_t launch_units(const CUtensorMap &tm, const CUtensorMap &tmo, const SignGemmParams &p, int units,
                         cudaStream_t stream)
{
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(units * P));
    cfg.blockDim = dim3(Shape<H, P, MODE>::kThreads);
    cfg.dynamicSmemBytes = Shape<H, P, MODE>::kSmem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = P == 2 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, sign_gemm_kernel<MODE, H, P>, tm, tmo, p);
}

// One contraction on a persistent grid: min(tiles, SMs) CTAs, or
// min(tiles, resident pairs) CTA pairs.
// A is x (modes 1 and 3, bf16) or z (mode 2, fp16; bf16 with bf16_ops),
// row-major with stride lda.
template <int MODE>
cudaError_t launch_sign_gemm(SignGemmParams p, const void *a, int64_t lda, const DeviceInfo &dev,
                             cudaStream_t stream)
{
    constexpr bool C1 = MODE == 1 || MODE == 3;
    const int pairs = prefill_pairs_enabled() ? dev.pair_slots : 0;
    const TilePlan tp = plan_tiles(p.M, p.N, p.K, dev.sm_count, pairs);
    const int H = tp.H;
    p.bn = tp.bn;
    CUtensorMap tm, tmo;
    std::memset(&tmo, 0, sizeof(tmo));
    cudaError_t e = encode_2d(&tm, a, p.M, p.K, lda, C1 || p.bf16_ops, BM * H);
    // the output: z fp16 (modes 1, 3; mode 3 bf16 on request) or y bf16 (mode 2), [M x N], stride ldo
    if (e == cudaSuccess && p.out != nullptr)
        e = encode_store_2d(&tmo, p.out, p.M, p.N, p.ldo, !C1 || (MODE == 3 && p.out_bf16));
    if (e != cudaSuccess) return e;
    if (tp.P == 2) {
        const int units = std::min(tp.tiles, dev.pair_slots);
        return H == 2 ? launch_units<MODE, 2, 2>(tm, tmo, p, units, stream)
                      : launch_units<MODE, 1, 2>(tm, tmo, p, units, stream);
    }
    const int units = std::min(tp.tiles, dev.sm_count);
    return H == 2 ? launch_units<MODE, 2, 1>(tm, tmo, p, units, stream)
                  : launch_units<MODE, 1, 1>(tm, tmo, p, units, stream);
}

}  // namespace

namespace {

// Opts a kernel into its shared memory; for pair kernels also counts the
// clusters of two that fit on the device at once (the fewest of any kernel).
template <int MODE, int H, int P>
cudaError_t prepare_kernel(DeviceInfo &dev)
{
    cudaError_t e = cudaFuncSetAttribute(sign_gemm_kernel<MODE, H, P>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Shape<H, P, MODE>::kSmem);
    if (e != cudaSuccess || P == 1) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)dev.sm_count);
    cfg.blockDim = dim3(Shape<H, P, MODE>::kThreads);
    cfg.dynamicSmemBytes = Shape<H, P, MODE>::kSmem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, sign_gemm_kernel<MODE, H, P>, &cfg);
    if (e != cudaSuccess) return e;
    dev.pair_slots = dev.pair_slots == 0 ? clusters : std::min(dev.pair_slots, clusters);
    return cudaSuccess;
}

}  // namespace

cudaError_t prefill_prepare_device(DeviceInfo &dev)
{
    cudaError_t e = get_encoder();
    dev.pair_slots = 0;
    if (e == cudaSuccess) e = prepare_kernel<1, 1, 1>(dev);
    if (e == cudaSuccess) e = prepare_kernel<2, 1, 1>(dev);
    if (e == cudaSuccess) e = prepare_kernel<1, 2, 1>(dev);
    if (e == cudaSuccess) e = prepare_kernel<2, 2, 1>(dev);
    if (e == cudaSuccess) e = prepare_kernel<1, 1, 2>(dev);
    if (e == cudaSuccess) e = prepare_kernel<2, 1, 2>(dev);
    if (e == cudaSuccess) e = prepare_kernel<1, 2, 2>(dev);
    if (e == cudaSuccess) e = prepare_kernel<2, 2, 2>(dev);
    // the backward pass's modes
    if (e == cudaSuccess) e = prepare_kernel<3, 1, 1>(dev);
    if (e == cudaSuccess) e = prepare_kernel<3, 2, 1>(dev);
    if (e == cudaSuccess) e = prepare_kernel<3, 1, 2>(dev);
    if (e == cudaSuccess) e = prepare_kernel<3, 2, 2>(dev);
    return e;
}

size_t prefill_workspace_bytes(int tokens, const int *ranks, int npaths)
{
    const size_t R = (size_t)ranks[0] + (npaths > 1 ? ranks[1] : 0);
    return (size_t)tokens * R * 2 + 256;
}

cudaError_t prefill_latent(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, uint16_t *z, int64_t ldz)
{
    const int M = a.tokens;
    const int r0 = a.path[0].rank, r1 = a.npaths > 1 ? a.path[1].rank : 0;
    const int R = r0 + r1;
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;

    // contraction 1: Z = (X . B1^T) (.) l
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
    p1.ldo = ldz;
    p1.status = dev.status;
    return launch_sign_gemm<1>(p1, a.x, a.ldx, dev, stream);
}

cudaError_t prefill_expand(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream, const uint16_t *z,
                           int64_t ldz)
{
    const int M = a.tokens;
    const int r0 = a.path[0].rank, r1 = a.npaths > 1 ? a.path[1].rank : 0;
    const int R = r0 + r1;
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;

    // contraction 2: Y = Z . B2^T
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
    return launch_sign_gemm<2>(p2, z, ldz, dev, stream);
}

cudaError_t bwd_contraction1(const Bwd1Args &b, const DeviceInfo &dev, cudaStream_t stream)
{
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    SignGemmParams p{};
    p.M = b.M;
    p.N = b.r0 + b.r1;
    p.K = b.K;
    p.r0 = b.r0;
    p.bits8 = even8(b.bits0, b.ld0) && (b.bits1 == nullptr || even8(b.bits1, b.ld1));
    p.bits0 = b.bits0;
    p.bld0 = b.ld0;
    p.s0 = b.s0;
    p.l0 = b.l0;
    if (b.bits1 != nullptr) {
        p.bits1 = b.bits1;
        p.bld1 = b.ld1;
        p.s1 = b.s1;
        p.l1 = b.l1;
    }
    p.out = b.out;
    p.ldo = b.ldo;
    p.status = dev.status;
    p.aux = b.aux;
    p.ldaux = b.ldaux;
    p.part0 = b.part;
    p.out_bf16 = b.out_bf16;
    p.aux_bf16 = b.aux_bf16;
    return launch_sign_gemm<3>(p, b.a, b.lda, dev, stream);
}

cudaError_t bwd_dx(const BwdDxArgs &b, const DeviceInfo &dev, cudaStream_t stream)
{
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    // contraction 2 in bf16: dx = A . B^T, B[i, k] = sign(V_p[i, k]) bf16(g_p[i])
    SignGemmParams p{};
    p.M = b.M;
    p.N = b.n_in;
    p.K = b.r0 + b.r1;
    p.r0 = b.r0;
    p.bits8 = even8(b.bits0, b.ld0) && (b.bits1 == nullptr || (b.r0 % 64 == 0 && even8(b.bits1, b.ld1)));
    p.bits0 = b.bits0;
    p.bld0 = b.ld0;
    p.s0 = b.g0;
    if (b.bits1 != nullptr) {
        p.bits1 = b.bits1;
        p.bld1 = b.ld1;
        p.s1 = b.g1;
    }
    p.out = b.dx;
    p.ldo = b.lddx;
    p.status = dev.status;
    p.bf16_ops = 1;
    return launch_sign_gemm<2>(p, b.a, b.lda, dev, stream);
}

cudaError_t prefill_forward(const ForwardArgs &a, const DeviceInfo &dev, cudaStream_t stream)
{
    const int R = a.path[0].rank + (a.npaths > 1 ? a.path[1].rank : 0);
    uint16_t *z = static_cast<uint16_t *>(a.workspace);  // [M x R] fp16
    const cudaError_t e = prefill_latent(a, dev, stream, z, R);
    return e != cudaSuccess ? e : prefill_expand(a, dev, stream, z, R);
}

}  // namespace lb
