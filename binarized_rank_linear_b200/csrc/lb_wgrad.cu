// lb_wgrad.cu - the scale gradients dh and dg of the backward pass as
// weight-gradient products on the tensor cores.
//
// Run backward by the chain rule, the layer's five steps (sesamedisk.com,
// "Samsung LittleBit 13B Model", "What the method actually computes",
// Proposition 1) give, per path p, with c = S_V^T (g (.) x) and
// a = S_U^T (h (.) dy),
//     dh_p[o] = sum_m dy[m, o] e_p[m, o] = sum_k sign(U_p[o, k]) l_p[k] G[o, k],   G = dy^T c,
//     dg_p[i] = sum_m x[m, i] dt_p[m, i] = sum_k sign(V_p[i, k]) H[i, k],          H = x^T (l (.) a),
// so the sum over tokens runs inside the MMA and each row's sum over k is a
// per-lane epilogue: no column dot across rows, and no product tile stored.
// The product's rows are the accumulator's lanes; its columns k run over the
// latents of both paths (path 0 below r0).
//
// Both operands are MN-major: A [tokens x rows] and B [tokens x R] are
// row-major with the tokens outermost, so a K-block (64 tokens) of A is 64
// rows of 128 bytes for each 64 rows of the product, and the same for B along
// k.  TMA brings them in with 128-byte swizzle, boxes of 64 (MN) x 64
// (tokens); the shared-memory descriptors then step 8192 bytes between
// 64-wide MN chunks (leading byte offset) and 1024 bytes between 8-token
// groups (stride byte offset), and an MMA of K = 16 tokens starts 2048 bytes
// further on.
//
// Persistent tiles of 256 rows o on a CTA pair (cta_group::2: CTA r holds
// rows 128 r .. of A and columns bn r / 2 .. of B; CTA 0 issues the MMAs),
// or of 128 rows on single CTAs, x bn columns k, optionally split over the
// tokens into `nsplit` parts; a unit (tile, part) leaves one partial per row
// and path, [ntn * nsplit][rows] per path, which the caller adds in a fixed
// order.  Warp 0 issues the TMA loads, warp 1 the MMAs, warps 2..5 drain the
// two double-buffered accumulators.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"
#include "lb_tc.cuh"

namespace lb {
namespace {

using namespace tc;

constexpr int WM = 128;                     // rows o per CTA (M = 128; a pair's MMA: 256)
constexpr int WBN = 256;                    // widest tile along k
constexpr int WBK = 64;                     // tokens per K-block
constexpr uint32_t BOX = 64 * 64 * 2;       // one TMA box: 64 MN x 64 tokens, 8 KB
constexpr uint32_t W_A = (WM / 64) * BOX;   // 16 KB: this CTA's rows of A
constexpr int kWThreads = 32 * 6;
// P = 1: a CTA stages all bn columns of B; P = 2: half of them (the pair's
// MMA takes columns 0 .. bn/2 - 1 from CTA 0 and the rest from CTA 1)
// (P = 2 leaves one stage's B bytes free after the last stage: what the
// MMA reads from a stage then lies inside the allocation whichever half of
// B it takes.)
template <int P>
struct WShape {
    static constexpr uint32_t kB = (WBN / P / 64) * BOX;  // 32 or 16 KB
    static constexpr uint32_t kPad = P == 2 ? kB : 0;
    static constexpr int kStages = P == 1 ? 4 : 6;
    static constexpr size_t kSmem = 1024 + (size_t)kStages * (W_A + kB) + kPad + 256;
};

struct WgradParams {
    int M;       // rows o of the product
    int N;       // columns k (R = r0 + r1)
    int K;       // tokens
    int bn;      // tile width along k: a multiple of 32, at most WBN
    int nsplit;  // parts of the token range per tile
    int kps;     // K-blocks per part (the last may be shorter)
    int r0;      // columns k below r0 are path 0
    const uint32_t *u0, *u1;  // packed rows of S_p (bit j of word w: column 32 w + j negative)
    int64_t uld0, uld1;
    const uint16_t *l0, *l1;  // latent scales (fp16), or null for 1
    float *part0, *part1;     // [ceil(N / bn) * nsplit][M] per path
    int *status;
};

// Shared-memory descriptor of an MN-major operand with 128-byte swizzle:
// 64-element MN chunks `lbo` bytes apart, 8-row K groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_mn(uint32_t addr, uint32_t lbo)
{
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}

template <int P>
__global__ void __launch_bounds__(kWThreads, 1)
    wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const WgradParams p)
{
    constexpr int WSTAGES = WShape<P>::kStages;
    constexpr uint32_t W_B = WShape<P>::kB;
    constexpr int PM = WM * P;  // rows o of a (pair's) tile
    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sA = base, sB = base + WSTAGES * W_A;
    const uint32_t bars = sB + WSTAGES * W_B + WShape<P>::kPad;
    // full[WSTAGES], empty[WSTAGES], acc_full[2], acc_empty[2], drain, then the tmem address
    const uint32_t full0 = bars, empty0 = bars + 8 * WSTAGES, accf0 = bars + 16 * WSTAGES;
    const uint32_t acce0 = accf0 + 16, drain = acce0 + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + (drain + 8 - raw));
    __shared__ int abort_shared;
    volatile int &abort_flag = abort_shared;

    const int rank = P == 2 ? (int)cluster_rank() : 0;
    const int tiles_m = (p.M + PM - 1) / PM, tiles_n = (p.N + p.bn - 1) / p.bn;
    const int nk = (p.K + WBK - 1) / WBK;
    const int units = tiles_m * tiles_n * p.nsplit;
    const int G = gridDim.x / P, c = blockIdx.x / P;  // persistent units: CTAs, or pairs
    const int my_units = c < units ? (units - c + G - 1) / G : 0;
    // unit t: columns (t % tiles_n), then rows, then the token part, so the
    // units running at once share their rows of A (the larger operand) in L2
    auto unit_kb = [&](int t, int &kb0, int &kb1) {
        const int sp = t / (tiles_m * tiles_n);
        kb0 = sp * p.kps;
        kb1 = min(nk, kb0 + p.kps);
    };

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < WSTAGES; ++s) {
                mbar_init(full0 + 8 * s, 1);
                mbar_init(empty0 + 8 * s, 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(accf0 + 8 * b, 1);
                mbar_init(acce0 + 8 * b, 4 * P);  // every epilogue warp (of the pair)
            }
            mbar_init(drain, 1);
            abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        if constexpr (P == 2)
            tmem_alloc_pair(smem_u32(tmem_slot), 512);
        else
            tmem_alloc(smem_u32(tmem_slot), 512);
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
        // ---------------- TMA: the A and B boxes of each K-block
        if (lane == 0) {
            int gb = 0, issued = 0;
            // this CTA's columns of B: all bn (P = 1), or half from bn/2 rank on
            const int bw = p.bn / P, nb = (bw + 63) / 64;
            const uint32_t stage_bytes = (uint32_t)(WM / 64 + nb) * BOX;
            for (int i = 0; i < my_units && !abort_flag; ++i) {
                const int t = c + i * G;
                const int o0 = ((t / tiles_n) % tiles_m) * PM + rank * WM;
                const int k0 = (t % tiles_n) * p.bn + rank * bw;
                int kb0, kb1;
                unit_kb(t, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++gb) {
                    const int s = gb % WSTAGES;
                    const uint32_t ph = (uint32_t)(gb / WSTAGES) & 1u;
                    if (!mbar_wait(empty0 + 8 * s, ph ^ 1u) || abort_flag) {
                        abort_flag = 1;
                        break;
                    }
                    if (P == 1) {
                        mbar_arrive_expect_tx(full0 + 8 * s, stage_bytes);
                        for (int j = 0; j < WM / 64; ++j)
                            tma_load_2d(sA + s * W_A + j * BOX, &tmA, o0 + 64 * j, kb * WBK, full0 + 8 * s);
                        for (int j = 0; j < nb; ++j)
                            tma_load_2d(sB + s * W_B + j * BOX, &tmB, k0 + 64 * j, kb * WBK, full0 + 8 * s);
                    } else {
                        // both CTAs' bytes complete on CTA 0's barrier, which CTA 0 arms
                        if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * s, 2 * stage_bytes);
                        for (int j = 0; j < WM / 64; ++j)
                            tma_load_2d_pair(sA + s * W_A + j * BOX, &tmA, o0 + 64 * j, kb * WBK, full_lead + 8 * s);
                        for (int j = 0; j < nb; ++j)
                            tma_load_2d_pair(sB + s * W_B + j * BOX, &tmB, k0 + 64 * j, kb * WBK, full_lead + 8 * s);
                    }
                    ++issued;
                }
            }
            if (abort_flag && P == 2 && rank == 1) {
                // this CTA cannot wait on CTA 0's barriers: give copies in
                // flight time to land (they take microseconds)
                const unsigned long long t0 = globaltimer();
                while (globaltimer() - t0 < 200000ull) {
                }
            } else if (abort_flag) {
                for (int q = (issued > WSTAGES ? issued - WSTAGES : 0); q < issued; ++q)
                    mbar_wait(full0 + 8 * (q % WSTAGES), (uint32_t)(q / WSTAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA: unit i accumulates in columns 256 (i % 2) ..
        // P = 2: CTA 0 issues the pair's MMAs and signals both CTAs; CTA 1
        // only waits for the last of them before it may free tensor memory.
        if (lane == 0 && P == 2 && rank == 1) {
            if (!mbar_wait(drain, 0)) abort_flag = 1;
        } else if (lane == 0) {
            // bf16 operands, fp32 accumulate, A and B MN-major, M = 128 P, N = bn
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                   ((uint32_t)(p.bn >> 3) << 17) | ((uint32_t)(PM >> 4) << 24);
            auto commit = [&](uint32_t bar) {
                if constexpr (P == 2)
                    umma_commit_pair(bar);
                else
                    umma_commit(bar);
            };
            int gb = 0;
            for (int i = 0; i < my_units && !abort_flag; ++i) {
                const int t = c + i * G;
                const int b = i & 1, use = i >> 1;
                int kb0, kb1;
                unit_kb(t, kb0, kb1);
                if (!mbar_wait(acce0 + 8 * b, (uint32_t)(use & 1) ^ 1u)) {
                    abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(b * WBN);
                for (int kb = kb0; kb < kb1; ++kb, ++gb) {
                    const int s = gb % WSTAGES;
                    const uint32_t ph = (uint32_t)(gb / WSTAGES) & 1u;
                    if (!mbar_wait(full0 + 8 * s, ph) || abort_flag) {
                        abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < WBK / 16; ++kk) {  // 16 tokens: 2048 bytes further on
                        const uint64_t ad = smem_desc_mn(sA + s * W_A + (uint32_t)kk * 2048u, BOX);
                        const uint64_t bd = smem_desc_mn(sB + s * W_B + (uint32_t)kk * 2048u, BOX);
                        const uint32_t acc_flag = (kb != kb0 || kk != 0) ? 1u : 0u;
                        if constexpr (P == 2)
                            umma_pair(acc, ad, bd, idesc, acc_flag);
                        else
                            umma(acc, ad, bd, idesc, acc_flag);
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
    } else {
        // ---------------- epilogue: warp w drains lanes 32 (w % 4) .. of the
        // accumulator; lane = row o.  Per 32-column chunk: the row's sign word
        // and the chunk's 32 scales (one per lane, broadcast by shuffles).
        const int quad = warp & 3;
        for (int i = 0; i < my_units; ++i) {
            const int t = c + i * G;
            const int b = i & 1, use = i >> 1;
            const int tn = t % tiles_n, sp = t / (tiles_m * tiles_n);
            const int o = ((t / tiles_n) % tiles_m) * PM + rank * WM + 32 * quad + lane;
            const int k0 = tn * p.bn;
            bool ok = !abort_flag && mbar_wait(accf0 + 8 * b, (uint32_t)(use & 1));
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                abort_flag = 1;
                break;
            }
            tc_fence_after();
            float s0 = 0.0f, s1 = 0.0f;
            for (int c32 = 0; c32 < p.bn && k0 + c32 < p.N; c32 += 32) {
                const int k = k0 + c32;
                const bool sec = k >= p.r0;
                const int kl = sec ? k - p.r0 : k;  // column within the path (a multiple of 32)
                const uint16_t *lv = sec ? p.l1 : p.l0;
                const float lj = lv != nullptr ? f16_bits_to_float(lv[kl + lane]) : 1.0f;
                const uint32_t word = o < p.M ? __ldg((sec ? p.u1 + (int64_t)o * p.uld1 : p.u0 + (int64_t)o * p.uld0) + (kl >> 5))
                                              : 0u;
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(b * WBN + c32), v);
                float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float lb = __shfl_sync(0xffffffffu, lj, j);
                    const float prod = lb * __uint_as_float(v[j]);
                    const float sgn = __uint_as_float(__float_as_uint(prod) ^ ((word << (31 - j)) & 0x80000000u));
                    if (j & 1)
                        a1 += sgn;
                    else
                        a0 += sgn;
                }
                if (sec)
                    s1 += a0 + a1;
                else
                    s0 += a0 + a1;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (P == 2 && rank == 1)
                    mbar_arrive_remote(acce_lead + 8 * b);
                else
                    mbar_arrive(acce0 + 8 * b);
            }
            if (o < p.M) {
                const int64_t row = (int64_t)(tn * p.nsplit + sp) * p.M + o;
                p.part0[row] = s0;
                if (p.part1 != nullptr) p.part1[row] = s1;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    // P = 2: neither CTA leaves (or frees its half of tensor memory) while
    // the other may still arrive on its barriers or read its shared memory
    if (P == 2) cluster_sync();
    if (abort_flag && threadIdx.x == 0) set_status(p.status, LB_ERR_DEVICE_TIMEOUT);
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        if constexpr (P == 2)
            tmem_dealloc_pair(tmem, 512);
        else
            tmem_dealloc(tmem, 512);
    }
}

}  // namespace

// Tile width, token split and partial count of the product for `rows` rows,
// R latent columns and `tokens` tokens on `sms` SMs.  The plan is
// made for CTA pairs (256-row tiles, sms / 2 of them at once) and kept for
// single CTAs, so both give the same token parts and the same sums.
WgradPlan wgrad_plan(int rows, int R, int tokens, int sms)
{
    WgradPlan w{};
    const int ntn = (R + WBN - 1) / WBN;
    w.bn = ((R + ntn - 1) / ntn + 31) & ~31;
    w.ntn = (R + w.bn - 1) / w.bn;
    const int tiles = ((rows + 2 * WM - 1) / (2 * WM)) * w.ntn;
    sms = std::max(1, sms / 2);
    const int nk = std::max(1, (tokens + WBK - 1) / WBK);
    // makespan in K-blocks: waves x (blocks per part + a unit's fixed cost of
    // about two K-blocks); at most wgrad_max_parts parts
    long best = -1;
    w.nsplit = 1;
    w.kps = nk;
    for (int ns = 1; ns <= std::min(nk, wgrad_max_parts(R, tokens) / w.ntn); ++ns) {
        const int kps = (nk + ns - 1) / ns;
        if ((ns - 1) * kps >= nk) continue;  // a part would be empty
        const long waves = (tiles * (long)ns + sms - 1) / sms;
        const long cost = waves * (kps + 2);
        if (best < 0 || cost < best) {
            best = cost;
            w.nsplit = ns;
            w.kps = kps;
        }
    }
    w.rows = w.ntn * w.nsplit;
    return w;
}

int wgrad_max_parts(int R, int tokens)
{
    return std::max((tokens + 31) / 32, (R + 31) / 32);
}

cudaError_t wgrad_prepare_device(const DeviceInfo &dev)
{
    (void)dev;
    cudaError_t e = cudaFuncSetAttribute(wgrad_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)WShape<1>::kSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(wgrad_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)WShape<2>::kSmem);
    return e;
}

cudaError_t wgrad_scale_grad(const WgradArgs &w, const DeviceInfo &dev, cudaStream_t stream)
{
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    const WgradPlan pl = wgrad_plan(w.rows, w.R, w.tokens, dev.sm_count);
    CUtensorMap ta, tb;
    // A: [tokens x rows], B: [tokens x R], both with the rows or columns contiguous
    e = encode_2d(&ta, w.a, w.tokens, w.rows, w.lda, true, 64);
    if (e == cudaSuccess) e = encode_2d(&tb, w.b, w.tokens, w.R, w.ldb, true, 64);
    if (e != cudaSuccess) return e;
    WgradParams p{};
    p.M = w.rows;
    p.N = w.R;
    p.K = w.tokens;
    p.bn = pl.bn;
    p.nsplit = pl.nsplit;
    p.kps = pl.kps;
    p.r0 = w.r0;
    p.u0 = w.bits0;
    p.u1 = w.bits1;
    p.uld0 = w.bld0;
    p.uld1 = w.bld1;
    p.l0 = w.l0;
    p.l1 = w.l1;
    p.part0 = w.part0;
    p.part1 = w.part1;
    p.status = dev.status;
    if (prefill_pairs_enabled() && dev.pair_slots > 0) {
        const int units = ((w.rows + 2 * WM - 1) / (2 * WM)) * pl.ntn * pl.nsplit;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3((unsigned)(2 * std::min(units, dev.pair_slots)));
        cfg.blockDim = dim3(kWThreads);
        cfg.dynamicSmemBytes = WShape<2>::kSmem;
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, wgrad_kernel<2>, ta, tb, p);
    }
    const int units = ((w.rows + WM - 1) / WM) * pl.ntn * pl.nsplit;
    wgrad_kernel<1><<<std::min(units, dev.sm_count), kWThreads, WShape<1>::kSmem, stream>>>(ta, tb, p);
    return cudaGetLastError();
}

}  // namespace lb
