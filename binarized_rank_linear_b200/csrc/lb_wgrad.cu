// lb_wgrad.cu - the h-gradient of the backward pass as a weight-gradient
// product on the tensor cores.
//
// With e_p = S_U,p (l_p (.) c_p) (sesamedisk.com, "Samsung LittleBit 13B
// Model", "What the method actually computes", Proposition 1, run backward by
// the chain rule),
//     dh_p[o] = sum_m dy[m, o] e_p[m, o] = sum_k sign(U_p[o, k]) l_p[k] G[o, k],
//     G = dy^T c   ([n_out x R], the tokens m as the contraction dimension),
// so the sum over tokens runs inside the MMA and each output row's sum over k
// is a per-lane epilogue: no column dot across rows, and no product tile
// stored.  G's rows o are the accumulator's lanes; its columns k run over the
// latents of both paths (path 0 below r0).
//
// Both operands are MN-major: dy [tokens x n_out] and c [tokens x R] are
// row-major with the tokens outermost, so a K-block (64 tokens) of A is 64
// rows of 128 bytes for each 64 columns o, and the same for B along k.  TMA
// brings them in with 128-byte swizzle, boxes of 64 (MN) x 64 (tokens); the
// shared-memory descriptors then step 8192 bytes between 64-wide MN chunks
// (leading byte offset) and 1024 bytes between 8-token groups (stride byte
// offset), and an MMA of K = 16 tokens starts 2048 bytes further on.
//
// Persistent single-CTA tiles of 128 rows o x bn columns k, optionally split
// over the tokens into `nsplit` parts; a unit (tile, part) leaves one partial
// per row and path, [ntn * nsplit][n_out] per path, which the caller adds in
// a fixed order.  Warp 0 issues the TMA loads, warp 1 the MMAs, warps 2..5
// drain the two double-buffered accumulators.
#include <algorithm>
#include <cstdint>
#include <cuda_runtime.h>

#include "lb_common.cuh"
#include "lb_internal.h"
#include "lb_tc.cuh"

namespace lb {
namespace {

using namespace tc;

constexpr int WM = 128;                     // rows o per tile (one MMA, M = 128)
constexpr int WBN = 256;                    // widest tile along k
constexpr int WBK = 64;                     // tokens per K-block
constexpr uint32_t BOX = 64 * 64 * 2;       // one TMA box: 64 MN x 64 tokens, 8 KB
constexpr uint32_t W_A = (WM / 64) * BOX;   // 16 KB
constexpr uint32_t W_B = (WBN / 64) * BOX;  // 32 KB
constexpr int WSTAGES = 4;
constexpr int kWThreads = 32 * 6;
constexpr size_t kWSmem = 1024 + (size_t)WSTAGES * (W_A + W_B) + 256;

struct WgradParams {
    int M;       // rows o (n_out)
    int N;       // columns k (R = r0 + r1)
    int K;       // tokens
    int bn;      // tile width along k: a multiple of 32, at most WBN
    int nsplit;  // parts of the token range per tile
    int kps;     // K-blocks per part (the last may be shorter)
    int r0;      // columns k below r0 are path 0
    const uint32_t *u0, *u1;  // packed rows of U_p (bit j of word w: column 32 w + j negative)
    int64_t uld0, uld1;
    const uint16_t *l0, *l1;  // latent scales (fp16)
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

__global__ void __launch_bounds__(kWThreads, 1)
    wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const WgradParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sA = base, sB = base + WSTAGES * W_A;
    const uint32_t bars = sB + WSTAGES * W_B;
    // full[WSTAGES], empty[WSTAGES], acc_full[2], acc_empty[2], drain, then the tmem address
    const uint32_t full0 = bars, empty0 = bars + 8 * WSTAGES, accf0 = bars + 16 * WSTAGES;
    const uint32_t acce0 = accf0 + 16, drain = acce0 + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem_raw + (drain + 8 - raw));
    __shared__ int abort_shared;
    volatile int &abort_flag = abort_shared;

    const int tiles_m = (p.M + WM - 1) / WM, tiles_n = (p.N + p.bn - 1) / p.bn;
    const int nk = (p.K + WBK - 1) / WBK;
    const int units = tiles_m * tiles_n * p.nsplit;
    const int G = gridDim.x, c = blockIdx.x;
    const int my_units = c < units ? (units - c + G - 1) / G : 0;
    // unit t: rows (t % tiles_m), then columns, then the token part
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
                mbar_init(acce0 + 8 * b, 4);
            }
            mbar_init(drain, 1);
            abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), 512);
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA: A (dy^T) and B (c) boxes of each K-block
        if (lane == 0) {
            int gb = 0, issued = 0;
            for (int i = 0; i < my_units && !abort_flag; ++i) {
                const int t = c + i * G;
                const int o0 = (t % tiles_m) * WM, k0 = ((t / tiles_m) % tiles_n) * p.bn;
                const int nb = (p.bn + 63) / 64;
                int kb0, kb1;
                unit_kb(t, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb, ++gb) {
                    const int s = gb % WSTAGES;
                    const uint32_t ph = (uint32_t)(gb / WSTAGES) & 1u;
                    if (!mbar_wait(empty0 + 8 * s, ph ^ 1u) || abort_flag) {
                        abort_flag = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(full0 + 8 * s, (uint32_t)(WM / 64 + nb) * BOX);
                    for (int j = 0; j < WM / 64; ++j)
                        tma_load_2d(sA + s * W_A + j * BOX, &tmA, o0 + 64 * j, kb * WBK, full0 + 8 * s);
                    for (int j = 0; j < nb; ++j)
                        tma_load_2d(sB + s * W_B + j * BOX, &tmB, k0 + 64 * j, kb * WBK, full0 + 8 * s);
                    ++issued;
                }
            }
            if (abort_flag)
                for (int q = (issued > WSTAGES ? issued - WSTAGES : 0); q < issued; ++q)
                    mbar_wait(full0 + 8 * (q % WSTAGES), (uint32_t)(q / WSTAGES) & 1u);
        }
    } else if (warp == 1) {
        // ---------------- MMA: unit i accumulates in columns 256 (i % 2) ..
        if (lane == 0) {
            // bf16 operands, fp32 accumulate, A and B MN-major, M = 128, N = bn
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                   ((uint32_t)(p.bn >> 3) << 17) | ((uint32_t)(WM >> 4) << 24);
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
                        umma(acc, ad, bd, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
                    }
                    umma_commit(empty0 + 8 * s);
                }
                if (abort_flag) break;
                umma_commit(accf0 + 8 * b);
            }
            umma_commit(drain);
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
            const int tn = (t / tiles_m) % tiles_n, sp = t / (tiles_m * tiles_n);
            const int o = (t % tiles_m) * WM + 32 * quad + lane;
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
                const float lj = f16_bits_to_float(lv[kl + lane]);
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
            if (lane == 0) mbar_arrive(acce0 + 8 * b);
            if (o < p.M) {
                const int64_t row = (int64_t)(tn * p.nsplit + sp) * p.M + o;
                p.part0[row] = s0;
                if (p.part1 != nullptr) p.part1[row] = s1;
            }
        }
    }
    __syncthreads();
    if (abort_flag && threadIdx.x == 0) set_status(p.status, LB_ERR_DEVICE_TIMEOUT);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

// Tile width, token split and partial count of the h-gradient product for
// n_out rows, R latent columns and `tokens` tokens on `sms` SMs.
WgradPlan wgrad_plan(int n_out, int R, int tokens, int sms)
{
    WgradPlan w{};
    const int ntn = (R + WBN - 1) / WBN;
    w.bn = ((R + ntn - 1) / ntn + 31) & ~31;
    w.ntn = (R + w.bn - 1) / w.bn;
    const int tiles = ((n_out + WM - 1) / WM) * w.ntn;
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
    return cudaFuncSetAttribute(wgrad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWSmem);
}

cudaError_t wgrad_dh(const WgradArgs &w, const DeviceInfo &dev, cudaStream_t stream)
{
    cudaError_t e = get_encoder();
    if (e != cudaSuccess) return e;
    const WgradPlan pl = wgrad_plan(w.n_out, w.R, w.tokens, dev.sm_count);
    CUtensorMap ta, tb;
    // dy: [tokens x n_out], MN (n_out) contiguous; c: [tokens x R]
    e = encode_2d(&ta, w.dy, w.tokens, w.n_out, w.lddy, true, 64);
    if (e == cudaSuccess) e = encode_2d(&tb, w.c, w.tokens, w.R, w.ldc, true, 64);
    if (e != cudaSuccess) return e;
    WgradParams p{};
    p.M = w.n_out;
    p.N = w.R;
    p.K = w.tokens;
    p.bn = pl.bn;
    p.nsplit = pl.nsplit;
    p.kps = pl.kps;
    p.r0 = w.r0;
    p.u0 = w.u0;
    p.u1 = w.u1;
    p.uld0 = w.uld0;
    p.uld1 = w.uld1;
    p.l0 = w.l0;
    p.l1 = w.l1;
    p.part0 = w.part0;
    p.part1 = w.part1;
    p.status = dev.status;
    const int units = ((w.n_out + WM - 1) / WM) * pl.ntn * pl.nsplit;
    const int grid = std::min(units, dev.sm_count);
    wgrad_kernel<<<grid, kWThreads, kWSmem, stream>>>(ta, tb, p);
    return cudaGetLastError();
}

}  // namespace lb
