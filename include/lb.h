/*
 * lb.h - C ABI of the LittleBit factored linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer.  LittleBit replaces a dense weight W [n_out x n_in] by binarized
 * low-rank factors and three scale vectors (sesamedisk.com, "Samsung LittleBit
 * 13B Model", section "How low-rank binarization works"; littlebitllm.com,
 * section "The method"):
 *
 *     W ~= diag(h) . sign(U) . diag(l) . sign(V)^T . diag(g)
 *
 * with U [n_out x r], V [n_in x r], h the row scale [n_out], g the column
 * scale [n_in] and l the latent scale [r].  The forward pass is taken in the
 * factored order of Proposition 1 (sesamedisk.com, section "What the method
 * actually computes"), per token x [n_in]:
 *
 *     y = h (.) ( sign(U) . ( l (.) ( sign(V)^T . ( g (.) x ) ) ) )
 *
 * With residual compensation a second path (U2, V2, h2, g2, l2) of the same
 * form is added to the first (sesamedisk.com, "How low-rank binarization
 * works", last paragraph; littlebitllm.com, "Pipeline", step 04).  The rank
 * per path follows from the bit budget (see lb_rank_for_budget).
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library never allocates, frees or synchronises inside lb_pack_signs or
 *     lb_linear_forward; both only enqueue work on `stream`.
 *   - `stream` is a cudaStream_t passed as a plain pointer (NULL = the legacy
 *     default stream).  The current CUDA device must own every pointer.
 *   - bf16 and fp16 values travel as their 16-bit patterns (uint16_t).
 *   - Arguments are checked on the host before anything is enqueued.  On any
 *     error nothing is launched and no output byte is written.
 *   - Every call is thread-safe; the library keeps only per-device cached
 *     attributes and one device status word per device (lb_device_status).
 *   - There is no CPU fallback: without a usable sm_100 device the compute
 *     calls return LB_ERR_NOT_SUPPORTED_DEVICE or LB_ERR_CUDA.
 */
#ifndef LB_H
#define LB_H

#include <stddef.h>
#include <stdint.h>

/* Symbols of the shared library are exported explicitly; everything else in
 * it is hidden. */
#if defined(LB_BUILDING) && defined(__GNUC__)
#define LB_API __attribute__((visibility("default")))
#else
#define LB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LB_OK = 0,
    LB_ERR_INVALID_ARGUMENT = 1,   /* null pointer, negative size, bad enum   */
    LB_ERR_UNSUPPORTED_SHAPE = 2,  /* a size outside what the kernels take    */
    LB_ERR_MISALIGNED = 3,         /* a pointer or stride breaks an alignment */
    LB_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed    */
    LB_ERR_DEVICE_TIMEOUT = 5,     /* a device-side wait gave up (async)      */
    LB_ERR_NOT_SUPPORTED_DEVICE = 6, /* the current device is not sm_100    */
    LB_ERR_WORKSPACE_TOO_SMALL = 7,  /* workspace_bytes below the query    */
    LB_ERR_RANGE = 8               /* an fp16 operand overflowed (async)      */
} lb_status;

typedef enum { LB_F32 = 0, LB_F16 = 1, LB_BF16 = 2, LB_I8 = 3 } lb_dtype;

/* Which factor a packed matrix holds.
 *   LB_FACTOR_U: source U [n_out x r]; packed rows are U's rows, packed along r.
 *   LB_FACTOR_V: source V [n_in x r]; packed rows are V^T's rows (one per
 *                latent index k), packed along n_in.                          */
typedef enum { LB_FACTOR_U = 0, LB_FACTOR_V = 1 } lb_factor;

/* One binarized path of the layer.  All pointers are device memory.
 *   u_bits : packed sign(U),   [n_out x u_ld] uint32 words (LB_FACTOR_U)
 *   vt_bits: packed sign(V)^T, [rank  x vt_ld] uint32 words (LB_FACTOR_V)
 *   h, g, l: fp16 row scale [n_out], column scale [n_in], latent scale [rank]
 *   rank   : r of this path
 *   u_ld, vt_ld: words per packed row; 0 means lb_packed_ld_words(rank) and
 *            lb_packed_ld_words(n_in).  Any value >= those is accepted.      */
typedef struct lb_path {
    const uint32_t *u_bits;
    const uint32_t *vt_bits;
    const uint16_t *h;
    const uint16_t *g;
    const uint16_t *l;
    int64_t rank;
    int64_t u_ld;
    int64_t vt_ld;
} lb_path;

/* Human-readable name of a status code (static storage, never NULL). */
LB_API const char *lb_status_string(lb_status status);

/* Packed layout.  Word w of a packed row holds columns 32w .. 32w+31; bit j
 * (value 1u << j) is 1 iff column 32w + j is -1.  The pages fix one bit per
 * factor entry, each entry +1 or -1 (sesamedisk.com, "How low-rank
 * binarization works"); the word layout is this library's own.  Unused bits
 * of the last word of a row, and any words past it up to the row's stride,
 * are written as 0.
 *
 * Returns ceil(cols / 32), the smallest legal stride in words (rows are
 * dense, 4-byte aligned), or -1 if cols <= 0. */
LB_API int64_t lb_packed_ld_words(int64_t cols);

/* Bytes of a packed factor at the smallest stride:
 *   LB_FACTOR_U: n_out rows x lb_packed_ld_words(rank) words x 4
 *   LB_FACTOR_V: rank rows  x lb_packed_ld_words(n_in) words x 4
 * `n_in_or_out` is n_out for U and n_in for V.  Returns 0 on a bad argument. */
LB_API size_t lb_packed_bytes(lb_factor kind, int64_t n_in_or_out, int64_t rank);

/* Rank per path from the bit budget.  The budget is eff * n_in * n_out sign
 * bits (linear layers only, scale vectors not counted: littlebitllm.com,
 * section "How small"); a path of rank r stores r * (n_in + n_out) of them
 * ("the rank sets the bit budget", sesamedisk.com, "How low-rank binarization
 * works"), and the residual path shares the same budget (same section).  So
 *     *rank = floor(eff_num * n_in * n_out / (eff_den * paths * (n_in + n_out)))
 * rounded down to a multiple of `align`, in exact integer arithmetic
 * (eff = eff_num / eff_den as a fraction, never a float).
 * Host only.  Errors: LB_ERR_INVALID_ARGUMENT for non-positive sizes, paths
 * outside {1, 2}, align < 1, a null `rank`, or products that overflow int64;
 * LB_ERR_UNSUPPORTED_SHAPE when the result would be 0 (*rank is then 0). */
LB_API lb_status lb_rank_for_budget(int64_t n_in, int64_t n_out, int64_t eff_num, int64_t eff_den,
                             int paths, int align, int64_t *rank);

/* Pack a factor's signs into the layout above, on `stream`.
 *   src      : device, `rows` rows of `cols` elements, row stride `src_ld`
 *              elements (>= cols), element type `dtype`.
 *              LB_FACTOR_U: src is U, rows = n_out, cols = r.
 *              LB_FACTOR_V: src is V, rows = n_in,  cols = r.
 *   dst      : device, LB_FACTOR_U: [rows x dst_ld_words]; LB_FACTOR_V:
 *              [cols x dst_ld_words] (V^T).  dst_ld_words >=
 *              lb_packed_ld_words(packed row length).  Every word of every
 *              destination row is written.
 * An element is -1 (bit 1) iff it is strictly negative: +0, -0 and NaN give
 * bit 0, -inf and negative subnormals bit 1 (the pages only say each entry is
 * +1 or -1; this is the library's reading, tested bit-exactly).
 * Alignment: src 4-byte aligned for f32, 2 for f16/bf16; dst 4-byte aligned.
 * One-off weight preparation, not on the forward path. */
LB_API lb_status lb_pack_signs(const void *src, lb_dtype dtype, lb_factor kind, int64_t rows,
                        int64_t cols, int64_t src_ld, uint32_t *dst, int64_t dst_ld_words,
                        void *stream);

/* Workspace that lb_linear_forward needs for these sizes (rank_residual = 0
 * without the residual path).  Holds the latent between the two contractions.
 * Returns 0 on a bad argument; a valid call may also need 0 bytes. */
LB_API size_t lb_forward_workspace_bytes(int64_t tokens, int64_t n_in, int64_t n_out,
                                  int64_t rank_main, int64_t rank_residual);

/* The layer's forward pass (Proposition 1, both paths fused), on `stream`.
 *   x        : device bf16 [tokens x n_in], row stride ldx elements
 *   main     : the primary path (required)
 *   residual : the residual path, or NULL for none
 *   y        : device bf16 [tokens x n_out], row stride ldy elements; written,
 *              never read.  y = sum over paths of h (.) sign(U)(l (.) sign(V)^T (g (.) x)),
 *              computed with fp32 accumulation and rounded to bf16 (nearest even).
 *   workspace: device scratch of at least lb_forward_workspace_bytes(...) bytes,
 *              16-byte aligned; its contents on entry do not matter.  Calls
 *              that share a workspace must be ordered on one stream.
 * Shapes: n_in, n_out and every rank a positive multiple of 32; ldx >= n_in,
 *   ldy >= n_out, both multiples of 8.  tokens >= 0; tokens == 0 is a no-op
 *   (nothing launched, pointers unchecked).
 * Alignment: x, y, u_bits, vt_bits, h, g, l and workspace 16-byte aligned.
 * Numerics: all sums accumulate in fp32 and y is rounded to bf16 once.
 *   1..4 tokens run on CUDA cores in fp32 throughout.  More tokens run on
 *   the tensor cores: contraction 1 with bf16 operands (x as given, g
 *   rounded to bf16), contraction 2 with fp16 operands (the latent z rounded
 *   to fp16, h exact); z must stay below 65504 in magnitude (else
 *   LB_ERR_RANGE is raised on the device status word and y is undefined).
 * Errors: LB_ERR_INVALID_ARGUMENT (null pointers, negative sizes),
 *   LB_ERR_UNSUPPORTED_SHAPE, LB_ERR_MISALIGNED, LB_ERR_WORKSPACE_TOO_SMALL,
 *   LB_ERR_NOT_SUPPORTED_DEVICE, LB_ERR_CUDA (launch failure).  Conditions
 *   found while the kernels run are reported by lb_device_status. */
LB_API lb_status lb_linear_forward(const uint16_t *x, int64_t tokens, int64_t n_in, int64_t n_out,
                            int64_t ldx, const lb_path *main, const lb_path *residual,
                            uint16_t *y, int64_t ldy, void *workspace, size_t workspace_bytes,
                            void *stream);

/* ---------------------------------------------------------- split halves
 * The two halves of lb_linear_forward on their own, with the r-wide latent
 * in caller memory.  For factorised key and value projections a model can
 * cache this latent instead of the full-width keys and values (sesamedisk.com,
 * "Samsung LittleBit 13B Model", section "The real result": the KV cache
 * shrinks because the smaller latent state is cached).
 *
 * Latent layout: z fp16 [tokens x ldz], row-major (token-major), row stride
 * ldz elements >= r_main + r_residual and a multiple of 8; row m holds the
 * main path's r_main latents, then the residual path's.  16-byte aligned.
 *
 * lb_latent_forward (steps 1-3 of Proposition 1):
 *     z[m][off_p + k] = l_p[k] * sum_i sign(V_p[i][k]) * g_p[i] * x[m][i]
 *   Uses vt_bits, vt_ld, g, l and rank of each path (u_bits and h are not
 *   read and may be NULL).  x as in lb_linear_forward.
 * lb_expand_forward (steps 4-5):
 *     y[m][o] = sum_p h_p[o] * sum_k sign(U_p[o][k]) * z[m][off_p + k]
 *   Uses u_bits, u_ld, h and rank (vt_bits, g and l are not read and may be
 *   NULL).  y as in lb_linear_forward.
 * Numerics (any number of tokens, all on the tensor cores): contraction 1 in
 *   bf16 x bf16 (g rounded to bf16), contraction 2 in fp16 x fp16 (h
 *   exact), fp32 accumulation; z is rounded to fp16 (nearest even) and must
 *   stay below 65504 in magnitude (else LB_ERR_RANGE on the device status
 *   word and z is undefined); y is rounded to bf16 once.
 * No workspace; nothing is allocated.  Errors as lb_linear_forward; tokens
 *   == 0 is a no-op.  A z written by lb_latent_forward and read by
 *   lb_expand_forward on the same stream needs no other synchronisation. */
LB_API lb_status lb_latent_forward(const uint16_t *x, int64_t tokens, int64_t n_in, int64_t ldx,
                            const lb_path *main, const lb_path *residual, uint16_t *z, int64_t ldz,
                            void *stream);
LB_API lb_status lb_expand_forward(const uint16_t *z, int64_t tokens, int64_t n_out, int64_t ldz,
                            const lb_path *main, const lb_path *residual, uint16_t *y, int64_t ldy,
                            void *stream);

/* ---------------------------------------------------------- host buffers
 * lb_linear_forward_host: the layer on x in host memory, y back to host
 * memory, in one call on `stream`: an asynchronous copy of x into x_dev, the
 * forward pass of lb_linear_forward on x_dev into y_dev, an asynchronous copy
 * of y_dev into y_host (one cudaMemcpyAsync each way).  For callers whose
 * activations live on the host; the library allocates nothing, so the device
 * buffers are the caller's.
 * For 1-128 tokens, when both host buffers are pinned memory mapped into the
 * device's address space (page-locked allocations are, with unified
 * addressing), x reaches x_dev through a kernel that reads it from host
 * memory in one pass instead of a copy, and the last kernel writes y into
 * y_host directly, leaving y_dev untouched: the same bytes cross the host
 * link, inside the kernel chain.  The result is the same to the bit.
 *   x_host : bf16 [tokens x n_in], rows contiguous (row stride n_in); pinned
 *            (page-locked) memory for the copy to be asynchronous
 *   y_host : bf16 [tokens x n_out], rows contiguous; pinned likewise.  Valid
 *            once the stream has reached the end of the call.
 *   x_dev, y_dev : device scratch of tokens x n_in and tokens x n_out bf16,
 *            16-byte aligned; their contents on entry do not matter
 *   the rest as lb_linear_forward (x_dev and y_dev take the roles of x and y,
 *   with ldx = n_in and ldy = n_out).
 * Errors as lb_linear_forward; LB_ERR_INVALID_ARGUMENT for a null host
 *   pointer.  A copy that fails to start returns LB_ERR_CUDA. */
LB_API lb_status lb_linear_forward_host(const uint16_t *x_host, int64_t tokens, int64_t n_in, int64_t n_out,
                                 const lb_path *main, const lb_path *residual, uint16_t *y_host,
                                 uint16_t *x_dev, uint16_t *y_dev, void *workspace, size_t workspace_bytes,
                                 void *stream);

/* ---------------------------------------------------------- sibling projections
 * Several layers that read the same input x, computed together: the query,
 * key and value projections of an attention block, or the gate and up
 * projections of an MLP.  Each is a LittleBit layer of its own (its own
 * factors, scales, ranks and output width; Proposition 1 of sesamedisk.com,
 * "Samsung LittleBit 13B Model", section "What the method actually
 * computes"); grouping them changes only how the work is launched, so that a
 * decoder block pays the launch and dependency latency once per group
 * instead of once per layer (littlebitllm.com, "How small": the speed claims
 * are per layer on a memory-bound decode).
 *
 * lb_projection: one layer of the group.
 *   n_out    : its output width (positive multiple of 32)
 *   main, residual : its paths, as for lb_linear_forward (residual may be NULL)
 *   y, ldy   : its output, device bf16 [tokens x ldy], ldy >= n_out, a multiple
 *              of 8, 16-byte aligned; written, never read.
 * lb_linear_forward_siblings: for every projection j,
 *     y_j = sum over its paths p of h_p (.) sign(U_p)(l_p (.) sign(V_p)^T (g_p (.) x)),
 *   the result of lb_linear_forward on x and that projection alone, with the
 *   same numerics (1..4 tokens: fp32 throughout on CUDA cores; more tokens:
 *   the tensor-core numerics of lb_linear_forward).  The output buffers must
 *   not overlap each other, x or the workspace.
 *   nproj: 1 .. LB_MAX_SIBLINGS.  Up to 128 tokens the whole group runs as one
 *   pair of launches; more tokens run each projection's own launches in turn.
 *   workspace: at least lb_siblings_workspace_bytes(...) bytes, 16-byte
 *   aligned, as for lb_linear_forward.
 * Errors as lb_linear_forward; additionally LB_ERR_INVALID_ARGUMENT for a bad
 *   nproj or a null proj.  Nothing is launched on an error found on the host. */
#define LB_MAX_SIBLINGS 4
typedef struct {
    int64_t n_out;
    const lb_path *main;
    const lb_path *residual;
    uint16_t *y;
    int64_t ldy;
} lb_projection;

/* Workspace for lb_linear_forward_siblings; 0 on a bad argument. */
LB_API size_t lb_siblings_workspace_bytes(int64_t tokens, int64_t n_in, int nproj, const lb_projection *proj);
LB_API lb_status lb_linear_forward_siblings(const uint16_t *x, int64_t tokens, int64_t n_in, int64_t ldx,
                                     int nproj, const lb_projection *proj, void *workspace,
                                     size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------- backward pass
 * lb_linear_backward: the gradients of a loss L with respect to the layer's
 * input and to every path's scale vectors, given dy = dL/dy.  The pages train
 * the layer by quantization-aware training through the factored pass
 * (littlebitllm.com, "Pipeline"; trove.briskstack.com, "How it works"), whose
 * steps are those of Proposition 1 (sesamedisk.com, "Samsung LittleBit 13B
 * Model", "What the method actually computes").  With the signs held fixed,
 * the chain rule through those steps gives, per path p and summed over tokens
 * m where marked:
 *     a_p  = sign(U_p)^T (h_p (.) dy)                (d L / d z_p)
 *     dl_p = sum_m a_p (.) c_p,    c_p = sign(V_p)^T (g_p (.) x)
 *     dt_p = sign(V_p) (l_p (.) a_p)                  (d L / d (g_p (.) x))
 *     dg_p = sum_m x (.) dt_p,     dx = sum_p g_p (.) dt_p
 *     dh_p = sum_m dy (.) e_p,     e_p = sign(U_p) (l_p (.) c_p)
 * The gradient through sign() to the real-valued factors needs the smooth
 * surrogate the pages name (SmoothSign) but do not define; it is not computed.
 *   x       : device bf16 [tokens x n_in], row stride ldx (the forward input)
 *   dy      : device bf16 [tokens x n_out], row stride lddy
 *   main, residual : the paths exactly as for lb_linear_forward (the same
 *             packed words; the call transposes them into the workspace)
 *   dx      : device bf16 [tokens x n_in], row stride lddx, or NULL for none;
 *             written, never read
 *   dh      : device fp32 [paths x n_out]: path 0's n_out values, then path 1's
 *   dg      : device fp32 [paths x n_in], the same order
 *   dl      : device fp32 [r_main + r_residual]: path 0's latents first
 *   workspace : at least lb_backward_workspace_bytes(...) bytes, 16-byte
 *             aligned, contents on entry irrelevant; calls sharing it must be
 *             ordered on one stream
 * Numerics: tensor-core products with fp32 accumulation, bf16 operands.
 *   c = S_V^T (g (.) x) and a = S_U^T (h (.) dy) (g and h rounded to bf16)
 *   are kept in bf16, a scaled by l; dh and dg come from dy^T c and x^T a
 *   with the tokens as the contraction, dx from a against V with g rounded
 *   to bf16.  Every sum runs in a fixed order (dl: 32-token blocks, then the
 *   blocks in order; dh, dg: the tokens inside the MMA, then tile columns and
 *   token parts in order): results are deterministic.  dx is rounded to bf16
 *   once; dh, dg and dl are fp32.
 * Shapes, alignment and strides as lb_linear_forward (dx like x; dh, dg, dl
 *   4-byte aligned).  tokens == 0 sets dh, dg and dl to zero and nothing else
 *   (x, dy and dx are then not read and may be NULL).
 * Errors: LB_ERR_INVALID_ARGUMENT (null pointers other than dx, negative
 *   sizes, short strides), LB_ERR_UNSUPPORTED_SHAPE, LB_ERR_MISALIGNED,
 *   LB_ERR_WORKSPACE_TOO_SMALL, LB_ERR_NOT_SUPPORTED_DEVICE, LB_ERR_CUDA; on
 *   an error found on the host nothing is launched and nothing is written. */
LB_API size_t lb_backward_workspace_bytes(int64_t tokens, int64_t n_in, int64_t n_out, int64_t rank_main,
                                          int64_t rank_residual);
LB_API lb_status lb_linear_backward(const uint16_t *x, const uint16_t *dy, int64_t tokens, int64_t n_in,
                                    int64_t n_out, int64_t ldx, int64_t lddy, const lb_path *main,
                                    const lb_path *residual, uint16_t *dx, int64_t lddx, float *dh, float *dg,
                                    float *dl, void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------- fixed scratch
 * lb_linear_forward_fixed_scratch: lb_linear_forward for 1..32 tokens with
 * no workspace argument.  The pages have no counterpart; this is a service of
 * this library.
 *
 * It is meant for callers that cannot give the library device memory at call
 * time: a plain C host program with no device allocator of its own, a
 * runtime that reserves all of its device memory once under a fixed budget,
 * or a latency-critical loop in which allocating (and the device-wide
 * synchronisation that cudaMalloc and cudaFree imply) is not allowed.  The
 * call allocates nothing.  The scratch it uses is a fixed array of
 * LB_FIXED_SCRATCH_BYTES that is part of the library's device code, one per
 * device.
 *
 * Arguments, results, numerics and errors are those of lb_linear_forward
 * without `workspace` / `workspace_bytes`, with these differences:
 *   - tokens must be 0..32 (the decode path); more -> LB_ERR_UNSUPPORTED_SHAPE;
 *   - a shape whose lb_forward_workspace_bytes exceeds LB_FIXED_SCRATCH_BYTES
 *     -> LB_ERR_WORKSPACE_TOO_SMALL (nothing is launched);
 *   - the first call on each device looks up the array's device address
 *     (once; later calls reuse it).  Make that first call, with the device
 *     current, before any stream capture.  If the lookup fails the call
 *     returns LB_ERR_CUDA;
 *   - `stream` must belong to the current device (NULL, the legacy default
 *     stream, always does): the array used is the current device's.  A
 *     stream of another device -> LB_ERR_INVALID_ARGUMENT.
 * Nothing in the array has to start at zero: each call writes every byte it
 * later reads.  All calls on one device share the one array, so two calls
 * that could run at the same time (different streams, or different host
 * threads without ordering between them) race and give undefined results;
 * order them, e.g. on one stream. */
#define LB_FIXED_SCRATCH_BYTES (1u << 20)
LB_API lb_status lb_linear_forward_fixed_scratch(const uint16_t *x, int64_t tokens, int64_t n_in,
                                          int64_t n_out, int64_t ldx, const lb_path *main,
                                          const lb_path *residual, uint16_t *y, int64_t ldy,
                                          void *stream);

/* Synchronise `stream`, then read and clear the current device's status word,
 * which kernels set when a device-side condition stops them (a bounded wait
 * that gave up, an fp16 overflow).  *out receives LB_OK or the first such
 * condition.  Returns LB_ERR_CUDA if the synchronisation itself fails. */
LB_API lb_status lb_device_status(void *stream, lb_status *out);

/* Whether the prefill contractions (more than 128 tokens) may run on CTA
 * pairs: thread-block clusters of two SMs that share each tensor-core MMA
 * (the default, 1), or only on single-CTA tiles (0).  Both give the same
 * results to the bit; pairs are faster wherever the device can co-schedule
 * them.  The setting is process-wide and applies to calls made after it
 * returns; a call already enqueued keeps the kernels it was given.  Returns
 * LB_ERR_INVALID_ARGUMENT unless `enable` is 0 or 1. */
LB_API lb_status lb_set_prefill_pairs(int enable);

/* Fault injection, for tests of the library's own failure handling; not
 * for production use.  No counterpart on the pages.
 * With enable = 1, every tcgen05 decode kernel (5..128 tokens) enqueued
 * afterwards gives up its bounded waits after wait_limit_ns (1 us .. 2 s)
 * instead of 2 s, and in each of them one producer warp of the first CTA
 * skips its arrival on its first stage barrier.  The MMA thread's wait on
 * that barrier then runs out: the kernel records LB_ERR_DEVICE_TIMEOUT on the
 * device status word, lets its copies and MMAs finish, frees its tensor
 * memory and returns (no trap, no hang); the outputs of such a call are
 * undefined.  enable = 0 restores the defaults for later calls.  The setting
 * is process-wide.  Errors: LB_ERR_INVALID_ARGUMENT for enable outside
 * {0, 1} or a limit outside the range. */
LB_API lb_status lb_debug_inject_stall(int enable, uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* LB_H */
