/*
 * gptq.h -- C ABI of libgptq.so: the GPTQ-family per-layer compensation solve on
 * NVIDIA B200 (sm_100a).
 *
 * Sources (cited by page title and section):
 *   [GPTQ blog] "GPTQ：量化一个权重之后怎样补偿输出误差" (charlestar.github.io)
 *   [ResComp]   "Rethinking Residual Errors in Compensation-based LLM Quantization"
 *               (papernotes.org), "关键设计" items 1-3
 *   [GPTAQ]     "GPTAQ: Efficient Finetuning-Free Quantization for Asymmetric
 *               Calibration" (Paper-Notes), "关键设计"
 *   [G2PTQ]     "G²PTQ: Improving LLM Post-Training Quantization with Generalized
 *               Gradient Compensation" (agihunt.info summary)
 *
 * Conventions shared by every call
 *   - All pointers named as device buffers are CUDA device memory owned by the
 *     caller. The library allocates nothing; scratch comes from a caller
 *     workspace of gptq_workspace_size() bytes (256-byte aligned).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream). No call synchronises the host.
 *   - The return value reports argument errors (GPTQ_ERR_ARG, GPTQ_ERR_WORKSPACE)
 *     and launch errors (GPTQ_ERR_CUDA) synchronously; nothing has been enqueued
 *     when it is not GPTQ_OK.
 *   - Numerical failures are found on the device and written to a caller-owned
 *     device int32 `status` word: the first failing kernel stores its
 *     gptq_status code there, later kernels of any call given the same word see
 *     a non-zero value and skip their work. The caller zeroes the word before a
 *     chain of calls and reads it after synchronising. This follows the blog's
 *     self-check ("用标准库核对二维补偿"), which refuses non-finite or non-PD input
 *     instead of repairing it.
 *   - Layout: W is nn.Linear order W[N][K] row-major (N output channels, K input
 *     coordinates): the blog's K x N weight matrix stored column-major, so row n
 *     is output channel n ([GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法" on
 *     N x K versus K x N). Token streams X are row-major [M][K].
 *   - Matrices named K x K are fp32 row-major with leading dimension K; a stack of
 *     g of them is contiguous, [g][K][K].
 */
#ifndef GPTQ_H
#define GPTQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GPTQ_API __attribute__((visibility("default")))
#else
#define GPTQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GPTQ_OK = 0,
    GPTQ_ERR_ARG = 1,        /* invalid argument (size, pointer, alignment, option) */
    GPTQ_ERR_NOT_PD = 2,     /* a Cholesky pivot is not clearly positive after damping */
    GPTQ_ERR_NONFINITE = 3,  /* NaN or Inf in an input or an intermediate */
    GPTQ_ERR_CUDA = 4,       /* a CUDA launch or API call failed */
    GPTQ_ERR_TIMEOUT = 5,    /* a bounded device wait ran out */
    GPTQ_ERR_WORKSPACE = 6,  /* workspace missing, misaligned or too small */
    GPTQ_ERR_BOUNDS = 7      /* an index check of the GPTQ_DEBUG_BOUNDS build failed (the
                                access was skipped); see gptq_bounds_report */
} gptq_status;

typedef enum { GPTQ_BF16 = 0, GPTQ_F32 = 1 } gptq_dtype;

/* Largest K (input coordinates) and N (output channels) any call accepts. */
#define GPTQ_MAX_DIM 65535

typedef enum {
    GPTQ_OP_PREPARE = 0,
    GPTQ_OP_RESIDUAL = 1,
    GPTQ_OP_QUANTIZE = 2,
    GPTQ_OP_QUANTIZE_GROUPED = 3,
    GPTQ_OP_FIRST_ORDER = 4
} gptq_op;

/* OR-ed into GPTQ_OP_QUANTIZE or GPTQ_OP_QUANTIZE_GROUPED: the workspace of a call
 * with cae != 0 (one more fp32 copy of W). */
#define GPTQ_WS_CAE 0x100

/*
 * gptq_accumulate_hessian -- H[g] += 2 * X^T diag(w[g]) X over one token chunk.
 *
 * [GPTQ blog] "Calibration 让量化看见输入方向": the layer objective's Hessian is
 * 2 X^T X, shared by all output channels and accumulated batch by batch without
 * keeping activations (factor 2 fixed by the two-weight example of "两个权重怎样互相补偿").
 * [G2PTQ]: with output-channel groups each group g has its own Hessian; here a
 * group's per-token weight w[g][m] scales token m's outer product.
 *
 *   H      device fp32 [g][K][K]; accumulated into (the caller zeroes it before the
 *          first chunk). Full symmetric storage is written: each entry above the
 *          diagonal and its mirror receive the same partial sums, in separate fp32
 *          reductions, so the two triangles agree to fp32 rounding (gptq_prepare
 *          reads the upper one).
 *   K      input coordinates, >= 1; bf16 streams need K % 8 == 0.
 *   g      number of Hessians (>= 1). With w == NULL, g must be 1.
 *   X      device [M][ldx] tokens, dtype xdtype. bf16: X and ldx 16-byte aligned
 *          (ldx % 8 == 0). ldx >= K.
 *   M      tokens in this chunk (>= 0; 0 is a no-op).
 *   w      device fp32 [g][ldw] per-token weights, or NULL for unit weights.
 *   status device int32 or NULL (see conventions): GPTQ_ERR_TIMEOUT if a bounded
 *          wait inside the tensor-core kernel ran out; the call is skipped when the
 *          word is already non-zero.
 *   Errors: GPTQ_ERR_ARG for bad sizes/alignment/dtype, GPTQ_ERR_CUDA on launch.
 *   Paths: bf16 streams with K >= 64 run on the tensor cores (tcgen05, TMA); with
 *   weights, each token's s * x is formed in fp32 and split into a bf16 pair so the
 *   product keeps ~16 bits. fp32 streams run the fp32 SIMT kernel.
 */
GPTQ_API gptq_status gptq_accumulate_hessian(float *H, int K, int g, const void *X, int xdtype,
                                    int64_t M, int64_t ldx, const float *w, int64_t ldw,
                                    int32_t *status, void *stream);

/*
 * gptaq_accumulate_cross -- C += 2 * (X_fp - X_q)^T X_q over one token chunk.
 *
 * [ResComp] item 2: r1 = w (X~ - X) with X~ the full-precision stream and X the
 * quantised stream; item 3 precomputes the cross statistic dX X^T (their row
 * convention; dX^T X here). The difference X_fp - X_q is formed exactly in fp32 on
 * the device from the two inputs, so no rounded dX is ever stored.
 *
 *   C      device fp32 [K][K], accumulated into (caller zeroes it first). Not
 *          symmetric: C[i][j] = 2 sum_m dX[m][i] X_q[m][j].
 *   X_fp, X_q  device [M][ldx] each, same dtype and leading dimension; alignment
 *          rules as gptq_accumulate_hessian.
 *   status device int32 or NULL, as in gptq_accumulate_hessian.
 *   bf16 streams with K >= 64 run on the tensor cores (the difference is split into
 *   a bf16 pair); fp32 streams run the fp32 SIMT kernel.
 */
GPTQ_API gptq_status gptaq_accumulate_cross(float *C, int K, const void *X_fp, const void *X_q,
                                   int xdtype, int64_t M, int64_t ldx, int32_t *status,
                                   void *stream);

/*
 * gptq_prepare -- dead coordinates, damping and the upper factor U, in place.
 *
 * [GPTQ blog] "Damping 与两个不同的分组参数": coordinates with H_kk == 0 are dead
 * (their diagonal is set to 1 here; their weights are zeroed by
 * gptq_quantize_layer), then H += percdamp * mean(diag H) * I.
 * "为什么 Cholesky Factor 不能当作原始逆矩阵": U is upper triangular with
 * U^T U = H^-1; row q of U carries the free-set inverse at q's step.
 * Computed as H = R R^T with R upper (Cholesky of the index-reversed matrix),
 * U = R^-1 (triangular inversion): no explicit H^-1 is formed. K a multiple of 32
 * from 256 up takes the tensor-core path (tf32 x3 products) when the workspace is
 * the size gptq_workspace_size() reports; other K, or a smaller workspace that
 * still holds the fp32 SIMT path's scratch (the damped diagonal and one level of
 * the inverse), take that SIMT path. Both give U to fp32 accuracy.
 *
 *   H        device fp32 [g][K][K] symmetric (the upper triangle is read). On
 *            return it holds U per group: upper triangle U, strict lower zero.
 *   percdamp >= 0 (0.01 is the pages' default).
 *   dead_out device uint8 [g][K] (1 = dead), or NULL.
 *   ws       device workspace of gptq_workspace_size(GPTQ_OP_PREPARE, K, 0, g, 0).
 *   status   device int32 (see conventions). GPTQ_ERR_NONFINITE for NaN/Inf in H,
 *            GPTQ_ERR_NOT_PD when a pivot p_j <= K * 2^-23 * Hd_jj (Hd the damped
 *            matrix): the pivot is below the factorisation's rounding size.
 *   Threads: the tensor-core path overlaps steps on a second stream of the library's
 *   own, with events ordering it against `stream`; that stream and its events are
 *   kept per (device, caller stream), so calls from several host threads on
 *   different streams are independent (each with its own workspace). Calls on one
 *   stream from several threads enqueue one at a time under a lock.
 */
GPTQ_API gptq_status gptq_prepare(float *H, int K, int g, float percdamp, uint8_t *dead_out,
                         void *ws, size_t ws_bytes, int32_t *status, void *stream);

/*
 * gptq_prepare_noalloc -- gptq_prepare without a caller workspace.
 *
 * The pages have no counterpart of this call; it exists for callers that cannot
 * allocate device memory when they need the factor, for example code running
 * inside a host application that owns every device allocation through its own
 * pool and hands plug-ins no workspace, or a latency-critical path that must not
 * take the device-wide synchronisation of cudaMalloc / cudaFree. It takes the same
 * arguments as gptq_prepare minus the workspace and allocates nothing: its scratch is
 * a fixed 16 MiB + 64 KiB array in the library's device memory, which every GPU that
 * loads the library holds until the process exits.
 *
 *   Path: the array stands in for gptq_prepare's workspace. Where gptq_prepare's full
 *   workspace fits it (K a multiple of 32 from 256 to 896 with g = 1, to 864 with
 *   g = 2, to 800 with g = 4) the call takes the tensor-core path with the same
 *   kernels as gptq_prepare; other sizes take the fp32 SIMT path, whose U agrees with
 *   gptq_prepare's to fp32 accuracy (not bit for bit).
 *   Limit: the SIMT path's scratch (the damped diagonal and one level of the
 *   triangular inverse, g groups) must fit the array: K <= 4096 with g = 1,
 *   K <= 2048 with g <= 4. Larger sizes return GPTQ_ERR_ARG before anything is
 *   enqueued.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before
 *   any stream capture.
 *   Sharing: every call on a device uses the same array, and the array keeps the
 *   last call's contents (nothing in it needs to start at zero). Calls whose
 *   kernels overlap on the GPU (for example on two streams at once) race on the
 *   array: serialise them.
 */
GPTQ_API gptq_status gptq_prepare_noalloc(float *H, int K, int g, float percdamp,
                                          uint8_t *dead_out, int32_t *status, void *stream);

/*
 * gptaq_residual -- P1 = [(C U^T) ⊙ M] U with M the strict upper mask.
 *
 * [ResComp] item 3: P1 = [(dX X^T L) ⊙ M_U] L^T with H^-1 = L L^T, i.e. L = U^T in
 * this layout; the strict mask makes row q equal C[q, F'] (H[F', F'])^-1 over the
 * coordinates after q ([GPTAQ] "基于最优脑压缩的闭式解"), the residual term the
 * sweep adds as w_q * P1[q, q+1:].
 *
 *   P1  device fp32 [K][K] output (strict upper; lower triangle and diagonal 0).
 *   C   device fp32 [K][K] from gptaq_accumulate_cross.
 *   U   device fp32 [K][K] from gptq_prepare (g = 1).
 *   ws  gptq_workspace_size(GPTQ_OP_RESIDUAL, K, 0, 1, 0) bytes.
 */
GPTQ_API gptq_status gptaq_residual(float *P1, const float *C, const float *U, int K, void *ws,
                           size_t ws_bytes, void *stream);

/*
 * gptq_quantize_layer -- the shared-order sweep with lazy blocks.
 *
 * [GPTQ blog] "GPTQ 怎样把逐个补偿变成可扩展算法": all channels take coordinates in
 * the same order; for coordinate j, q = s (c - z) with
 * c = clamp(round_half_even(w_j / s) + z, 0, 2^b - 1), E_j = (w_j - q) / U_jj, and
 * W_k -= U_jk E_j for the block's later k at once; at the block end the far
 * coordinates get W_far -= U[blk, far]^T E_blk. With P1 the GPTAQ row term
 * w_j^pre * P1[j, k] is added the same way.
 * With cae != 0 the compensation-aware error term of [ResComp] "关键设计" items 1-3
 * is added too: the row (w_j^(0) - w_j^pre) * P2[j, k], P2 = [((H + C) U^T) ⊙ M] U
 * with H the undamped Gram and C the GPTAQ cross statistic (C = 0 without P1), and
 * w^(0) the weights the sweep starts from (dead coordinates zeroed). P2 is not an
 * argument: as U^T U is the inverse of H plus a diagonal, P2 = P1 + I - diag(U)^-1 U
 * exactly, so the call needs only U (and P1).
 * Scale: per output channel s = 2 max_k |W[n][k]| / (2^b - 1) from W as given
 * (before dead coordinates are zeroed), s = 1 for an all-zero channel; zero
 * point z = 2^(b-1) ([G2PTQ] symmetric per-channel; [GPTQ blog] 4-bit grid
 * {-8..7} as codes 0..15 with zero point 8).
 *
 *   W          device [N][K] weights, dtype wdtype. Read; overwritten with the
 *              reconstruction s (c - z) when write_back != 0.
 *   U          device fp32 [groups][K][K] from gptq_prepare; channel n uses
 *              group n / (N / groups).
 *   groups     1..8, N % groups == 0.
 *   bits       2, 3, 4 or 8.  blocksize 16, 32, 64 or 128.
 *   P1         device fp32 [K][K] from gptaq_residual, or NULL (plain GPTQ).
 *              Requires groups == 1.
 *   cae        0, or 1 for the compensation-aware error term (any groups).
 *   dead       device uint8 [groups][K] from gptq_prepare, or NULL (none dead).
 *   scales_in  device fp32 [N] fixed scales, or NULL (min-max as above).
 *   scales_out device fp32 [N] the scales used, or NULL.
 *   codes      device uint8 [N][K] codes c (required).
 *   loss       device fp32 [N] with 1/2 sum_j E_j^2 per channel, or NULL; E_j is the
 *              rounding error of the value quantised, (w_j^pre - q) / U_jj, with or
 *              without cae.
 *   ws         gptq_workspace_size(GPTQ_OP_QUANTIZE | (cae ? GPTQ_WS_CAE : 0), K, N,
 *              groups, blocksize) bytes.
 *   status     device int32: GPTQ_ERR_NONFINITE for NaN/Inf in W or scales.
 */
GPTQ_API gptq_status gptq_quantize_layer(void *W, int wdtype, int N, int K, const float *U, int groups,
                                int bits, int blocksize, const float *P1, int cae,
                                const uint8_t *dead,
                                const float *scales_in, float *scales_out, uint8_t *codes,
                                float *loss, int write_back, void *ws, size_t ws_bytes,
                                int32_t *status, void *stream);

/*
 * gptq_act_order -- the act-order processing order of the input coordinates.
 *
 * [GPTQ blog] "Damping 与两个不同的分组参数": act-order processes the input
 * coordinates by the Hessian diagonal from large to small; they are restored after
 * quantisation. perm[q] is the coordinate fixed at step q: decreasing H_kk, ties by
 * lower index. Call it on the accumulated H (before gptq_prepare), so dead
 * coordinates (H_kk = 0) come last.
 *
 *   H     device fp32 [K][K] (read).
 *   perm  device int32 [K] (written).
 *   Errors: GPTQ_ERR_ARG for K out of range or NULL pointers.
 */
GPTQ_API gptq_status gptq_act_order(const float *H, int K, int32_t *perm, void *stream);

/*
 * gptq_permute_hessian -- out[i][j] = H[perm[i]][perm[j]] (K x K fp32, out of place):
 * the Hessian (or the GPTAQ cross statistic C) in the processing order, for
 * gptq_prepare / gptaq_residual ahead of an ordered quantisation.
 *
 *   out, H  device fp32 [K][K], distinct buffers.  perm  device int32 [K].
 */
GPTQ_API gptq_status gptq_permute_hessian(float *out, const float *H, int K, const int32_t *perm,
                                          void *stream);

/*
 * gptq_quantize_layer_grouped -- gptq_quantize_layer with input-dimension groups and
 * an optional processing order (one Hessian, groups == 1).
 *
 * [GPTQ blog] "Damping 与两个不同的分组参数": blocksize organises the computation,
 * groupsize changes the representation: each output channel takes one scale per
 * group of input coordinates; the group parameters are either re-estimated during
 * compensation or fixed beforehand (static groups); with act-order the coordinates,
 * the group index and the permutation are restored consistently.
 *   - static_groups == 0: groups are processing positions [gG, (g+1)G); when the
 *     sweep enters group g, s[n][g] = 2 max |w| / (2^b - 1) over channel n's current
 *     (already compensated) weights of the group.
 *   - static_groups != 0: groups are the original columns [gG, (g+1)G) and s[n][g] is
 *     taken from W as given before the sweep.
 * Reconstruction: W_hat[n][k] = scales_out[n][g_idx[k]] * (codes[n][k] - z).
 *
 *   U          device fp32 [K][K] from gptq_prepare on the Hessian in processing
 *              order (gptq_permute_hessian with perm), or on H itself when perm is
 *              NULL.
 *   groupsize  32, 64 or 128, dividing blocksize (blocksize 32, 64 or 128); or 0 for
 *              one per-channel scale (gptq_quantize_layer's) with the order of perm.
 *   perm       device int32 [K] processing order (gptq_act_order), or NULL (natural).
 *   P1         device fp32 [K][K] from gptaq_residual in processing order, or NULL.
 *   cae        as gptq_quantize_layer; w^(0) is taken in processing order.
 *   dead       device uint8 [K] in processing order (gptq_prepare's dead_out), or NULL.
 *   scales_out device fp32 [N][ceil(K / groupsize)] ([N] when groupsize == 0), or NULL.
 *   g_idx_out  device int32 [K] group of each original coordinate (0 when
 *              groupsize == 0), or NULL.
 *   codes      device uint8 [N][K] in the original coordinate order (required).
 *   W, bits, loss, write_back, status: as gptq_quantize_layer (write-back in the
 *              original order).
 *   ws         gptq_workspace_size(GPTQ_OP_QUANTIZE_GROUPED | (cae ? GPTQ_WS_CAE : 0), K,
 *              N, 1, blocksize) bytes.
 */
GPTQ_API gptq_status gptq_quantize_layer_grouped(void *W, int wdtype, int N, int K, const float *U,
                                                 int bits, int blocksize, int groupsize,
                                                 int static_groups, const int32_t *perm,
                                                 const float *P1, int cae, const uint8_t *dead,
                                                 float *scales_out, int32_t *g_idx_out,
                                                 uint8_t *codes, float *loss, int write_back,
                                                 void *ws, size_t ws_bytes, int32_t *status,
                                                 void *stream);

/*
 * gptq_pack_codes -- codes [N][K] (uint8, < 2^bits) as low-bit words.
 *
 * [GPTQ blog] "落在格点上与真正存成低位权重是两步": codes on the grid are storage only
 * once packed into wider integer containers, kept with scale, zero point and layout.
 * Layout (the pages fix none): per output channel n, code k occupies bits
 * [bits k, bits k + bits) of a little-endian bit stream whose bit t is bit t mod 32
 * of words[n][t / 32]; 32 / bits whole codes per word for bits 2, 4, 8, and 32 codes
 * per 3 words for bits 3 (some codes straddle two words). The row's last word has
 * its unused high bits zero; words past ceil(K bits / 32) are not touched. The
 * reconstruction is s (c - z) with z = 2^(bits-1) and the scales (and g_idx) of the
 * quantisation call, in the original coordinate order.
 *
 *   codes     device uint8, row n at codes + n ld_codes (ld_codes >= K). Only the
 *             low `bits` bits of each code are read.
 *   words     device uint32, row n at words + n ld_words
 *             (ld_words >= ceil(K bits / 32)).
 *   N >= 0 (0: nothing to do), 1 <= K; bits 2, 3, 4 or 8.
 *   Errors: GPTQ_ERR_ARG for sizes, strides or bits out of range, NULL pointers.
 */
GPTQ_API gptq_status gptq_pack_codes(const uint8_t *codes, int N, int K, int64_t ld_codes,
                                     int bits, uint32_t *words, int64_t ld_words, void *stream);

/* gptq_unpack_codes -- the inverse of gptq_pack_codes (same layout and arguments). */
GPTQ_API gptq_status gptq_unpack_codes(const uint32_t *words, int N, int K, int64_t ld_words,
                                       int bits, uint8_t *codes, int64_t ld_codes, void *stream);

/*
 * gptq_first_order_shift -- the first-order (gradient) term as a shifted start:
 * W <- W - beta G H^-1 per output channel, with H^-1 = U^T U.
 *
 * [G2PTQ] summary: the compensation keeps GPTQ's second-order update and adds the
 * first-order term of an exact gradient G of the block objective, scaled by a
 * trust-region factor beta in [0, 1]. The pages print no formula. Reading: the
 * objective per channel is the quadratic model beta g^T d + 1/2 d^T H d around the
 * given weights; sequential OBQ on it is GPTQ started from the model's minimiser
 * w - beta H^-1 g. So: shift an fp32 copy of W with this call, then quantise that
 * copy with gptq_quantize_layer (its scales come from the shifted weights, as GPTQ
 * takes them from the weights it is given).
 *
 *   W      device fp32 [N][K], shifted in place.
 *   U      device fp32 [K][K] from gptq_prepare (g = 1).
 *   G      device [N][K] gradient, dtype gdtype (GPTQ_BF16 or GPTQ_F32).
 *   beta   in [0, 1] (gptq_trust_region_beta).
 *   gamma  device double, or NULL: sum_n g_n H^-1 g_n^T; the model's loss change
 *          along the step is -(beta - beta^2 / 2) gamma.
 *   ws     gptq_workspace_size(GPTQ_OP_FIRST_ORDER, K, N, 1, 0) bytes.
 *   Errors: GPTQ_ERR_ARG for sizes, dtype, beta outside [0, 1] or NULL pointers.
 */
GPTQ_API gptq_status gptq_first_order_shift(float *W, int N, int K, const float *U, const void *G,
                                            int gdtype, float beta, double *gamma, void *ws,
                                            size_t ws_bytes, int32_t *status, void *stream);

/*
 * gptq_trust_region_beta -- host: the largest beta in [0, 1] whose first-order loss
 * change stays within alpha times the GPTQ term's: (beta - beta^2/2) gamma <=
 * alpha loss_gptq ([G2PTQ] summary: beta bounds the first-order step by alpha times
 * the GPTQ term's loss change; alpha is searched per block on [0, 3]). loss_gptq is
 * the sweep's loss (sum of gptq_quantize_layer's loss output); gamma as above.
 * gamma <= 0 gives 1; a negative or NaN ratio gives 0.
 */
GPTQ_API float gptq_trust_region_beta(float alpha, double loss_gptq, double gamma);

/*
 * gptq_selftest_timeout -- a diagnostic of the failure path every bounded device wait
 * of the library shares: one kernel waits on a barrier that nothing arrives on; when
 * the wait budget (about a second) runs out it sets GPTQ_ERR_TIMEOUT in *status and
 * returns. Nothing faults or traps: the context stays usable afterwards.
 *
 *   status  device int32 (required).
 */
GPTQ_API gptq_status gptq_selftest_timeout(int32_t *status, void *stream);

/*
 * Kernel timing by class -- a benchmark diagnostic (the pages have no counterpart).
 *
 * gptq_profile_enable(1) starts a window: from then on the library records a pair of
 * CUDA events around every launch of the classes below, on the stream that launch
 * uses (nothing is recorded while a stream is being captured into a CUDA graph);
 * gptq_profile_enable(0) stops recording. gptq_profile_read synchronises the
 * window's events of one class and returns their summed elapsed time (ms) and the
 * number of launches. The events add a little host work per launch; leave profiling
 * off outside measurements.
 */
typedef enum {
    GPTQ_PROF_SWEEP = 0,     /* in-block sweep kernels of gptq_quantize_layer(_grouped) */
    GPTQ_PROF_UPDATE = 1,    /* tensor-core lazy (near / far) updates */
    GPTQ_PROF_DIAG = 2,      /* diagonal-block factor of gptq_prepare */
    GPTQ_PROF_TC32 = 3,      /* tf32 x3 tensor-core products (factor, inverse, residual, shift) */
    GPTQ_PROF_SPLIT = 4,     /* splits of fp32 operands into tf32 / bf16 pairs */
    GPTQ_PROF_KINDS = 5
} gptq_prof_kind;

GPTQ_API gptq_status gptq_profile_enable(int on);
GPTQ_API gptq_status gptq_profile_read(int kind, double *ms, int *launches);

/*
 * gptq_profile_timeline -- the window's records in launch order: for record i,
 * kind[i] (a gptq_prof_kind), lane[i] (the stream it ran on, numbered 0, 1, ... in
 * order of first appearance in the window) and its begin and end times in ms from
 * the first record's begin event. At most `max` records are written (all arrays
 * host, `max` entries); *count receives the number of records in the window, which
 * may exceed `max`. Synchronises the window's events. GPTQ_ERR_ARG on a NULL pointer
 * or max < 0.
 */
GPTQ_API gptq_status gptq_profile_timeline(int max, int *kind, int *lane, double *begin_ms,
                                           double *end_ms, int *count);

/*
 * gptq_bounds_report -- records of the index-check build (a debugging aid standing in
 * for a memory checker; the pages have no counterpart).
 *
 * The library built with GPTQ_DEBUG_BOUNDS (libgptq_dbg.so; python -m
 * post_weight_quantization_solve_b200.build --debug-bounds) checks, in its kernels,
 * tile origins against the product or block they belong to, TMA box coordinates
 * against their tensor and the 16-byte rule on the innermost coordinate, and computed
 * output offsets against the output's extent. A failed check skips the access (never
 * a trap), counts the failure and stores GPTQ_ERR_BOUNDS in the call's status word.
 *
 *   enabled  host int: 1 in the checking build, 0 otherwise (then the rest is zero).
 *   count    host int: failed checks since the last reset.
 *   site     host int: the first failure's site: 1 self-test, 2 tf32x3 GEMM tile,
 *            3 tf32x3 GEMM TMA coordinate, 4 tf32x3 GEMM output element, 5 tf32x3
 *            GEMM pair element, 6 Gram load box, 7 Gram reduction box, 8 sweep load
 *            box, 9 sweep output offset, 10 lazy-update load box, 11 lazy-update
 *            output element, 12 diagonal block; 0 when count is 0.
 *   index    host int64: the first failure's offset or coordinate.
 *   reset    non-zero: clear the records after reading them.
 * Synchronises the device (reads device records). GPTQ_ERR_ARG on a NULL pointer,
 * GPTQ_ERR_CUDA when a record cannot be read.
 */
GPTQ_API gptq_status gptq_bounds_report(int *enabled, int *count, int *site, int64_t *index,
                                        int reset);

/*
 * gptq_bounds_selftest -- checking build only: one thread runs one check that always
 * fails (site 1; no memory is accessed), so that a test sees the record and the
 * status word change. Other builds return GPTQ_ERR_ARG and enqueue nothing.
 *
 *   status  device int32 (required): receives GPTQ_ERR_BOUNDS.
 */
GPTQ_API gptq_status gptq_bounds_selftest(int32_t *status, void *stream);

/*
 * gptq_chain_latency -- one thread runs `steps` steps (a multiple of 8, >= 8) of the
 * sweep's dependent chain for one coordinate: the previous error applied to the
 * coordinate (FMA), the scale, round-half-even and clamp to the grid, and the
 * normalised error (FMA, multiply), each step depending on the last. Writes, to the
 * device buffer `out` (3 floats): SM clock cycles per step, nanoseconds per step, and
 * a value that keeps the chain live. K steps of this chain bound a sweep over K
 * coordinates from below, however many channels run in parallel. A diagnostic (the
 * pages have no counterpart).
 */
GPTQ_API gptq_status gptq_chain_latency(float *out, int steps, void *stream);

/* Workspace bytes for an operation (gptq_op); 0 when none is needed. */
GPTQ_API size_t gptq_workspace_size(int op, int K, int N, int g, int blocksize);

/* Number of kernels this process has enqueued through the library so far
 * (a host-side counter; for launch accounting in benchmarks). */
GPTQ_API unsigned long long gptq_kernel_launches(void);

/* Static, NUL-terminated description of a status code. */
GPTQ_API const char *gptq_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_H */
