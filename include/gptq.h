/*
 * gptq.h -- C ABI of libgptq.so, a B200 (sm_100a) implementation of GPTQ
 * single-layer post-training weight quantization.
 *
 * The method (itwiki "GPTQ" article, sections "문제 설정", "OBQ에서 GPTQ로",
 * "알고리즘" and "실무 변형"; blog "GPTQ를 밑바닥부터 구현하며 배운 것들",
 * section 3): given a linear layer's weights W [d_out, d_in] and its
 * calibration inputs X [n, d_in], find W^ on a low-bit grid that keeps
 * ||W X^T - W^ X^T||^2 small.  Four stream-ordered stages:
 *
 *   gptq_hessian_accumulate   H += 2 X^T X            (per calibration batch)
 *   gptq_prepare_hinv         U = upper Cholesky factor of (H + lambda I)^-1
 *   gptq_quantize_layer       blocked column sweep + lazy trailing updates
 *                             + packing of the codes
 *   gptq_rtn_layer            round-to-nearest on the same grid (baseline)
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer named *_dev / W / X / H / U / codes / scales / zeros / Q / ws
 *    is DEVICE memory owned by the caller.  The library never allocates or
 *    frees device memory.  Host-side validation happens before any CUDA call:
 *    an invalid argument returns an error code and launches nothing.
 *  - Matrices are dense, row-major, with no padding (row stride = columns).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls only enqueue work; they return before it runs.
 *  - Errors found on the device (a non-positive pivot, non-finite values, a
 *    wait that ran out of time) are recorded in a per-device status word;
 *    gptq_get_status() synchronizes the stream, returns it and clears it.
 *    No kernel traps, asserts or waits without a bound.
 *  - Sizes: d_in must be a multiple of 128 and at most 32768; d_out >= 1;
 *    pointers to float / uint32 data must be 16-byte aligned.
 *  - Calls on different streams may run concurrently if they touch
 *    different buffers and workspaces; the status word is shared.
 */
#ifndef GPTQ_H
#define GPTQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GPTQ_OK = 0,
    GPTQ_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or workspace  */
    GPTQ_ERR_UNSUPPORTED = 2,   /* valid for the method, not for this build   */
    GPTQ_ERR_NOT_PD = 3,        /* damped H not positive definite             */
    GPTQ_ERR_NONFINITE = 4,     /* NaN/Inf met in H, U, W or the grid         */
    GPTQ_ERR_GRID = 5,          /* grid not representable in fp16             */
    GPTQ_ERR_TIMEOUT = 6,       /* a bounded device-side wait gave up         */
    GPTQ_ERR_CUDA = 7           /* a CUDA runtime call failed                 */
} gptq_status;

typedef enum { GPTQ_F32 = 0, GPTQ_BF16 = 1 } gptq_dtype;

/* Version of this ABI (bumped on any incompatible change). */
int gptq_abi_version(void);

/* Number of kernels this library has enqueued in this process so far (all
 * devices and streams).  A diagnostic: the difference across a region of
 * code is how many of this library's kernels that region launched. */
uint64_t gptq_launch_count(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* gptq_status_string(int status);

/* ------------------------------------------------------------------------
 * Stage 1 -- Hessian accumulation.
 * Source: blog "GPTQ를 밑바닥부터 구현하며 배운 것들", section 3 (H = 2 X^T X
 * from the inputs captured at each linear layer); itwiki "GPTQ",
 * "최소 구현" (H = 2 X^T X, X laid out [n, d_in]) and its closing paragraph
 * (H accumulated per layer over the calibration data).
 *
 * H[a][b] += 2 * sum_r X[r][a] * X[r][b]   for all 0 <= a <= b < d_in.
 *
 *   X      device, [n, d_in] row-major, bf16 (xdt = GPTQ_BF16) or fp32
 *          (xdt = GPTQ_F32), 16-byte aligned.  n may be 0 (no-op).
 *   H      device, [d_in, d_in] fp32, 16-byte aligned.  Caller zeroes it
 *          before the first batch (gptq_fill_f32) and calls this once per
 *          batch.  The upper triangle (b >= a) is the result; entries below
 *          the diagonal may be written with their (symmetric) values inside
 *          tiles that straddle the diagonal and are otherwise left untouched.
 *   ws     device workspace of at least gptq_hessian_workspace_size(xdt, n,
 *          d_in) bytes (0 for bf16: ws may be NULL).  fp32 inputs are split
 *          into three bf16 terms there.
 * Products run on the tensor cores: bf16 x bf16 with fp32 accumulation
 * (exact products); fp32 X is split x = h + m + l into bf16 terms and the six
 * leading cross products are accumulated (about fp32 accuracy).
 * ---------------------------------------------------------------------- */
size_t gptq_hessian_workspace_size(int dtype, int64_t n, int64_t d_in);
int gptq_hessian_accumulate(const void* X, int dtype, int64_t n, int64_t d_in,
                            float* H, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Stage 1 over several calibration batches in one call: the same result as
 * calling gptq_hessian_accumulate on X[0], X[1], ... in order, with the same
 * H, dtype, d_in, workspace and stream (source as above: H accumulated over
 * the calibration data).
 *
 *   X      HOST array of `count` device pointers; X[i] is [n[i], d_in]
 *          row-major, 16-byte aligned (may be NULL where n[i] = 0).
 *   n      HOST array of `count` row counts, each 0 <= n[i] < 2^31.
 *   ws     as above, sized for the largest batch (fp32 only).
 * Returns GPTQ_ERR_INVALID_ARG (launching nothing) if any argument is
 * invalid.  Faster than separate calls for bf16 X: each batch's kernel
 * waits for the previous batch's only before it updates H, so their
 * contractions overlap on the GPU.  The batches must not be written by the
 * GPU while the call's kernels run (they are read as the stream reaches
 * them).
 * ---------------------------------------------------------------------- */
int gptq_hessian_accumulate_batches(const void* const* X, const int64_t* n, int count, int dtype,
                                    int64_t d_in, float* H, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Stage 2 -- dampening and the upper Cholesky factor of the inverse.
 * Source: itwiki "GPTQ", "GPTQ의 세 가지 변경" row 3 (add 1% of the mean
 * diagonal; only the Cholesky form of H^-1 is needed, computed once up
 * front); "알고리즘" (H^-1 <- Cholesky(H^-1)^T); "최소 구현" (chol ->
 * cholesky_inverse -> chol(upper)).
 *
 * lambda = percdamp * mean(diag H);  U upper triangular with
 * U^T U = (H + lambda I)^-1.  Computed as U = P L'^-1 P with P the index
 * reversal and L' = chol(P (H + lambda I) P) -- the same U as the pages'
 * chain by uniqueness of the Cholesky factor -- in fp32.
 *
 *   H        device [d_in, d_in] fp32; only the upper triangle is read; not
 *            modified.
 *   U        device [d_in, d_in] fp32 output; the strict lower triangle is
 *            set to 0.  On failure U is filled with NaN.
 *   info_dev device int32 (may be NULL): 0 on success, else k+1 where k is
 *            the step (0-based, in the order the factorization visits the
 *            columns of H: last column first) whose pivot was not positive
 *            and finite.  The status word gets GPTQ_ERR_NOT_PD (or
 *            GPTQ_ERR_NONFINITE for a NaN/Inf pivot).
 *   ws       >= gptq_prepare_hinv_workspace_size(d_in) bytes.
 * The work forks from `stream` onto three library-owned streams (the
 * factorization's chain, its look-ahead updates, the inverse) and joins back
 * before the call's last kernel; later work on `stream` sees U complete.
 * Deterministic: every element receives its updates in a fixed order, so the
 * same H gives the same U bit for bit on every call.  A
 * device has four such sets.  A caller stream keeps the set it got first, so
 * calls on up to four different streams run concurrently (independent
 * layers); further streams share the sets, and calls sharing a set run one
 * after the other.  A set's streams and events are created by the first call
 * that gets it; a caller that records these calls into a stream capture
 * makes one call on that stream before the capture begins.
 * ---------------------------------------------------------------------- */
size_t gptq_prepare_hinv_workspace_size(int64_t d_in);
int gptq_prepare_hinv(const float* H, int64_t d_in, float percdamp, float* U,
                      int* info_dev, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Stages 3-5 -- the blocked column sweep with lazy trailing updates and the
 * packed output.
 * Source: itwiki "GPTQ", "알고리즘" (Algorithm 1), "GPTQ의 세 가지 변경" rows
 * 1-2 (one column order for all rows; updates inside a block of B columns,
 * then one matrix product for the rest), "최소 구현" (per-row asymmetric
 * min/max grid), "실무 변형" (group quantization, grid from the latest
 * updated weights); blog, section 5 (store integer codes, not fp32).
 *
 * For each block i = 0, B, 2B, ... and each column j of the block:
 *   c = clamp(rint(w_j / s) + z, 0, maxq);  q = s (c - z);
 *   E[:, j-i] = (w_j - q) / U[j][j];  W[:, j:i+B] -= E[:, j-i] U[j, j:i+B];
 * then W[:, i+B:] -= E U[i:i+B, i+B:].  That trailing update is applied in
 * the deferred super-block form, exact in real arithmetic: blocks are taken
 * in super-blocks of S columns (S = d_in if d_in <= 1024; else 1024, or the
 * largest multiple of groupsize up to 1024, or B for groups wider than
 * 1024); after each block its E updates only the rest of its super-block,
 * and after a super-block's last block the columns beyond it get one product
 * with the whole super-block's E (S deep).  The order is fixed: the same
 * inputs give the same bits on every call.
 * Grid: s32 = max(wmax - wmin, 1e-8) / maxq (fp32), s = fp16(s32) (2^-14 if
 * that rounds to 0), z = fp16(rint(-wmin / s)); per row from the original W
 * (groupsize = -1), or per group of `groupsize` columns from the current W
 * when the sweep reaches the group's first column.
 *
 *   W        device [d_out, d_in] fp32 working copy, OVERWRITTEN (holds the
 *            partially updated weights afterwards; not a result).
 *   U        device [d_in, d_in] fp32 from gptq_prepare_hinv (upper read).
 *   bits     2, 3, 4 or 8 (maxq = 2^bits - 1).
 *   blocksize must be 128.
 *   groupsize -1 (one grid per row) or a multiple of 128 dividing d_in.
 *   codes    device uint32 [d_out, d_in * bits / 32]: per row a little-endian
 *            bit stream, code k in stream bits [k*bits, (k+1)*bits).
 *   scales, zeros  device fp16 bit patterns (uint16) [d_out, n_groups],
 *            n_groups = 1 or d_in / groupsize.
 *   Q        device [d_out, d_in] fp32 dequantized weights, or NULL.
 *   ws       >= gptq_quantize_workspace_size(d_out, d_in, blocksize) bytes.
 * ---------------------------------------------------------------------- */
size_t gptq_quantize_workspace_size(int64_t d_out, int64_t d_in, int blocksize);
int gptq_quantize_layer(float* W, int64_t d_out, int64_t d_in, const float* U,
                        int bits, int blocksize, int groupsize,
                        uint32_t* codes, uint16_t* scales, uint16_t* zeros,
                        float* Q, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Stages 3-5 without a caller workspace.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory where
 * they quantize -- a host framework whose memory pool owns every device
 * buffer and hands out only inputs and outputs, or a serving process that
 * reserves its memory budget at start-up and may not call cudaMalloc later
 * (the call can fail once the budget is taken, and it synchronizes the
 * device).
 *
 * Same arguments, results and errors as gptq_quantize_layer, minus ws and
 * ws_bytes.  The scratch it needs (E [d_out, min(d_in, 1024)] and U^T
 * [d_in, d_in], each kept as two fp32 arrays -- the tf32-rounded part and the
 * remainder -- for the tensor-core trailing products, each array rounded up to
 * 256 bytes) lives in one 40 MiB device array inside the library, which every
 * GPU that loads the library holds until the process exits.  Sizes that need
 * more than 40 MiB (about d_out * min(d_in, 1024) * 8 + d_in * d_in * 8
 * bytes) return GPTQ_ERR_UNSUPPORTED and launch nothing: e.g. d_in = 1024
 * works for d_out up to 4096, d_in = 2048 for d_out up to 1024, d_in = 512 for
 * d_out up to 9728; d_in = 2304 does not fit at all.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress with that device current); make that first call
 *    before any stream capture begins.
 *  - It calls no cudaMalloc, cudaFree or other allocating routine.
 *  - All calls on a device share the one array, which keeps the last call's
 *    contents (nothing in it needs to start at zero).  Calls whose work
 *    overlaps on the GPU (different streams, not ordered) race on it: order
 *    them on one stream or with events.
 * ---------------------------------------------------------------------- */
int gptq_quantize_layer_noalloc(float* W, int64_t d_out, int64_t d_in, const float* U,
                                int bits, int blocksize, int groupsize,
                                uint32_t* codes, uint16_t* scales, uint16_t* zeros,
                                float* Q, void* stream);

/* ------------------------------------------------------------------------
 * Baseline -- round to nearest on the same grid, no compensation.
 * Source: itwiki "GPTQ", "문제 설정" (RTN moves each weight to its nearest
 * grid point without looking at the inputs).  Group grids come from the
 * original W.  Arguments as for gptq_quantize_layer; W is not modified.
 * ---------------------------------------------------------------------- */
int gptq_rtn_layer(const float* W, int64_t d_out, int64_t d_in, int bits, int groupsize,
                   uint32_t* codes, uint16_t* scales, uint16_t* zeros, float* Q,
                   void* stream);

/* ------------------------------------------------------------------------
 * Act-order -- the columns in order of decreasing Hessian diagonal.
 * Source: itwiki "GPTQ", "실무 변형" (act-order: the columns whose inputs
 * carry the largest diag(H) are quantized first; it helps models with
 * outlier channels).  The sweep itself is unchanged: it runs on the permuted
 * problem.  A layer quantized with act-order is
 *
 *   gptq_act_order_perm(H, d_in, perm)                     processing order
 *   gptq_permute_hessian(H, d_in, perm, Hp)                Hp = H[perm][:, perm]
 *   gptq_prepare_hinv(Hp, ...)                             U of the permuted H
 *   gptq_permute_columns(W, d_out, d_in, perm, 0, W)       W = W[:, perm]
 *   gptq_quantize_layer(W, ..., U, ..., Q)                 codes in processing order
 *   gptq_permute_columns(Q, d_out, d_in, perm, 1, Q)       Q back to W's order
 *
 * codes, scales and zeros stay in processing order (a group is `groupsize`
 * consecutive columns of that order); column k of the codes belongs to
 * column perm[k] of W.  Dampening does not depend on the order.
 *
 * gptq_act_order_perm: perm[k] = index of the column processed k-th: the
 * indices sorted by diag(H) descending, equal values (-0 equal to +0) in
 * increasing index order, NaN after every number.  Always a permutation.
 *   H     device [d_in, d_in] fp32 (only the diagonal is read), 16-byte aligned.
 *   perm  device int32 [d_in] output, 4-byte aligned, not inside H.
 *
 * gptq_permute_hessian: Hp[a][b] = Hs[perm[a]][perm[b]] for all a, b, where Hs
 * is the symmetric matrix whose upper triangle is H's (the lower triangle of
 * H is not read).  Hp is written whole (both triangles).
 *   H, Hp device [d_in, d_in] fp32, 16-byte aligned, not overlapping.
 *   perm  device int32 [d_in], a permutation of 0 .. d_in-1.  An entry
 *         outside that range is recorded as GPTQ_ERR_INVALID_ARG in the status
 *         word and the outputs it selects are NaN (nothing is read out of
 *         bounds).
 *
 * gptq_permute_columns: for every row r of a [rows, cols] fp32 matrix,
 *   inverse = 0:  dst[r][k] = src[r][perm[k]]     (into processing order)
 *   inverse = 1:  dst[r][perm[k]] = src[r][k]     (back to the original order)
 *   src, dst device, 16-byte aligned; either the same array (in place) or
 *         not overlapping.  rows in [0, 2^24]; cols like d_in (a multiple of
 *         128, at most 32768).
 *   perm  device int32 [cols] as above; entries outside [0, cols) are
 *         recorded as GPTQ_ERR_INVALID_ARG and select NaN; with inverse = 1,
 *         slots of dst that no entry reaches are NaN.
 * All three return GPTQ_ERR_INVALID_ARG (launching nothing) for a bad size,
 * pointer, alignment or overlap.
 * ---------------------------------------------------------------------- */
int gptq_act_order_perm(const float* H, int64_t d_in, int32_t* perm, void* stream);
int gptq_permute_hessian(const float* H, int64_t d_in, const int32_t* perm, float* Hp, void* stream);
int gptq_permute_columns(const float* src, int64_t rows, int64_t cols, const int32_t* perm, int inverse,
                         float* dst, void* stream);

/* ------------------------------------------------------------------------
 * Inference -- the layer output computed from the stored form (W4A16).
 * Source: itwiki "GPTQ", "결과" (a dedicated kernel unpacks the weights as
 * it needs them at inference and cuts the per-token latency against FP16);
 * blog "GPTQ를 밑바닥부터 구현하며 배운 것들", section 5 (production
 * implementations store INT4 codes and dequantize them during inference).
 *
 *   y[t][r] = sum_k s[r][g(k)] * (c[r][k] - z[r][g(k)]) * x[t][perm[k]]
 *
 * for tokens t < m and rows r < d_out; g(k) = k / groupsize (0 for a per-row
 * grid); c, s, z as gptq_quantize_layer writes them (processing order).
 *   codes   device uint32 [d_out, d_in * bits / 32], 16-byte aligned.
 *   scales, zeros  device fp16 bit patterns [d_out, n_groups].
 *   bits    4 (2, 3 and 8 return GPTQ_ERR_UNSUPPORTED in this build).
 *   groupsize  -1 or a multiple of 128 dividing d_in.
 *   perm    device int32 [d_in] (act-order: code column k multiplies input
 *           column perm[k]) or NULL (natural order).  An entry outside
 *           [0, d_in) is recorded as GPTQ_ERR_INVALID_ARG in the status word
 *           and its input is taken as NaN.
 *   x       device bf16 bit patterns [m, d_in] row-major, 16-byte aligned;
 *           0 <= m <= 8 (m = 0: nothing to do).
 *   y       device fp32 [m, d_out] row-major output.
 *   ws      device workspace of gptq_dequant_gemv_workspace_size(m, d_in,
 *           perm != NULL) bytes, 16-byte aligned: x in processing order as
 *           fp16, scaled by a power of two per 128-column block, with each
 *           block's sum and scale.
 * Every product c * x is exact: each 128-column block of x is scaled by 2^-e
 * so that its largest magnitude lies in [2^14, 2^15), which keeps every bf16
 * value down to 2^-28 of that maximum exact in fp16 (smaller ones round to
 * fp16's subnormals); codes and scaled x meet on the tensor cores with fp32
 * accumulation; each block is scaled and offset in fp32,
 * 2^e s (sum c x - z sum x).
 * ---------------------------------------------------------------------- */
size_t gptq_dequant_gemv_workspace_size(int64_t m, int64_t d_in, int with_perm);
int gptq_dequant_gemv(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                      int64_t d_in, int bits, int groupsize, const int32_t* perm, const uint16_t* x, int64_t m,
                      float* y, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Inference -- the weights rebuilt from the stored form.
 * Source: note "Model Quantization", section "주요 양자화 기법", the GPTQ
 * entry (at inference the INT4 weights are restored to FP16 for the
 * computation); blog "GPTQ를 밑바닥부터 구현하며 배운 것들", section 5 (codes
 * stored, dequantized for use).  A product with more tokens than
 * gptq_dequant_gemv takes (prefill) is this call plus a plain library GEMM.
 *
 *   out[r][perm[k]] = s[r][g(k)] * (c[r][k] - z[r][g(k)])
 *
 * for every row r < d_out and code column k < d_in (processing order);
 * perm = NULL: out[r][k].  g(k) = k / groupsize (0 for a per-row grid).
 *   codes   device uint32 [d_out, d_in * bits / 32], 4-byte aligned;
 *           bits 2, 3, 4 or 8.
 *   scales, zeros  device fp16 bit patterns [d_out, n_groups].
 *   perm    device int32 [d_in], 16-byte aligned, or NULL.  An entry outside
 *           [0, d_in) is recorded as GPTQ_ERR_INVALID_ARG and skipped; a
 *           column that no entry reaches is NaN.
 *   out_dtype  0 fp32: s (c - z) rounded once (exact whenever it fits 24
 *              bits, as it always does for the integer zero points the
 *              quantizer writes); 1 bf16, 2 fp16: that fp32 value rounded to
 *              nearest even.
 *   out     device [d_out, d_in] of that type, row-major, 16-byte aligned.
 * ---------------------------------------------------------------------- */
int gptq_dequantize(const uint32_t* codes, const uint16_t* scales, const uint16_t* zeros, int64_t d_out,
                    int64_t d_in, int bits, int groupsize, const int32_t* perm, int out_dtype, void* out,
                    void* stream);

/* ------------------------------------------------------------------------
 * Helpers on the same stream (not steps of the method).
 * ---------------------------------------------------------------------- */
/* dst[i] = (float) src[i] for bf16 bit patterns src (a bf16 layer's fp32
 * working copy). src 16-byte aligned is not required; dst is. */
int gptq_widen_bf16(const uint16_t* src, float* dst, int64_t count, void* stream);
/* p[i] = value for i < count (zeroing H before the first batch). */
int gptq_fill_f32(float* p, int64_t count, float value, void* stream);

/* Synchronizes `stream`, returns the first device-side error recorded since
 * the last call (GPTQ_OK if none) and clears it.  *detail_out (may be NULL)
 * receives a code-specific detail (a row or pivot index).  Returns
 * GPTQ_ERR_CUDA if the synchronization itself failed. */
int gptq_get_status(void* stream, int* detail_out);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_H */
