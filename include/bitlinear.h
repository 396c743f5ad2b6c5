/*
 * bitlinear.h -- C ABI of libbitlinear.so, the B200 (sm_100a) BitNet b1.58 BitLinear
 * forward pass.
 *
 * Conventions shared by every entry point
 *   - Data pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates, frees or copies on these calls and never synchronises; each call only
 *     enqueues kernels on `stream` (a cudaStream_t passed as void*; NULL = legacy
 *     default stream) and returns.
 *   - Dimensions are int64_t.  Matrices are dense row-major: W is [N, K] (nn.Linear
 *     convention, N = out features, K = in features), X / x_q are [M, K], y is [M, N].
 *   - Base pointers must be 16-byte aligned (cudaMalloc and PyTorch allocations are).
 *   - Argument errors are detected on the host before any launch and leave every
 *     output untouched.  A launch error returns BL_ERR_CUDA (the CUDA error code is
 *     kept for bitlinear_last_cuda_error()).  Faults inside a kernel surface at the
 *     caller's next synchronisation of `stream`, as for any CUDA kernel.
 *   - Optional `err_word` (device int32, may be NULL): kernels OR status bits into it
 *     (BL_ERRBIT_*) for conditions only the device can see.  The caller zeroes it.
 *   - Calls are reentrant: there is no hidden state besides the last CUDA error code.
 *
 * Packed ternary weight format (the only weight format the forward reads)
 *   uint8 [N, K/4], row-major, K % 4 == 0.  Byte j of row n holds the codes of
 *   elements k = 4j + i (i = 0..3) in bits 2i..2i+1, least significant first:
 *   00 -> 0, 01 -> +1, 10 -> -1.  11 is never written by this library; the forward
 *   reads it as 0.
 *
 * Sources (page title -- section):
 *   [B158] "1-bit & Ternary LLMs (BitNet b1.58)" -- "How it works (real mechanics)",
 *          block "BitNet b1.58 (Feb 2024)": gamma = (1/nm) sum |W_ij|,
 *          W~ = RoundClip(W / (gamma + eps), -1, 1).
 *   [BIN]  same page, block "BitNet (Oct 2023)": absmax per-token activation
 *          quantisation and y = W~ . Quant(LN(x)) . (beta gamma / Q_b).
 *   [STE]  same page, "Training: shadow weights + the straight-through estimator":
 *          y = (W_eff @ x_q) * scale, an integer matmul plus one float rescale.
 *   [CH2]  "What 1.58 Bits Actually Changes" -- "How the low-bit linear path works":
 *          per-token signed 8-bit activations without a zero point; +1 adds, -1
 *          subtracts, 0 skips; packed ternary values are loaded and unpacked.
 *
 * Readings where the pages are silent: round = half to even; gamma includes eps
 * everywhere (division and output scale); Q_b = 127 with clip [-128, 127]; true IEEE
 * division for W / gamma and 127 / absmax; y = acc * gamma / s_m.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BL_API __attribute__((visibility("default")))
#else
#define BL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BL_OK = 0,
    BL_ERR_INVALID_ARG = 1,       /* NULL pointer, non-positive size, eps <= 0 or not finite */
    BL_ERR_UNSUPPORTED_SHAPE = 2, /* K % 4 != 0, or a size whose int32 sums could overflow */
    BL_ERR_MISALIGNED = 3,        /* a base pointer is not 16-byte aligned */
    BL_ERR_WORKSPACE = 4,         /* workspace NULL or smaller than bitlinear_workspace_size */
    BL_ERR_CUDA = 5,              /* a launch or attribute call failed */
    BL_ERR_TIMEOUT = 6,           /* (err_word bit) a bounded device wait gave up */
    BL_ERR_BAD_CODE = 7           /* (err_word bit) an input code outside {-1, 0, +1} */
} bl_status;

/* Bits OR-ed into the optional device err_word.  BL_ERRBIT_INDEX is set only by a library
 * built with device index checks (BL_DEBUG_CHECKS=1, a debugging build): a kernel found an
 * index outside its buffer, recorded it here and skipped that access. */
#define BL_ERRBIT_BAD_CODE 0x1
#define BL_ERRBIT_TIMEOUT 0x2
#define BL_ERRBIT_INDEX 0x4

typedef enum {
    BL_OUT_F32 = 0,  /* y as fp32 */
    BL_OUT_BF16 = 1, /* y as bf16 (round to nearest even of the fp32 value) */
    BL_OUT_I32 = 2   /* the raw int32 accumulators acc = x_q . c^T, no rescale */
} bl_dtype;

typedef enum {
    BL_PATH_AUTO = 0,   /* GEMV for M <= 16 (or shapes the tensor-core paths cannot tile); for
                           16 < M <= 64 the GEMV fed by asynchronous copies up to 32 tokens
                           (stride-4 x_q), else the small-batch tcgen05 kernel; tiled tcgen05
                           above 64 tokens */
    BL_PATH_GEMV = 1,   /* register-unpack GEMV, any M (token tiles of 16) */
    BL_PATH_TC = 2,     /* tcgen05 kind::i8 tiled path (single SM or SM pair, by shape); K % 64 == 0 */
    BL_PATH_TC_1SM = 3, /* the tcgen05 path forced to single-SM tiles (testing) */
    BL_PATH_TC_2SM = 4, /* the tcgen05 path forced to SM-pair (cta_group::2) tiles (testing) */
    BL_PATH_SKINNY = 5, /* the tcgen05 small-batch kernel (K split over a cluster when rows
                           are few); K % 64 == 0 */
    BL_PATH_GEMV_STREAM = 6, /* the GEMV kernel fed by per-thread asynchronous copies (testing):
                                M <= 64, x_q in BL_XQ_K16_STRIDE4, K % 64 == 0, K <= 2^17, and
                                at most 64 (48 for M > 16) sixteen-row tiles of N per SM; other
                                shapes return BL_ERR_UNSUPPORTED_SHAPE */
    BL_PATH_GEMV_TMA = 7     /* the persistent TMA-fed GEMV kernel (testing): M <= 16, x_q in
                                BL_XQ_K16_STRIDE4, K % 128 == 0, K <= 2^17, and between 1 and
                                32 sixteen-row tiles of N per SM; other shapes return
                                BL_ERR_UNSUPPORTED_SHAPE */
} bl_path;

/* Storage order of x_q within each row.
 *   BL_XQ_ROWMAJOR     element k at byte k (the plain [M, K] int8 matrix).
 *   BL_XQ_K16_EVENODD  K % 16 == 0; inside every group of 16 consecutive elements
 *                      (k = 16q + e) the bytes hold the elements in the order
 *                      e = 0,2,4,6, 8,10,12,14, 1,3,5,7, 9,11,13,15 (element e sits at
 *                      byte 16q + 8(e%2) + 4(e/8) + (e%8)/2).  The values are the same;
 *                      this order matches a cheaper unpack of the packed weights, so
 *                      the forward runs faster on it.
 *   BL_XQ_K16_STRIDE4  K % 16 == 0; inside every group of 16 consecutive elements the
 *                      bytes hold e = 0,4,8,12, 1,5,9,13, 2,6,10,14, 3,7,11,15 (element e
 *                      sits at byte 16q + 4(e%4) + e/4).  This order matches the unpack
 *                      with the fewest integer instructions, which the fastest decode
 *                      and prefill kernels use. */
typedef enum {
    BL_XQ_ROWMAJOR = 0,
    BL_XQ_K16_EVENODD = 1,
    BL_XQ_K16_STRIDE4 = 2
} bl_xq_layout;

/* Bytes of device workspace bitlinear_quantize_weights needs for an [N, K] matrix
 * (fp64 partial sums of |W|).  Depends on N*K only; 0 for a non-positive size. */
BL_API size_t bitlinear_workspace_size(int64_t N, int64_t K);

/* [B158] absmean ternarisation and packing of one weight matrix.
 *   W          in  : fp32 [N, K] row-major, device.
 *   eps        in  : > 0, finite; gamma = fp32(mean|W|) + eps (fp32 add).
 *   gamma_out  out : device fp32 scalar; written by the kernels, never read back here.
 *   packed_out out : device uint8 [N, K/4] in the packed format above.
 *   ws, ws_bytes   : device workspace of at least bitlinear_workspace_size(N, K) bytes,
 *                    scratch for the duration of the enqueued work.
 * The sum of |W| is accumulated in fp64 per thread and per block, and the block
 * partials are summed in a fixed order, so gamma is deterministic from run to run.
 * Codes: clip(rint(W / gamma), -1, 1) with an IEEE fp32 division.
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE (K % 4), BL_ERR_MISALIGNED,
 * BL_ERR_WORKSPACE, BL_ERR_CUDA. */
BL_API bl_status bitlinear_quantize_weights(const float *W, int64_t N, int64_t K, float eps,
                                     float *gamma_out, uint8_t *packed_out,
                                     void *ws, size_t ws_bytes, void *stream);

/* [B158] the RoundClip step alone, with the scale supplied by the caller.
 *   W      in  : fp32 [N, K], device.
 *   gamma  in  : device fp32 scalar, the full divisor (mean|W| + eps), > 0.
 *   packed_out out : device uint8 [N, K/4].
 * Errors: as bitlinear_quantize_weights, without BL_ERR_WORKSPACE. */
BL_API bl_status bitlinear_quantize_weights_with_scale(const float *W, int64_t N, int64_t K,
                                                const float *gamma, uint8_t *packed_out,
                                                void *stream);

/* [CH2] pack ternary codes given as int8.
 *   codes      in  : int8 [N, K] in {-1, 0, +1}, device.
 *   packed_out out : device uint8 [N, K/4].
 *   err_word   out : optional; BL_ERRBIT_BAD_CODE is OR-ed in if any code is outside
 *                    {-1, 0, +1}; such a code is written as 00 (zero).
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE, BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_pack(const int8_t *codes, int64_t N, int64_t K, uint8_t *packed_out,
                         int32_t *err_word, void *stream);

/* [BIN] + [CH2] per-token absmax int8 quantisation with no zero point.
 *   X      in  : bf16 [M, K] as raw uint16 bit patterns, device.  Finite values.
 *   eps    in  : > 0, finite.
 *   xq_out out : int8 [M, K], device: clip(rint(x * s_m), -128, 127).
 *   s_out  out : fp32 [M], device: s_m = 127 / max(max_k |x_mk|, eps) (IEEE division).
 * Any K >= 1 is accepted.  Errors: BL_ERR_INVALID_ARG, BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_quantize_act(const uint16_t *X, int64_t M, int64_t K, float eps,
                                 int8_t *xq_out, float *s_out, void *stream);

/* bitlinear_quantize_act writing x_q in the given layout (see bl_xq_layout).
 * The k16 layouts need K % 16 == 0 and K <= 2^30 (else BL_ERR_UNSUPPORTED_SHAPE). */
BL_API bl_status bitlinear_quantize_act_layout(const uint16_t *X, int64_t M, int64_t K, float eps,
                                               int8_t *xq_out, float *s_out, bl_xq_layout layout,
                                               void *stream);

/* Kind of the per-token normalisation in front of the quantiser. */
typedef enum {
    BL_NORM_RMS = 0,   /* RMSNorm: mu = 0 */
    BL_NORM_LAYER = 1  /* LayerNorm without a bias: mu = mean of the token */
} bl_norm_kind;

/* [BIN] Quant(LN(x)): the normalisation in front of the activation quantiser, fused
 * with it ("LN = LayerNorm before quant"; [B158]: the b1.58 models use the LLaMA-style
 * RMSNorm).  Per token m:
 *   mu = 0 (BL_NORM_RMS) or sum_k x_mk / K (BL_NORM_LAYER)
 *   v = sum_k (x_mk - mu)^2 / K;   r = 1 / sqrt(v + norm_eps)
 * in double precision, then mu and r rounded once to fp32;
 *   x_n = ((x_mk - mu) * r) * w_k    (fp32, w = norm_weight, or 1 when NULL)
 * then the quantiser of bitlinear_quantize_act on x_n:
 *   s_m = 127 / max(max_k |x_n|, eps);   x_q = clip(rint(x_n * s_m), -128, 127).
 * The sums run in a parallel order; a sequential sum differs by ~1e-16 relative, which
 * changes mu or r only when they lie that close to an fp32 rounding boundary.
 *   X           in  : bf16 [M, K] as raw uint16 bit patterns, device.  Finite values.
 *   norm_weight in  : fp32 [K], device, or NULL.
 *   norm_kind   in  : bl_norm_kind.
 *   norm_eps    in  : >= 0, finite.
 *   eps         in  : > 0, finite.
 *   xq_out      out : int8 [M, K], device, in the given layout (see bl_xq_layout).
 *   s_out       out : fp32 [M], device.
 * K % 8 == 0 (K % 16 == 0 for the k16 layouts), K <= 2^30 (else
 * BL_ERR_UNSUPPORTED_SHAPE).  Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE,
 * BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_norm_quantize_act(const uint16_t *X, const float *norm_weight, int64_t M, int64_t K,
                                             bl_norm_kind norm_kind, float norm_eps, float eps, int8_t *xq_out,
                                             float *s_out, bl_xq_layout layout, void *stream);

/* [BIN] + [STE] + [CH2] the BitLinear forward from quantised operands:
 *   acc[m, n] = sum_k x_q[m, k] * c[n, k]   (exact, int32)
 *   y[m, n]   = float(acc[m, n]) * (gamma / s[m])   (fp32: the quotient and the product
 *               are each rounded to nearest, so y is within 2^-23 relative of the exact
 *               value; bf16 output is the round-to-nearest-even of that fp32 value)
 *   xq      in  : int8 [M, K], device.
 *   s       in  : fp32 [M], device (ignored for BL_OUT_I32 but must be valid).
 *   packed  in  : uint8 [N, K/4] packed codes, device.
 *   gamma   in  : device fp32 scalar.
 *   out     out : [M, N] of out_dtype, device.
 *   err_word out: optional; BL_ERRBIT_TIMEOUT if a bounded device wait gave up (the
 *                 output is then incomplete).
 * M <= 16 runs the register-unpack GEMV; 16 < M <= 64 the small-batch tcgen05 kernel (up
 * to 32 tokens with x_q in BL_XQ_K16_STRIDE4, the GEMV fed by asynchronous copies where its
 * shape conditions hold) and larger M the tiled tcgen05 kind::i8 path, when K % 64 == 0
 * (else the GEMV).  K * 127 must stay below 2^31.
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE, BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_forward(const int8_t *xq, const float *s, const uint8_t *packed,
                            const float *gamma, int64_t M, int64_t N, int64_t K, void *out,
                            bl_dtype out_dtype, int32_t *err_word, void *stream);

/* bitlinear_forward with the kernel choice forced (testing both paths at any M). */
BL_API bl_status bitlinear_forward_path(const int8_t *xq, const float *s, const uint8_t *packed,
                                 const float *gamma, int64_t M, int64_t N, int64_t K, void *out,
                                 bl_dtype out_dtype, int32_t *err_word, bl_path path,
                                 void *stream);

/* A test of the bounded device waits (the source pages have no counterpart): the forward
 * of bitlinear_forward_layout on one of the kernels that wait for TMA loads
 * (BL_PATH_TC_1SM, BL_PATH_SKINNY, or BL_PATH_GEMV_TMA -- BL_PATH_GEMV is read as
 * BL_PATH_GEMV_TMA here -- with its shape conditions), in which every wait gives up after
 * wait_limit_ns (0 < wait_limit_ns <= 2 s; the forward entry points use 2 s) and the
 * load producer of each block stops after stall_after_loads loads.  The waits for the
 * next load then run out: the kernel stops its other roles, lets every copy and MMA in
 * flight finish, frees its tensor memory, ORs BL_ERRBIT_TIMEOUT into err_word and
 * returns; the output is left incomplete.  If a block needs no more loads than
 * stall_after_loads it finishes normally.  The next call on the stream runs as usual.
 * Errors: those of bitlinear_forward_layout; BL_ERR_INVALID_ARG for another path or a
 * limit out of range, BL_ERR_UNSUPPORTED_SHAPE for a shape the TMA-fed GEMV does not take. */
BL_API bl_status bitlinear_forward_stall_test(const int8_t *xq, const float *s, const uint8_t *packed,
                                              const float *gamma, int64_t M, int64_t N, int64_t K, void *out,
                                              bl_dtype out_dtype, int32_t *err_word, bl_xq_layout xq_layout,
                                              bl_path path, uint64_t wait_limit_ns, int32_t stall_after_loads,
                                              void *stream);

/* bitlinear_quantize_weights for callers that cannot allocate device memory.  The
 * source pages have no counterpart to this entry point; it exists for the library's
 * users.  Callers such as a serving loop that must not call cudaMalloc (which can
 * synchronise the whole device), a plug-in whose host framework owns all device
 * memory, or a deployment with a device memory budget fixed at start-up have no
 * workspace to pass.  This variant keeps the fp64 partial sums of |W| in a fixed
 * array inside the library instead:
 *   - The array holds 1184 doubles (9472 bytes).  Every GPU that loads the library
 *     keeps it until the process exits.  Every shape accepted by
 *     bitlinear_quantize_weights fits; a shape that would need more partial sums
 *     than the array holds returns BL_ERR_WORKSPACE.
 *   - Every call looks up the array's device address with the caller's device current
 *     (cudaGetSymbolAddress).  On the first call on a device that lookup may make the
 *     CUDA driver load this library's device code (lazy module loading), which places
 *     the array, with the kernels, in device memory.  Make that first call before any
 *     stream capture.
 *   - The call itself allocates and frees nothing (no cudaMalloc, no cudaFree, no
 *     allocating library routine).
 *   - All calls share the one array.  Calls that run at the same time on the GPU
 *     (for example on two streams) race and corrupt each other's gamma.  Serialise
 *     them.  A call never reads what an earlier call left in the array.
 * Arguments, results and the other errors are those of bitlinear_quantize_weights. */
BL_API bl_status bitlinear_quantize_weights_noalloc(const float *W, int64_t N, int64_t K, float eps,
                                                    float *gamma_out, uint8_t *packed_out,
                                                    void *stream);

/* bitlinear_forward_path reading x_q stored in the given layout (see bl_xq_layout);
 * the result is the same for every layout.  The k16 layouts need K % 16 == 0.  With
 * BL_XQ_K16_STRIDE4 the tensor-core paths need K <= 2^17 (BL_PATH_AUTO runs the GEMV
 * above that; a forced BL_PATH_TC* returns BL_ERR_UNSUPPORTED_SHAPE). */
BL_API bl_status bitlinear_forward_layout(const int8_t *xq, const float *s, const uint8_t *packed,
                                          const float *gamma, int64_t M, int64_t N, int64_t K, void *out,
                                          bl_dtype out_dtype, int32_t *err_word, bl_xq_layout xq_layout,
                                          bl_path path, void *stream);

/* bitlinear_forward_layout with one weight scale per output row, for several BitLinear
 * matrices stacked along N (q/k/v, or up/gate) that keep their own absmean gamma
 * ([B158]: gamma is a per-matrix mean), run as one launch:
 *   y[m, n] = float(acc[m, n]) * (gamma_rows[n] / s[m])
 *   gamma_rows in : fp32 [N], device, 16-byte aligned; every other argument, result
 *                   and error as for bitlinear_forward_layout (BL_OUT_I32 ignores it).
 * Stack the packed rows of the matrices and fill gamma_rows with each matrix's gamma
 * repeated over its rows. */
BL_API bl_status bitlinear_forward_rowscale(const int8_t *xq, const float *s, const uint8_t *packed,
                                            const float *gamma_rows, int64_t M, int64_t N, int64_t K, void *out,
                                            bl_dtype out_dtype, int32_t *err_word, bl_xq_layout xq_layout,
                                            bl_path path, void *stream);

/* ----------------------------------------------------------------------------------
 * 1.6-bit weight format (TL5): five codes per byte.
 * [B158] "What it is (the intuition)": ternary weights pack to about 1.6 bits each in
 * practice; [CH2]: several values per storage unit, unpacked where they are used.
 * 3^5 = 243 <= 256, so a byte holds five codes (1.6 bits each, 20% fewer weight bytes
 * than the 2-bit format).
 *   uint8 [N, bitlinear_tl5_row_bytes(K)], row-major, K % 16 == 0.  A row is cut into
 *   blocks of 80 codes along K, 16 bytes per block; byte j (0..15) of block b holds the
 *   codes of k = 80 b + 16 p + j for p = 0..4 as the base-3 number
 *   v = sum_p (c_p + 1) 3^(4-p) (p = 0 most significant), stored in 8-bit fixed point
 *   B = ceil(256 v / 243) and read back as v = floor(243 B / 256).  Every byte value
 *   reads as five valid codes.  Codes past K (the missing planes of a last, partial
 *   block) are written as 0 and ignored by the forward.
 * ---------------------------------------------------------------------------------- */

/* Bytes per row of the TL5 format: 16 * ceil(K / 80); 0 if K <= 0 or K % 16 != 0. */
BL_API int64_t bitlinear_tl5_row_bytes(int64_t K);

/* Pack int8 codes into the TL5 format.
 *   codes   in  : int8 [N, K] in {-1, 0, +1}, device.
 *   tl5_out out : uint8 [N, bitlinear_tl5_row_bytes(K)], device.
 *   err_word out: optional; BL_ERRBIT_BAD_CODE is OR-ed in if a code is outside
 *                 {-1, 0, +1}; such a code is written as 0.
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE (K % 16), BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_pack_tl5(const int8_t *codes, int64_t N, int64_t K, uint8_t *tl5_out,
                                    int32_t *err_word, void *stream);

/* Convert the 2-bit packed format (uint8 [N, K/4], as written by
 * bitlinear_quantize_weights) into the TL5 format; a 2-bit code 11 becomes 0.
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE (K % 16), BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_repack_tl5(const uint8_t *packed, int64_t N, int64_t K, uint8_t *tl5_out,
                                      void *stream);

/* The BitLinear forward of bitlinear_forward with the weights in the TL5 format:
 *   acc[m, n] = sum_k x_q[m, k] c[n, k] (exact int32), y = float(acc) * (gamma / s[m]).
 *   xq  in : int8 [M, K] row-major (BL_XQ_ROWMAJOR), device.
 *   tl5 in : uint8 [N, bitlinear_tl5_row_bytes(K)], device.
 *   s, gamma, out, out_dtype: as for bitlinear_forward.
 * A decode kernel (one warp per output row, tokens in groups of up to 16): meant for
 * small M; larger M re-reads the weights once per 16 tokens.  K % 16 == 0,
 * K * 128 < 2^31, M <= 65535 * 16.
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE, BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_forward_tl5(const int8_t *xq, const float *s, const uint8_t *tl5,
                                       const float *gamma, int64_t M, int64_t N, int64_t K, void *out,
                                       bl_dtype out_dtype, void *stream);

/* ----------------------------------------------------------------------------------
 * Straight-through backward (quantisation-aware training).
 * [STE] the forward uses the ternary weights; the backward treats the quantisation as
 * the identity, so the gradient reaches the full-precision shadow weights.  For the
 * forward y[m, n] = (sum_k c[n, k] x_q[m, k]) * gamma / s[m] with both quantisers
 * passed straight through (d x_q / d x = s; gamma and s held constant):
 *   dX[m, k] = gamma * sum_n dY[m, n] c[n, k]
 *   dW[n, k] = gamma * sum_m dY[m, n] x_q[m, k] / s[m]
 * dX is the gradient for the quantiser's input (the normalised activations), dW the
 * gradient for the shadow weights.  Both run on the tensor cores (bf16 operands, fp32
 * accumulation): the codes and x_q are exact in bf16, and the fp32 factor (dY, or
 * dY * (1 / s[m]) with the reciprocal rounded to fp32) is split into two bf16 parts
 * hi + lo that together carry it to within 2^-16 relative; both parts meet the same
 * exact operand, so every product is exact and the sums round in fp32 (in the tensor
 * cores' order).  The result is scaled by gamma once.
 * ---------------------------------------------------------------------------------- */

/*   dY     in  : fp32 [M, N], device.
 *   packed in  : uint8 [N, K/4] 2-bit codes (the forward's weights), device.
 *   gamma  in  : device fp32 scalar.
 *   dX     out : fp32 [M, K], device.
 * K % 4 == 0; M, N, K < 2^31.
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE, BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_ste_backward_input(const float *dY, const uint8_t *packed, const float *gamma,
                                              int64_t M, int64_t N, int64_t K, float *dX, void *stream);

/*   dY    in  : fp32 [M, N], device.
 *   xq, s in  : the forward's int8 [M, K] row-major activations and fp32 [M] scales, device.
 *   gamma in  : device fp32 scalar.
 *   dW    out : fp32 [N, K], device.
 * K % 4 == 0; M, N, K < 2^31.
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_UNSUPPORTED_SHAPE, BL_ERR_MISALIGNED, BL_ERR_CUDA. */
BL_API bl_status bitlinear_ste_backward_weight(const float *dY, const int8_t *xq, const float *s,
                                               const float *gamma, int64_t M, int64_t N, int64_t K, float *dW,
                                               void *stream);

/* CUDA error code (cudaError_t as int) of the last BL_ERR_CUDA on the calling thread. */
BL_API int bitlinear_last_cuda_error(void);

/* Static string naming a bl_status value. */
BL_API const char *bitlinear_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
