/*
 * bitlinear_oracle.c -- plain, slow, single-threaded CPU oracle of the BitNet b1.58
 * BitLinear forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA library; it is written
 * from the definitions on the source pages, step by step, with no blocking, fusion or
 * reordering beyond what those definitions state.
 *
 * Sources (page title -- section):
 *   [B158]  "1-bit & Ternary LLMs (BitNet b1.58)" -- "How it works (real mechanics)",
 *           block "BitNet b1.58 (Feb 2024)": gamma = (1/nm) sum_ij |W_ij|,
 *           W~ = RoundClip(W / (gamma + eps), -1, 1), RoundClip(x,a,b) = max(a, min(b, round(x))).
 *   [BIN]   same page, block "BitNet (Oct 2023)": absmax per-token activation quantiser
 *           Quant(x) = Clip(x * Q_b / ||x||_inf, ...) and the forward
 *           y = W~ . Quant(LN(x)) . (beta * gamma / Q_b)  (one float rescale at the end).
 *   [STE]   same page, "Training: shadow weights + the straight-through estimator":
 *           gamma = |W|.mean(); W_tern = round_clip(W/(gamma+eps)); y = (W @ x_q) * scale.
 *   [CH2]   "What 1.58 Bits Actually Changes" -- "How the low-bit linear path works":
 *           per-token signed 8-bit activations with no zero point; +1 adds, -1 subtracts,
 *           0 skips; a GPU implementation packs several ternary values per storage unit.
 *   [MR]    "1.58 bits: what BitNet promised and what it required" -- "Three values per
 *           weight": absmean, activations at 8 bits per token without a zero point.
 *
 * Readings taken where the pages are silent (each is listed with its reason in the
 * design notes of this repository):
 *   - round() is round-half-to-even (rintf under the default FE_TONEAREST mode).
 *   - eps is a caller argument; gamma as used everywhere (division and output scale)
 *     is mean|W| + eps, the addition done in fp32.
 *   - the activation scale is Q_b = 127 with clip range [-128, 127]:
 *     s = 127 / max(absmax, eps); x_q = clip(round(x * s), -128, 127).
 *   - divisions are true IEEE fp32 divisions, never a reciprocal multiply.
 *   - 2-bit code format: 00 -> 0, 01 -> +1, 10 -> -1, four codes per byte along K,
 *     code of element k = 4j + i at bits 2i..2i+1 of byte j (LSB first), rows of K/4 bytes.
 *     Code 11 is never written; when decoded it reads as 0.
 *   - output y = acc * gamma / s, evaluated in double and rounded once to fp32; bf16
 *     output is the round-to-nearest-even of that fp32 value.
 *
 * Build: plain C99, no SIMD intrinsics, no -ffast-math, -ffp-contract=off.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* ---------------------------------------------------------------- weights -- */

/* [B158] gamma = (1/nm) sum |W_ij|, then + eps.  The sum runs in index order in
 * double precision; the quotient is rounded to fp32 and eps is added in fp32. */
float oracle_absmean_gamma(const float *W, int64_t N, int64_t K, float eps)
{
    double sum = 0.0;
    int64_t n, k;
    for (n = 0; n < N; ++n)
        for (k = 0; k < K; ++k)
            sum += fabs((double)W[n * K + k]);
    float mean = (float)(sum / (double)(N * K));
    float gamma = mean + eps;
    return gamma;
}

/* [B158] RoundClip(W / gamma, -1, 1) with gamma already holding the + eps term.
 * One IEEE fp32 division per weight, round half to even, clip to [-1, 1]. */
void oracle_ternarise(const float *W, int64_t N, int64_t K, float gamma, int8_t *codes)
{
    int64_t i;
    for (i = 0; i < N * K; ++i) {
        float q = rintf(W[i] / gamma);
        if (q < -1.0f) q = -1.0f;
        if (q > 1.0f) q = 1.0f;
        codes[i] = (int8_t)q;
    }
}

/* 2-bit code of one ternary value: 0 -> 00, +1 -> 01, -1 -> 10.  Returns -1 for a
 * value outside {-1, 0, +1}. */
static int encode_code(int8_t c)
{
    if (c == 0) return 0;
    if (c == 1) return 1;
    if (c == -1) return 2;
    return -1;
}

/* [CH2] packing: four codes per byte along K, element k = 4j + i at bits 2i..2i+1 of
 * byte j of its row.  Invalid codes are written as 00 and counted; the count is
 * returned. */
int64_t oracle_pack(const int8_t *codes, int64_t N, int64_t K, uint8_t *packed)
{
    int64_t bad = 0, n, j;
    int i;
    int64_t KB = K / 4;
    for (n = 0; n < N; ++n) {
        for (j = 0; j < KB; ++j) {
            unsigned byte = 0;
            for (i = 0; i < 4; ++i) {
                int e = encode_code(codes[n * K + 4 * j + i]);
                if (e < 0) { ++bad; e = 0; }
                byte |= (unsigned)e << (2 * i);
            }
            packed[n * KB + j] = (uint8_t)byte;
        }
    }
    return bad;
}

/* Inverse of oracle_pack: 00 -> 0, 01 -> +1, 10 -> -1, 11 -> 0. */
void oracle_unpack(const uint8_t *packed, int64_t N, int64_t K, int8_t *codes)
{
    int64_t n, k;
    int64_t KB = K / 4;
    for (n = 0; n < N; ++n) {
        for (k = 0; k < K; ++k) {
            unsigned byte = packed[n * KB + k / 4];
            unsigned c = (byte >> (2 * (k % 4))) & 3u;
            codes[n * K + k] = (int8_t)(c == 1u ? 1 : (c == 2u ? -1 : 0));
        }
    }
}

/* ------------------------------------------------ 1.6-bit packing (TL5) -- */

/* [B158] "What it is (the intuition)": a ternary weight carries log2(3) ~ 1.58 bits
 * and packs to about 1.6 bits in practice; [CH2]: several ternary values share a
 * storage unit and are unpacked where they are used.  Reading: five values per byte,
 * since 3^5 = 243 <= 256, which is 1.6 bits per value exactly.  The layout (reading;
 * the pages fix none):
 *   - digit t = c + 1 in {0, 1, 2} for code c in {-1, 0, +1};
 *   - a row is cut into blocks of 80 values along K, block b taking 16 bytes; byte j
 *     (0..15) of block b holds the values k = 80 b + 16 p + j for p = 0..4 as the
 *     base-3 number v = sum_p t_p 3^(4-p) (p = 0 the most significant digit);
 *   - the byte holds v in 8-bit fixed point, B = ceil(v * 256 / 243), and is read
 *     back as v = floor(B * 243 / 256), which is defined for every byte value;
 *   - positions k >= K of the last block are written as code 0 and never read.
 * A row takes 16 * ceil(K / 80) bytes; K is a multiple of 16. */
int64_t oracle_tl5_row_bytes(int64_t K)
{
    return 16 * ((K + 79) / 80);
}

/* Codes outside {-1, 0, +1} are written as 0 and counted; the count is returned. */
int64_t oracle_pack_tl5(const int8_t *codes, int64_t N, int64_t K, uint8_t *packed)
{
    int64_t bad = 0, n, b, j;
    int p;
    int64_t RB = oracle_tl5_row_bytes(K);
    for (n = 0; n < N; ++n) {
        for (b = 0; b < RB / 16; ++b) {
            for (j = 0; j < 16; ++j) {
                unsigned v = 0;
                for (p = 0; p < 5; ++p) {
                    int64_t k = 80 * b + 16 * p + j;
                    int t = 1;
                    if (k < K) {
                        int8_t code = codes[n * K + k];
                        if (code == -1 || code == 0 || code == 1)
                            t = code + 1;
                        else
                            ++bad;
                    }
                    v = 3 * v + (unsigned)t;
                }
                packed[n * RB + 16 * b + j] = (uint8_t)((v * 256u + 242u) / 243u);
            }
        }
    }
    return bad;
}

/* Inverse of oracle_pack_tl5 for every byte value. */
void oracle_unpack_tl5(const uint8_t *packed, int64_t N, int64_t K, int8_t *codes)
{
    int64_t n, k;
    int64_t RB = oracle_tl5_row_bytes(K);
    for (n = 0; n < N; ++n) {
        for (k = 0; k < K; ++k) {
            int64_t b = k / 80, r = k % 80;
            int p = (int)(r / 16), i;
            unsigned byte = packed[n * RB + 16 * b + r % 16];
            unsigned v = byte * 243u / 256u;
            unsigned w = 1;
            for (i = 0; i < 4 - p; ++i) w *= 3u;
            codes[n * K + k] = (int8_t)((int)(v / w % 3u) - 1);
        }
    }
}

/* ------------------------------------------------------------ activations -- */

/* bf16 -> fp32 is exact: the bf16 bit pattern is the top half of the fp32 one. */
static float bf16_bits_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* [BIN] absmax per token, [CH2]/[MR] per token with no zero point, scaled to the
 * signed 8-bit range Q_b = 127:
 *   a = max_k |x_k|;  s = 127 / max(a, eps);  x_q = clip(round(x * s), -128, 127).
 * x * s is one fp32 multiply; round is half to even. */
void oracle_quantize_act(const uint16_t *X, int64_t M, int64_t K, float eps,
                         int8_t *xq, float *s_out)
{
    int64_t m, k;
    for (m = 0; m < M; ++m) {
        float a = 0.0f;
        for (k = 0; k < K; ++k) {
            float v = fabsf(bf16_bits_to_float(X[m * K + k]));
            if (v > a) a = v;
        }
        float s = 127.0f / fmaxf(a, eps);
        s_out[m] = s;
        for (k = 0; k < K; ++k) {
            float q = rintf(bf16_bits_to_float(X[m * K + k]) * s);
            if (q < -128.0f) q = -128.0f;
            if (q > 127.0f) q = 127.0f;
            xq[m * K + k] = (int8_t)q;
        }
    }
}

/* [BIN] Quant(LN(x)): the per-token normalisation in front of the activation
 * quantiser ("LN = LayerNorm before quant"; [B158]: b1.58 adopts LLaMA-style components, the
 * RMSNorm among them).  For each token:
 *   kind 0 (RMSNorm):   mu = 0
 *   kind 1 (LayerNorm): mu = (sum_k x_k) / K
 *   v = (sum_k (x_k - mu)^2) / K;   r = 1 / sqrt(v + norm_eps)
 * with the sums, mu, v and r in double precision (sums in index order); mu and r are
 * then rounded once to fp32, and each element is normalised in fp32, one IEEE rounding
 * per operation, left to right:
 *   x_n[k] = ((x_k - mu) * r) * w_k   (w = the per-channel norm weight, 1 when absent).
 * x_n then goes through the activation quantiser of oracle_quantize_act, in fp32:
 *   a = max_k |x_n[k]|;  s = 127 / max(a, eps);  x_q = clip(round(x_n * s), -128, 127).
 * xn_out (may be NULL) receives x_n. */
void oracle_norm_quantize_act(const uint16_t *X, const float *w, int64_t M, int64_t K, int kind,
                              float norm_eps, float eps, int8_t *xq, float *s_out, float *xn_out)
{
    int64_t m, k;
    float *xn = (float *)malloc((size_t)K * sizeof(float));
    if (xn == NULL) return;
    for (m = 0; m < M; ++m) {
        double mu = 0.0, v = 0.0;
        if (kind == 1) {
            for (k = 0; k < K; ++k) mu += (double)bf16_bits_to_float(X[m * K + k]);
            mu = mu / (double)K;
        }
        for (k = 0; k < K; ++k) {
            double d = (double)bf16_bits_to_float(X[m * K + k]) - mu;
            v += d * d;
        }
        v = v / (double)K;
        const float mu32 = (float)mu;
        const float r32 = (float)(1.0 / sqrt(v + (double)norm_eps));
        float a = 0.0f;
        for (k = 0; k < K; ++k) {
            const float wk = (w != NULL) ? w[k] : 1.0f;
            const float d32 = bf16_bits_to_float(X[m * K + k]) - mu32;
            const float t32 = d32 * r32;
            xn[k] = t32 * wk;
            if (fabsf(xn[k]) > a) a = fabsf(xn[k]);
        }
        const float s = 127.0f / fmaxf(a, eps);
        s_out[m] = s;
        for (k = 0; k < K; ++k) {
            float q = rintf(xn[k] * s);
            if (q < -128.0f) q = -128.0f;
            if (q > 127.0f) q = 127.0f;
            xq[m * K + k] = (int8_t)q;
            if (xn_out != NULL) xn_out[m * K + k] = xn[k];
        }
    }
    free(xn);
}

/* --------------------------------------------------------------- forward -- */

/* [CH2] acc[m][n] = sum_k x_q[m][k] * c[n][k] with c in {-1, 0, +1}: the product is
 * "add x", "subtract x" or "skip", accumulated exactly in int64.  Returns the number
 * of sums that do not fit in int32 (those are stored saturated). */
int64_t oracle_int_matmul(const int8_t *xq, const int8_t *codes, int64_t M, int64_t N,
                          int64_t K, int32_t *acc)
{
    int64_t over = 0, m, n, k;
    for (m = 0; m < M; ++m) {
        for (n = 0; n < N; ++n) {
            int64_t sum = 0;
            for (k = 0; k < K; ++k) {
                int8_t c = codes[n * K + k];
                if (c == 1) sum += xq[m * K + k];
                else if (c == -1) sum -= xq[m * K + k];
            }
            if (sum > INT32_MAX) { ++over; sum = INT32_MAX; }
            if (sum < INT32_MIN) { ++over; sum = INT32_MIN; }
            acc[m * N + n] = (int32_t)sum;
        }
    }
    return over;
}

/* [BIN]/[STE] the single float rescale: y = acc * gamma / s_m, in double, rounded
 * once to fp32. */
void oracle_dequant(const int32_t *acc, const float *s, float gamma, int64_t M, int64_t N,
                    float *y)
{
    int64_t m, n;
    for (m = 0; m < M; ++m)
        for (n = 0; n < N; ++n)
            y[m * N + n] = (float)((double)acc[m * N + n] * (double)gamma / (double)s[m]);
}

/* The rescale with one weight scale per output row, for several matrices stacked
 * along N (each keeps its own absmean gamma, [B158]): y[m][n] = acc[m][n] * gamma_n / s[m],
 * evaluated in double and rounded once to fp32, as in oracle_dequant. */
void oracle_dequant_rows(const int32_t *acc, const float *s, const float *gamma_rows, int64_t M, int64_t N,
                         float *y)
{
    int64_t m, n;
    for (m = 0; m < M; ++m)
        for (n = 0; n < N; ++n)
            y[m * N + n] = (float)((double)acc[m * N + n] * (double)gamma_rows[n] / (double)s[m]);
}

/* fp32 -> bf16 with round to nearest, ties to even (finite inputs). */
void oracle_f32_to_bf16(const float *y, int64_t n, uint16_t *out)
{
    int64_t i;
    for (i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &y[i], sizeof u);
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7FFFu + lsb;
        out[i] = (uint16_t)(u >> 16);
    }
}

/* Whole forward from the packed format: decode every row of the packed matrix, form
 * the exact integer products, then rescale.  out_kind: 0 = fp32, 1 = bf16 bits,
 * 2 = raw int32 accumulators.  codes_tmp must hold N*K bytes, acc_tmp M*N int32. */
int64_t oracle_forward(const int8_t *xq, const float *s, const uint8_t *packed, float gamma,
                       int64_t M, int64_t N, int64_t K, int out_kind, void *out,
                       int8_t *codes_tmp, int32_t *acc_tmp, float *y_tmp)
{
    oracle_unpack(packed, N, K, codes_tmp);
    int64_t over = oracle_int_matmul(xq, codes_tmp, M, N, K, acc_tmp);
    if (out_kind == 2) {
        memcpy(out, acc_tmp, (size_t)(M * N) * sizeof(int32_t));
        return over;
    }
    if (out_kind == 0) {
        oracle_dequant(acc_tmp, s, gamma, M, N, (float *)out);
        return over;
    }
    oracle_dequant(acc_tmp, s, gamma, M, N, y_tmp);
    oracle_f32_to_bf16(y_tmp, M * N, (uint16_t *)out);
    return over;
}

/* The forward from the 1.6-bit format: decode it, then the same integer products and
 * rescale as oracle_forward. */
int64_t oracle_forward_tl5(const int8_t *xq, const float *s, const uint8_t *packed, float gamma,
                           int64_t M, int64_t N, int64_t K, int out_kind, void *out,
                           int8_t *codes_tmp, int32_t *acc_tmp, float *y_tmp)
{
    oracle_unpack_tl5(packed, N, K, codes_tmp);
    int64_t over = oracle_int_matmul(xq, codes_tmp, M, N, K, acc_tmp);
    if (out_kind == 2) {
        memcpy(out, acc_tmp, (size_t)(M * N) * sizeof(int32_t));
        return over;
    }
    if (out_kind == 0) {
        oracle_dequant(acc_tmp, s, gamma, M, N, (float *)out);
        return over;
    }
    oracle_dequant(acc_tmp, s, gamma, M, N, y_tmp);
    oracle_f32_to_bf16(y_tmp, M * N, (uint16_t *)out);
    return over;
}

/* ------------------------------------------- straight-through backward (STE) -- */

/* [STE] the forward uses the ternary weights while the gradient reaches the shadow
 * weights as if the quantisation were the identity.  With this library's forward
 * y[m,n] = (sum_k c[n,k] x_q[m,k]) * gamma / s[m], and both quantisers passed straight
 * through (x_q = round(s x) with d x_q / d x = s, gamma and s held constant):
 *   dX[m,k] = gamma * sum_n dY[m,n] c[n,k]
 *   dW[n,k] = gamma * sum_m dY[m,n] x_q[m,k] / s[m]
 * Both sums run in index order in double precision and are rounded once to fp32.
 * codes_tmp must hold N*K bytes. */
void oracle_ste_grad_input(const float *dY, const uint8_t *packed, float gamma, int64_t M, int64_t N,
                           int64_t K, float *dX, int8_t *codes_tmp)
{
    int64_t m, n, k;
    oracle_unpack(packed, N, K, codes_tmp);
    for (m = 0; m < M; ++m) {
        for (k = 0; k < K; ++k) {
            double sum = 0.0;
            for (n = 0; n < N; ++n)
                sum += (double)dY[m * N + n] * (double)codes_tmp[n * K + k];
            dX[m * K + k] = (float)((double)gamma * sum);
        }
    }
}

void oracle_ste_grad_weight(const float *dY, const int8_t *xq, const float *s, float gamma, int64_t M,
                            int64_t N, int64_t K, float *dW)
{
    int64_t m, n, k;
    for (n = 0; n < N; ++n) {
        for (k = 0; k < K; ++k) {
            double sum = 0.0;
            for (m = 0; m < M; ++m)
                sum += (double)dY[m * N + n] * (double)xq[m * K + k] / (double)s[m];
            dW[n * K + k] = (float)((double)gamma * sum);
        }
    }
}
