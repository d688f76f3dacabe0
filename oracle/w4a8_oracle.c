/*
 * CPU oracle for the W4A8 per-output-channel quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, obviously correct
 * statement of what the layer computes. Only the test-suite, the package's
 * smoke check and the benchmark's CPU-baseline leg may load it; the product
 * path never calls it and shares no code with it.
 *
 * Method: Keras guide "INT4 quantization in Keras", section "How it works",
 * steps 1-6, and section "What Keras does in INT4 mode":
 *   1. per-output-channel symmetric abs-max scale for each weight matrix;
 *   2. weights quantized to [-8, 7] and packed two per byte;
 *   3. activations scaled and quantized to INT8 dynamically at inference;
 *   4. packed INT4 unpacked to INT8 (values still in the INT4 range);
 *   5. INT8 x INT8 matmul accumulated in INT32;
 *   6. result dequantized with (input_scale * per_channel_kernel_scale).
 * Constants the page leaves open are read as follows (each is a reading, not
 * a quote): weight scale sw = 7 / max|W[:,n]| used as a multiplier; rounding
 * half to even; clamp after rounding; nibbles packed along K with the even k
 * in the low nibble; zero column -> sw = 1; per-row activation scale
 * sx = 127 / max|X[m,:]| (1 for an all-zero row), INT8 clamp [-127, 127];
 * dequantization y = float(acc) / (sx * sw).
 *
 * W8A8 (the INT8 path that the same page says INT4 extends, section "How it
 * works", closing paragraph): steps 1-6 with 8-bit weights and no packing.
 * The page names that path without its constants; read here as the INT4
 * path's arithmetic with the 8-bit symmetric range of its own activation
 * step: sw = 127 / max|W[:,n]| (1 for a zero column), q = clamp(rne(w * sw),
 * -127, 127), one byte per code, rows of ldw8 >= K bytes with zero pad.
 *
 * Asymmetric INT4 with a zero point (the uniform quantization of the "INT4"
 * concept page, section 4.1, asymmetric form; the formulas of the "4-bit
 * Integer Quantization for LLMs" page, section "Weight quantization"), per
 * output channel, with the activations as in step 3. The pages give
 * scale = (max - min) / (2^4 - 1), q = round(w / scale) + zero_point in
 * [0, 15] and w ~ (q - zero_point) * scale. Read here as: the multiplier
 * sa = 15 / (max - min) (1 when max == min) in place of the division, like
 * the symmetric scale; the integer zero point zp = -rne(min * sa), so that
 * the minimum maps to code 0; q = clamp(rne(w * sa) + zp, 0, 15) (the clamp
 * binds only when a tie lifts the maximum to 16); codes packed unsigned, two
 * per byte along K, even k in the low nibble; the product
 * acc = sum_k xq * (q - zp) and y = float(acc) / (sx * sa).
 *
 * Group-wise INT4 (the "INT4" concept page, section 4.2, group quantization:
 * each group of group_size weights along the input axis, e.g. 128, has its own
 * scale and zero point; the "4-bit Integer Quantization for LLMs" page's
 * quantization configuration names group_size 128): read as the zero-point
 * rule above applied to every (output channel n, group g of G consecutive k)
 * separately, the last group ragged when G does not divide K. The product is
 * the INT32 partial sum of each group, dequantized by its own scale and
 * summed over the groups in increasing g in float32:
 *   y = sum_g float(sum_{k in g} xq * (q - zp[n][g])) / (sx * sa[n][g]).
 *
 * Inputs outside the statement: non-finite values, and rows or weight
 * columns whose scale overflows float32 (a row abs-max below 127 / FLT_MAX,
 * a column abs-max below 7 / FLT_MAX): the pages define no scale there. Finite
 * scales whose product sx * sw overflows or underflows stay inside it and give
 * the IEEE quotient (acc / inf, acc / 0).
 *
 * Layer chaining (the minimal model's Dense -> Dense, each layer quantizing
 * its own float32 input): a layer's input row scale comes from that row's
 * abs-max whatever hands the maximum over, so a chain of linear() calls is
 * the statement of a chained model (mlp() below).
 *
 * Precision: the page's model is float32 end to end (its inputs are cast with
 * astype("float32")), and float32 decides every integer code, so each step
 * below runs in float32 with IEEE round-to-nearest. Build flags:
 * -O2 -ffp-contract=off -fno-fast-math (no FMA contraction).
 *
 * Every loop is the plain definition: no blocking, no fusion, no reordering.
 *
 * Return codes: 0 = ok, 1 = invalid argument, 2 = INT32 accumulator overflow.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_OVERFLOW 2

/* Round a float32 to the nearest integer, ties to even (the default IEEE
 * rounding mode, which nearbyintf follows). */
static float round_half_even(float t) { return nearbyintf(t); }

static int clamp_int(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* ---------------------------------------------------------------------------
 * Step 1: per-output-channel symmetric abs-max weight scale.
 * W is the Keras kernel layout [K][N] (row stride ldw floats); column n is
 * output channel n. sw[n] = 7 / max_k |W[k][n]|, or 1 for an all-zero column.
 * ------------------------------------------------------------------------- */
int oracle_weight_scales(const float *W, int K, int N, int ldw, float *sw)
{
    if (!W || !sw || K < 1 || N < 1 || ldw < N) return ORACLE_BAD_ARG;
    for (int n = 0; n < N; ++n) {
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(W[(size_t)k * ldw + n]);
            if (a > amax) amax = a;
        }
        sw[n] = (amax == 0.0f) ? 1.0f : 7.0f / amax;
    }
    return ORACLE_OK;
}

/* Step 2 for one element: q = clamp(round_half_even(w * sw), -8, 7). */
int oracle_quantize_weight(float w, float sw)
{
    float t = w * sw;
    return clamp_int((int)round_half_even(t), -8, 7);
}

/* Step 2 (packing): byte j of row n holds k = 2j in its low nibble and
 * k = 2j + 1 in its high nibble, each a two's-complement 4-bit value. */
static uint8_t nibble_of(int q) { return (uint8_t)(q & 0xF); }

/* Step 2 (packing) over a matrix of codes: Q[N][K] int8 in [-8, 7] ->
 * Wp[N][ldp]. Every byte of a row past the nibble of k = K-1 (the odd-K pad
 * nibble included) is 0. */
int oracle_w4_pack(const int8_t *Q, int K, int N, uint8_t *Wp, int ldp)
{
    if (!Q || !Wp || K < 1 || N < 1 || ldp < (K + 1) / 2) return ORACLE_BAD_ARG;
    for (int n = 0; n < N; ++n) {
        uint8_t *row = Wp + (size_t)n * ldp;
        memset(row, 0, (size_t)ldp);
        for (int k = 0; k < K; ++k) {
            int q = Q[(size_t)n * K + k];
            if (q < -8 || q > 7) return ORACLE_BAD_ARG;
            uint8_t nib = nibble_of(q);
            if (k % 2 == 0)
                row[k / 2] |= nib;
            else
                row[k / 2] |= (uint8_t)(nib << 4);
        }
    }
    return ORACLE_OK;
}

/* Steps 1-2 without packing: W[K][N] -> Q[N][K] codes and sw[N]. */
int oracle_w4_quantize(const float *W, int K, int N, int ldw, int8_t *Q, float *sw)
{
    if (!W || !Q || !sw || K < 1 || N < 1 || ldw < N) return ORACLE_BAD_ARG;
    int rc = oracle_weight_scales(W, K, N, ldw, sw);
    if (rc) return rc;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k)
            Q[(size_t)n * K + k] = (int8_t)oracle_quantize_weight(W[(size_t)k * ldw + n], sw[n]);
    return ORACLE_OK;
}

/* Steps 1-2: quantize W[K][N] and pack into Wp[N][ldp] (bytes). */
int oracle_w4_quantize_pack(const float *W, int K, int N, int ldw,
                            uint8_t *Wp, int ldp, float *sw)
{
    if (!W || !Wp || !sw || K < 1 || N < 1 || ldw < N || ldp < (K + 1) / 2)
        return ORACLE_BAD_ARG;
    int8_t *Q = (int8_t *)malloc((size_t)N * K);
    if (!Q) return ORACLE_BAD_ARG;
    int rc = oracle_w4_quantize(W, K, N, ldw, Q, sw);
    if (!rc) rc = oracle_w4_pack(Q, K, N, Wp, ldp);
    free(Q);
    return rc;
}

/* Step 4: the INT4 value of nibble k of packed row n, sign-extended. */
int oracle_unpack_weight(const uint8_t *Wp, int ldp, int n, int k)
{
    uint8_t byte = Wp[(size_t)n * ldp + k / 2];
    int v = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    return (v >= 8) ? v - 16 : v;
}

/* Step 4 over a whole matrix: Q[N][K] int8 from Wp[N][ldp]. */
int oracle_w4_unpack(const uint8_t *Wp, int K, int N, int ldp, int8_t *Q)
{
    if (!Wp || !Q || K < 1 || N < 1 || ldp < (K + 1) / 2) return ORACLE_BAD_ARG;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k)
            Q[(size_t)n * K + k] = (int8_t)oracle_unpack_weight(Wp, ldp, n, k);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 3: dynamic per-row abs-max INT8 activation quantization.
 * X[M][ldx] float32 -> Xq[M][ldq] int8 (bytes K..ldq-1 of a row are 0) and
 * sx[m] = 127 / max_k |X[m][k]| (1 for an all-zero row);
 * xq = clamp(round_half_even(x * sx), -127, 127).
 * ------------------------------------------------------------------------- */
int oracle_a8_quantize_rows(const float *X, int M, int K, int ldx,
                            int8_t *Xq, int ldq, float *sx)
{
    if (M < 0 || K < 1 || ldx < K || ldq < K) return ORACLE_BAD_ARG;
    if (M == 0) return ORACLE_OK;
    if (!X || !Xq || !sx) return ORACLE_BAD_ARG;
    for (int m = 0; m < M; ++m) {
        const float *x = X + (size_t)m * ldx;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(x[k]);
            if (a > amax) amax = a;
        }
        float s = (amax == 0.0f) ? 1.0f : 127.0f / amax;
        sx[m] = s;
        int8_t *q = Xq + (size_t)m * ldq;
        memset(q, 0, (size_t)ldq);
        for (int k = 0; k < K; ++k) {
            float t = x[k] * s;
            q[k] = (int8_t)clamp_int((int)round_half_even(t), -127, 127);
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Steps 4-5: acc[m][n] = sum_k xq[m][k] * q[n][k], accumulated exactly (int64)
 * and required to fit INT32, as the page's INT32 accumulator does.
 * ------------------------------------------------------------------------- */
int oracle_gemm_s32(const int8_t *Xq, int M, int K, int ldq,
                    const uint8_t *Wp, int N, int ldp,
                    int32_t *acc, int ldacc)
{
    if (M < 0 || K < 1 || N < 1 || ldq < K || ldp < (K + 1) / 2 || ldacc < N)
        return ORACLE_BAD_ARG;
    if (M == 0) return ORACLE_OK;
    if (!Xq || !Wp || !acc) return ORACLE_BAD_ARG;
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int k = 0; k < K; ++k)
                s += (int64_t)Xq[(size_t)m * ldq + k] * (int64_t)oracle_unpack_weight(Wp, ldp, n, k);
            if (s > INT32_MAX || s < INT32_MIN) return ORACLE_OVERFLOW;
            acc[(size_t)m * ldacc + n] = (int32_t)s;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 6 and the Dense epilogue: y = float(acc) / (sx[m] * sw[n]);
 * then y + b[n] when a bias is given; then ReLU (y > 0 ? y : +0) when asked.
 * (The minimal model's first Dense layer carries a bias and a ReLU.)
 * ------------------------------------------------------------------------- */
int oracle_dequant(const int32_t *acc, int M, int N, int ldacc,
                   const float *sx, const float *sw, const float *bias, int relu,
                   float *Y, int ldy)
{
    if (M < 0 || N < 1 || ldacc < N || ldy < N) return ORACLE_BAD_ARG;
    if (M == 0) return ORACLE_OK;
    if (!acc || !sx || !sw || !Y) return ORACLE_BAD_ARG;
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            float d = sx[m] * sw[n];
            float y = (float)acc[(size_t)m * ldacc + n] / d;
            if (bias) y = y + bias[n];
            if (relu) y = (y > 0.0f) ? y : 0.0f;
            Y[(size_t)m * ldy + n] = y;
        }
    }
    return ORACLE_OK;
}

/* float32 -> bfloat16 bits, round to nearest, ties to even (finite inputs). */
uint16_t oracle_f32_to_bf16(float y)
{
    uint32_t u;
    memcpy(&u, &y, sizeof u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

int oracle_f32_to_bf16_array(const float *y, size_t count, uint16_t *out)
{
    if (!y || !out) return ORACLE_BAD_ARG;
    for (size_t i = 0; i < count; ++i) out[i] = oracle_f32_to_bf16(y[i]);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * The whole forward of one quantized Dense layer, steps 3-6, on float32
 * input X[M][K] and packed weights. Xq/sx/acc are caller-provided scratch
 * (Xq: M*K bytes, sx: M floats, acc: M*N int32).
 * ------------------------------------------------------------------------- */
int oracle_linear(const float *X, int M, int K, int ldx,
                  const uint8_t *Wp, int ldp, const float *sw, int N,
                  const float *bias, int relu,
                  int8_t *Xq, float *sx, int32_t *acc,
                  float *Y, int ldy)
{
    int rc = oracle_a8_quantize_rows(X, M, K, ldx, Xq, K, sx);
    if (rc) return rc;
    rc = oracle_gemm_s32(Xq, M, K, K, Wp, N, ldp, acc, N);
    if (rc) return rc;
    return oracle_dequant(acc, M, N, N, sx, sw, bias, relu, Y, ldy);
}

/* ---------------------------------------------------------------------------
 * W8A8, steps 1-2: per-output-channel scale sw[n] = 127 / max_k |W[k][n]|
 * (1 for an all-zero column) and codes q = clamp(rne(w * sw), -127, 127),
 * stored one per byte: Q8[N][ldw8], bytes k >= K of each row 0.
 * ------------------------------------------------------------------------- */
int oracle_w8_quantize(const float *W, int K, int N, int ldw, int8_t *Q8, int ldw8, float *sw)
{
    if (!W || !Q8 || !sw || K < 1 || N < 1 || ldw < N || ldw8 < K) return ORACLE_BAD_ARG;
    for (int n = 0; n < N; ++n) {
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(W[(size_t)k * ldw + n]);
            if (a > amax) amax = a;
        }
        sw[n] = (amax == 0.0f) ? 1.0f : 127.0f / amax;
        int8_t *row = Q8 + (size_t)n * ldw8;
        memset(row, 0, (size_t)ldw8);
        for (int k = 0; k < K; ++k) {
            float t = W[(size_t)k * ldw + n] * sw[n];
            row[k] = (int8_t)clamp_int((int)round_half_even(t), -127, 127);
        }
    }
    return ORACLE_OK;
}

/* W8A8, step 5: acc[m][n] = sum_k xq[m][k] * q8[n][k], exact (int64) and
 * required to fit INT32. */
int oracle_gemm8_s32(const int8_t *Xq, int M, int K, int ldq,
                     const int8_t *Q8, int N, int ldw8,
                     int32_t *acc, int ldacc)
{
    if (M < 0 || K < 1 || N < 1 || ldq < K || ldw8 < K || ldacc < N) return ORACLE_BAD_ARG;
    if (M == 0) return ORACLE_OK;
    if (!Xq || !Q8 || !acc) return ORACLE_BAD_ARG;
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int k = 0; k < K; ++k)
                s += (int64_t)Xq[(size_t)m * ldq + k] * (int64_t)Q8[(size_t)n * ldw8 + k];
            if (s > INT32_MAX || s < INT32_MIN) return ORACLE_OVERFLOW;
            acc[(size_t)m * ldacc + n] = (int32_t)s;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Asymmetric INT4 with a zero point, steps 1-2 per output channel:
 * sa[n] = 15 / (max_k W[k][n] - min_k W[k][n]) (1 when they are equal),
 * zp[n] = -rne(min_k W[k][n] * sa[n]), q = clamp(rne(w * sa[n]) + zp[n], 0, 15),
 * packed as unsigned nibbles: byte j of row n = q[2j] | q[2j+1] << 4, every
 * byte past the nibble of k = K-1 zero.
 * ------------------------------------------------------------------------- */
int oracle_w4z_quantize_pack(const float *W, int K, int N, int ldw, uint8_t *Wp, int ldp,
                             float *sa, int32_t *zp)
{
    if (!W || !Wp || !sa || !zp || K < 1 || N < 1 || ldw < N || ldp < (K + 1) / 2) return ORACLE_BAD_ARG;
    for (int n = 0; n < N; ++n) {
        float lo = W[n], hi = W[n];
        for (int k = 1; k < K; ++k) {
            float w = W[(size_t)k * ldw + n];
            if (w < lo) lo = w;
            if (w > hi) hi = w;
        }
        float range = hi - lo;
        sa[n] = (range == 0.0f) ? 1.0f : 15.0f / range;
        zp[n] = -(int32_t)round_half_even(lo * sa[n]);
        uint8_t *row = Wp + (size_t)n * ldp;
        memset(row, 0, (size_t)ldp);
        for (int k = 0; k < K; ++k) {
            float t = W[(size_t)k * ldw + n] * sa[n];
            int q = clamp_int((int)round_half_even(t) + zp[n], 0, 15);
            if (k % 2 == 0)
                row[k / 2] |= (uint8_t)q;
            else
                row[k / 2] |= (uint8_t)(q << 4);
        }
    }
    return ORACLE_OK;
}

/* The unsigned code of nibble k of packed row n (zero-point layout). */
static int zp_code(const uint8_t *Wp, int ldp, int n, int k)
{
    uint8_t byte = Wp[(size_t)n * ldp + k / 2];
    return (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
}

/* acc[m][n] = sum_k xq[m][k] * (q[n][k] - zp[n]), exact (int64) and required
 * to fit INT32. */
int oracle_gemm_z_s32(const int8_t *Xq, int M, int K, int ldq, const uint8_t *Wp, int N, int ldp,
                      const int32_t *zp, int32_t *acc, int ldacc)
{
    if (M < 0 || K < 1 || N < 1 || ldq < K || ldp < (K + 1) / 2 || ldacc < N) return ORACLE_BAD_ARG;
    if (M == 0) return ORACLE_OK;
    if (!Xq || !Wp || !zp || !acc) return ORACLE_BAD_ARG;
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int k = 0; k < K; ++k)
                s += (int64_t)Xq[(size_t)m * ldq + k] * (int64_t)(zp_code(Wp, ldp, n, k) - zp[n]);
            if (s > INT32_MAX || s < INT32_MIN) return ORACLE_OVERFLOW;
            acc[(size_t)m * ldacc + n] = (int32_t)s;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Group-wise INT4: the zero-point rule per (output channel n, group g of G
 * consecutive k; the last group holds K - G * (ng - 1) of them), ng =
 * ceil(K / G). sa, zp are [N][ng]. Codes packed as for the zero-point form
 * (unsigned nibbles, even k low, zero pad).
 * ------------------------------------------------------------------------- */
int oracle_w4g_quantize_pack(const float *W, int K, int N, int ldw, int G, uint8_t *Wp, int ldp,
                             float *sa, int32_t *zp)
{
    if (!W || !Wp || !sa || !zp || K < 1 || N < 1 || G < 1 || ldw < N || ldp < (K + 1) / 2) return ORACLE_BAD_ARG;
    const int ng = (K + G - 1) / G;
    for (int n = 0; n < N; ++n) {
        uint8_t *row = Wp + (size_t)n * ldp;
        memset(row, 0, (size_t)ldp);
        for (int g = 0; g < ng; ++g) {
            const int k0 = g * G, k1 = (k0 + G < K) ? k0 + G : K;
            float lo = W[(size_t)k0 * ldw + n], hi = lo;
            for (int k = k0 + 1; k < k1; ++k) {
                float w = W[(size_t)k * ldw + n];
                if (w < lo) lo = w;
                if (w > hi) hi = w;
            }
            float range = hi - lo;
            float s = (range == 0.0f) ? 1.0f : 15.0f / range;
            int32_t z = -(int32_t)round_half_even(lo * s);
            sa[(size_t)n * ng + g] = s;
            zp[(size_t)n * ng + g] = z;
            for (int k = k0; k < k1; ++k) {
                float t = W[(size_t)k * ldw + n] * s;
                int q = clamp_int((int)round_half_even(t) + z, 0, 15);
                if (k % 2 == 0)
                    row[k / 2] |= (uint8_t)q;
                else
                    row[k / 2] |= (uint8_t)(q << 4);
            }
        }
    }
    return ORACLE_OK;
}

/* Group-wise product: per (m, n) the INT32 partial sum of each group (exact,
 * int64, required to fit INT32), dequantized by that group's scale and the
 * row scale, summed over increasing g in float32; then bias and ReLU as in
 * oracle_dequant. acc_g (M * N * ng int32) receives the partial sums. */
int oracle_linear_g_q(const int8_t *Xq, const float *sx, int M, int K, int ldq, const uint8_t *Wp, int N,
                      int ldp, int G, const float *sa, const int32_t *zp, const float *bias, int relu,
                      int32_t *acc_g, float *Y, int ldy)
{
    if (M < 0 || K < 1 || N < 1 || G < 1 || ldq < K || ldp < (K + 1) / 2 || ldy < N) return ORACLE_BAD_ARG;
    if (M == 0) return ORACLE_OK;
    if (!Xq || !sx || !Wp || !sa || !zp || !acc_g || !Y) return ORACLE_BAD_ARG;
    const int ng = (K + G - 1) / G;
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            float y = 0.0f;
            for (int g = 0; g < ng; ++g) {
                const int k0 = g * G, k1 = (k0 + G < K) ? k0 + G : K;
                int64_t s = 0;
                for (int k = k0; k < k1; ++k)
                    s += (int64_t)Xq[(size_t)m * ldq + k] *
                         (int64_t)(zp_code(Wp, ldp, n, k) - zp[(size_t)n * ng + g]);
                if (s > INT32_MAX || s < INT32_MIN) return ORACLE_OVERFLOW;
                acc_g[((size_t)m * N + n) * ng + g] = (int32_t)s;
                float d = sx[m] * sa[(size_t)n * ng + g];
                y = y + (float)s / d;
            }
            if (bias) y = y + bias[n];
            if (relu) y = (y > 0.0f) ? y : 0.0f;
            Y[(size_t)m * ldy + n] = y;
        }
    }
    return ORACLE_OK;
}
