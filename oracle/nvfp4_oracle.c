/*
 * nvfp4_oracle.c -- plain, slow, obviously-correct CPU oracle for the NVFP4
 * W4A4 linear layer.  TEST INFRASTRUCTURE ONLY: it is called by the test
 * suite, by the smoke check and by the benchmark's CPU-baseline leg, never by
 * the product path.  It shares no source with the CUDA library.
 *
 * What it follows:
 *  - NVFP4 elements are 4-bit E2M1 codes; every 16 consecutive codes share
 *    one E4M3 scale (thevalue.engineering, "NVFP4 W4A4 quantization
 *    compresses 27B hybrid models", section "Challenging the Recurrence
 *    Fragility Assumption").  The 16-element grouping is also on
 *    freegardner.com, "Quantizing All Layers Reveals Recurrent Memory Is
 *    Robust", section "Block Scaling and the Geography of Outliers", and on
 *    the kipquest.com paper page "Why Gated DeltaNet Survives 4-Bit
 *    Quantization", section "The deep dive".
 *  - W4A4: weights and activations both in NVFP4 (kipquest.com, "The
 *    abstract").
 *  - Each calibrated module carries its own FP32 global scale (kipquest.com,
 *    "The abstract" and "The deep dive").
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - global scale g = fl32(amax / 2688), 2688 = 6 * 448; g = 1 if amax == 0.
 *    g is a decode multiplier: x ~= code * scale * g.
 *  - block scale s = E4M3_RNE_satfinite( fl32( fl32(bamax / 6) / g ) ).
 *  - element code  = E2M1_RNE_satfinite( fl32( x / fl32(s * g) ) ), and the
 *    code is +-0 (sign of x) when s == 0.  Negative values that round to zero
 *    keep their sign (code 0x8).
 *  - packing: byte i of a row holds element 2i in the low nibble and element
 *    2i+1 in the high nibble.
 *  - scale-factor memory layout: 128-row x 4-block tiles of 512 bytes, see
 *    oracle_sf_offset().
 *  - the GEMM is the fp64 matmul of the dequantised operands.
 *
 * Rounding to E2M1 and E4M3 is done by enumerating every representable value
 * and taking the nearest one (ties to the even code); there is no bit trick.
 * All fp32 arithmetic uses plain float variables; build with
 * -ffp-contract=off so that no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---------------------------------------------------------------- decoding */

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.  Exponent 0
 * is subnormal: value = mantissa * 0.5. */
double oracle_e2m1_decode(int code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double v;
    if (e == 0)
        v = 0.5 * m;
    else
        v = (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
    return sign ? -v : v;
}

/* E4M3 (the "fn" variant: no infinities, only S.1111.111 is NaN): bit 7 sign,
 * bits 6..3 exponent (bias 7), bits 2..0 mantissa.  Exponent 0 is subnormal:
 * value = mantissa/8 * 2^-6. */
double oracle_e4m3_decode(int byte)
{
    int sign = (byte >> 7) & 1;
    int e = (byte >> 3) & 15;
    int m = byte & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = (m / 8.0) * ldexp(1.0, -6);
    else
        v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return sign ? -v : v;
}

/* ---------------------------------------------------------------- encoding */

/* Round-to-nearest over an enumerated, increasing list of non-negative
 * magnitudes; on an exact tie take the candidate whose code is even. */
static int nearest_even_code(double a, const double *vals, const int *codes, int n)
{
    int best = 0;
    double bestd = fabs(a - vals[0]);
    for (int i = 1; i < n; i++) {
        double d = fabs(a - vals[i]);
        if (d < bestd || (d == bestd && (codes[i] & 1) == 0 && (codes[best] & 1) == 1)) {
            best = i;
            bestd = d;
        }
    }
    return codes[best];
}

/* E2M1 round-to-nearest-even with saturation to +-6.  NaN is outside the
 * contract (never produced for finite inputs). */
int oracle_e2m1_encode(float y)
{
    double vals[8];
    int codes[8];
    for (int c = 0; c < 8; c++) {
        codes[c] = c;
        vals[c] = oracle_e2m1_decode(c);
    }
    double a = fabs((double)y);
    int mag;
    if (a >= 6.0)
        mag = 7;
    else
        mag = nearest_even_code(a, vals, codes, 8);
    return (signbit(y) ? 8 : 0) | mag;
}

/* E4M3 round-to-nearest-even with saturation to 448, for a non-negative
 * input (block scales are never negative).  Returns the byte. */
int oracle_e4m3_encode_nonneg(float v)
{
    static double vals[127];
    static int codes[127];
    static int init = 0;
    if (!init) {
        for (int c = 0; c < 127; c++) {
            codes[c] = c;
            vals[c] = oracle_e4m3_decode(c);
        }
        init = 1;
    }
    double a = (double)v;
    if (!(a > 0.0))
        return 0;
    if (a >= 448.0)
        return 0x7E;
    return nearest_even_code(a, vals, codes, 127);
}

/* ------------------------------------------------------------ bf16 helpers */

float oracle_bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a double to the nearest bfloat16 (ties to even), returning the bits.
 * Finite inputs only. */
uint16_t oracle_double_to_bf16(double x)
{
    if (x == 0.0)
        return signbit(x) ? 0x8000 : 0x0000;
    int e;
    frexp(fabs(x), &e);               /* |x| in [2^(e-1), 2^e) */
    int ulp_exp = (e - 1) - 7;        /* 8 significant bits */
    if (ulp_exp < -133)
        ulp_exp = -133;               /* bf16 subnormal spacing */
    double q = ldexp(x, -ulp_exp);
    double r = nearbyint(q);          /* default mode: round half to even */
    double v = ldexp(r, ulp_exp);
    float f = (float)v;               /* exact: v has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------- global scale (g) */

/* max |x| over rows [r0, r1) of a row-major bf16 matrix with leading dim ld. */
float oracle_rows_amax(const uint16_t *x, int64_t r0, int64_t r1, int64_t K, int64_t ld)
{
    float m = 0.0f;
    for (int64_t r = r0; r < r1; r++)
        for (int64_t k = 0; k < K; k++) {
            float v = fabsf(oracle_bf16_to_float(x[r * ld + k]));
            if (v > m)
                m = v;
        }
    return m;
}

float oracle_global_scale(float amax)
{
    if (amax == 0.0f)
        return 1.0f;
    float g = amax / 2688.0f;
    return g;
}

/* ------------------------------------------------------ block quantization */

/* Quantize rows [0, rows) of x (bf16 bits, leading dim ld, K % 16 == 0)
 * with global scale g[r] for row r.  Writes packed codes [rows, K/2] and
 * logical (row-major, unswizzled) scale bytes [rows, K/16]. */
void oracle_quantize_rows(const uint16_t *x, int64_t rows, int64_t K, int64_t ld,
                          const float *g_row, uint8_t *codes, uint8_t *scales)
{
    int64_t nb = K / 16;
    for (int64_t r = 0; r < rows; r++) {
        float g = g_row[r];
        for (int64_t b = 0; b < nb; b++) {
            const uint16_t *blk = x + r * ld + b * 16;
            float bamax = 0.0f;
            for (int i = 0; i < 16; i++) {
                float v = fabsf(oracle_bf16_to_float(blk[i]));
                if (v > bamax)
                    bamax = v;
            }
            float t = bamax / 6.0f;
            float s32 = t / g;
            int sbyte = oracle_e4m3_encode_nonneg(s32);
            scales[r * nb + b] = (uint8_t)sbyte;
            float s = (float)oracle_e4m3_decode(sbyte);
            float d = s * g;
            for (int i = 0; i < 16; i += 2) {
                int c[2];
                for (int j = 0; j < 2; j++) {
                    float xv = oracle_bf16_to_float(blk[i + j]);
                    if (d == 0.0f) {
                        c[j] = signbit(xv) ? 8 : 0;
                    } else {
                        float y = xv / d;
                        c[j] = oracle_e2m1_encode(y);
                    }
                }
                codes[r * (K / 2) + b * 8 + i / 2] = (uint8_t)(c[0] | (c[1] << 4));
            }
        }
    }
}

/* Dequantize rows: out[r, k] = e2m1(code) * e4m3(scale) * g[r], in fp64. */
void oracle_dequant_rows(const uint8_t *codes, const uint8_t *scales, int64_t rows,
                         int64_t K, const float *g_row, double *out)
{
    int64_t nb = K / 16;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < K; k++) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            int c = (k & 1) ? (byte >> 4) : (byte & 15);
            double s = oracle_e4m3_decode(scales[r * nb + k / 16]);
            out[r * K + k] = oracle_e2m1_decode(c) * s * (double)g_row[r];
        }
}

/* -------------------------------------------------- scale-factor layout */

/* Swizzled scale-factor layout consumed by the block-scaled tensor-core MMA:
 * the logical [rows, K/16] scale matrix is padded to a multiple of 128 rows
 * and 4 block-columns and cut into 128 x 4 tiles of 512 bytes.  Tiles are
 * stored K-tile-fastest: tile (rt, ct) starts at (rt * CT + ct) * 512, CT =
 * ceil(K/64).  Inside a tile, row r and block column c sit at
 * (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4). */
int64_t oracle_sf_offset(int64_t r, int64_t c, int64_t K)
{
    int64_t ct_count = (K / 16 + 3) / 4;
    int64_t rt = r / 128, ct = c / 4;
    int64_t tile = rt * ct_count + ct;
    int64_t rr = r % 128;
    return tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (c % 4);
}

int64_t oracle_sf_bytes(int64_t rows, int64_t K)
{
    int64_t rpad = (rows + 127) / 128 * 128;
    int64_t cpad = (K / 16 + 3) / 4 * 4;
    return rpad * cpad;
}

/* logical [rows, K/16] -> swizzled buffer of oracle_sf_bytes(rows, K) bytes
 * (padding bytes are zero). */
void oracle_swizzle_scales(const uint8_t *logical, int64_t rows, int64_t K, uint8_t *out)
{
    int64_t nb = K / 16;
    memset(out, 0, (size_t)oracle_sf_bytes(rows, K));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < nb; c++)
            out[oracle_sf_offset(r, c, K)] = logical[r * nb + c];
}

void oracle_unswizzle_scales(const uint8_t *swz, int64_t rows, int64_t K, uint8_t *logical)
{
    int64_t nb = K / 16;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < nb; c++)
            logical[r * nb + c] = swz[oracle_sf_offset(r, c, K)];
}

/* ------------------------------------------------------------------- GEMM */

/* For each requested output (m, n):
 *   C[i] = sum_k  A^[m,k] * W^[n,k]      (fp64, k ascending)
 *   B[i] = sum_k |A^[m,k] * W^[n,k]|
 * with A^ = e2m1(a) * e4m3(sa) * g_a and W^ = e2m1(w) * e4m3(sw) * g_w[n].
 * Codes are packed [rows, K/2]; scales are logical [rows, K/16]. */
void oracle_linear_sampled(const uint8_t *a_codes, const uint8_t *a_scales, float g_a,
                           const uint8_t *w_codes, const uint8_t *w_scales, const float *g_w_row,
                           int64_t K, const int64_t *ms, const int64_t *ns, int64_t count,
                           double *C, double *B)
{
    int64_t nb = K / 16;
    for (int64_t i = 0; i < count; i++) {
        int64_t m = ms[i], n = ns[i];
        double acc = 0.0, bound = 0.0;
        for (int64_t k = 0; k < K; k++) {
            uint8_t ab = a_codes[m * (K / 2) + k / 2];
            uint8_t wb = w_codes[n * (K / 2) + k / 2];
            int ac = (k & 1) ? (ab >> 4) : (ab & 15);
            int wc = (k & 1) ? (wb >> 4) : (wb & 15);
            double a = oracle_e2m1_decode(ac) * oracle_e4m3_decode(a_scales[m * nb + k / 16]) * (double)g_a;
            double w = oracle_e2m1_decode(wc) * oracle_e4m3_decode(w_scales[n * nb + k / 16]) * (double)g_w_row[n];
            acc += a * w;
            bound += fabs(a * w);
        }
        C[i] = acc;
        B[i] = bound;
    }
}

/* -------------------------------------------------------- MLP intermediate */

/* h = bf16( silu(gate) * up ), silu(v) = v / (1 + exp(-v)), evaluated in
 * fp64 from the bf16 inputs.  gate_up is [rows, 2F] (gate = first F columns,
 * up = last F columns); h is [rows, F]. */
void oracle_swiglu(const uint16_t *gate_up, int64_t rows, int64_t F, int64_t ld, uint16_t *h)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t j = 0; j < F; j++) {
            double gv = oracle_bf16_to_float(gate_up[r * ld + j]);
            double uv = oracle_bf16_to_float(gate_up[r * ld + F + j]);
            double s = gv / (1.0 + exp(-gv));
            h[r * F + j] = oracle_double_to_bf16(s * uv);
        }
}

/* --------------------------------------------- FP8 KV-cache quantization */
/*
 * The attention KV cache in FP8 with a calibrated per-tensor scale.  The pages
 * recommend shipping calibrated cache scales and report that, calibrated,
 * they cost no accuracy (freegardner.com, "Quantizing All Layers Reveals Recurrent Memory Is
 * Robust", section "The Calibrated Cache That Ships for Free";
 * thevalue.engineering, "NVFP4 W4A4 quantization compresses 27B hybrid
 * models", section "Efficiency Gains and Serving Optimization"; the
 * kipquest.com abstract).  The pages give no formula.  Readings: one FP32
 * decode scale s per cache tensor (x ~= e4m3(code) * s), calibrated as
 * s = fl32(amax / 448) (1 if amax == 0, as for the NVFP4 global scale), and
 * code = E4M3_RNE_satfinite(fl32(x / s)) with the sign bit copying the sign
 * of x, so negative values that round to zero give 0x80.
 */

/* Signed E4M3: the magnitude by enumeration (oracle_e4m3_encode_nonneg),
 * the sign bit from the input. */
int oracle_e4m3_encode(float y)
{
    int m = oracle_e4m3_encode_nonneg(fabsf(y));
    return signbit(y) ? (m | 0x80) : m;
}

float oracle_fp8_kv_scale(float amax)
{
    if (amax == 0.0f)
        return 1.0f;
    float s = amax / 448.0f;
    return s;
}

/* out[r, c] = E4M3(fl32(x[r, c] / s)) for a row-major bf16 matrix (leading
 * dimension ld) into a byte matrix with leading dimension ldo. */
void oracle_fp8_kv_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, float s, uint8_t *out,
                            int64_t ldo)
{
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) {
            float y = oracle_bf16_to_float(x[r * ld + c]) / s;
            out[r * ldo + c] = (uint8_t)oracle_e4m3_encode(y);
        }
}
