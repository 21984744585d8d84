/*
 * mq_oracle.c -- plain, slow CPU reference of the NVFP4 prefill linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark load it.  The product library never links, loads or
 * calls it, and it shares no code, table or constant generator with the CUDA
 * sources.
 *
 * Source of the method: "Mix-Quant: Quantized Prefilling, Precise Decoding
 * for Agentic LLMs", section 3.3 ("NVFP4 Microscaling Quantization for
 * Prefilling"), Eq. 2 (element quantization and dequantization) and Eq. 3
 * (amax block scale), and the surrounding format description: E2M1 element
 * values, groups of g = 16 consecutive elements sharing an FP8-E4M3 block
 * scale, one tensor-level scale, round-to-nearest with clipping, layouts
 * aligned with the GEMM (K) dimension.  The prefill path is W4A4 and the
 * decode path stays BF16 (same section, "Prefill-Decode Disaggregation
 * Deployment").
 *
 * Readings where the paper leaves a step open (each one is also listed in
 * the design notes of the repository):
 *   - q_max = 6, the largest finite E2M1 magnitude (Eq. 3 text).
 *   - Tensor scale alpha = amax(|x|) / (6 * 448) in FP32; alpha = 1 for an
 *     all-zero tensor.  The paper only says the tensor scale prevents global
 *     saturation; this choice puts the largest block scale exactly at the
 *     E4M3 maximum 448.
 *   - Pi_E4M3: round to nearest, ties to even mantissa, values above 448
 *     clip to 448 (satfinite), subnormals kept.
 *   - Pi_FP4: round to nearest, ties to even mantissa, magnitudes above 6
 *     clip to 6 ("with clipping"); the sign bit of x is kept, so a negative
 *     value that rounds to zero gives the code 0x8.
 *   - Eq. 2's quotient x / (alpha * sigma) is evaluated in FP32 as
 *     |x| * fl(1 / fl(alpha * sigma)); a block with alpha * sigma == 0 gets
 *     all-zero magnitudes.  Eq. 3's quotient is fl(amax_b / fl(alpha * 6)).
 *   - Packing: element k of a row goes to byte k/2, even k in the low nibble.
 *   - Scale optimization (mentioned once, never defined): an opt-in search
 *     per block over the Eq. 3 scale code and its two E4M3 neighbours,
 *     keeping the one with the smallest binary32 squared error (ties keep
 *     the Eq. 3 scale); off by default.
 *
 * Floating point: IEEE binary32 / binary64 with no contraction (compile with
 * -ffp-contract=off) and no fast-math.  Dequantization and every matmul are
 * in binary64.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* The eight non-negative E2M1 magnitudes, in code order 0..7.  E2M1 has one
 * sign bit, two exponent bits (bias 1) and one mantissa bit; exponent 0 is
 * subnormal (0 and 0.5).  Codes 8..15 are the negatives. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(unsigned code)
{
    double m = E2M1_MAG[code & 7u];
    return (code & 8u) ? -m : m;
}

/* E4M3 (the "FN" variant used by NVFP4 block scales): sign, 4 exponent bits
 * with bias 7, 3 mantissa bits; exponent field 0 is subnormal
 * (m/8 * 2^-6); S.1111.111 is NaN and there are no infinities. */
double orc_e4m3_value(unsigned code)
{
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    double v;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -v : v;
}

/* Values of all 256 E4M3 codes, filled once when the library loads. */
static double E4M3_VAL[256];

__attribute__((constructor)) static void orc_init_tables(void)
{
    for (unsigned c = 0; c < 256u; ++c) E4M3_VAL[c] = orc_e4m3_value(c);
}

/* Pi_E4M3 for a non-negative scale s: the nearest of the 127 finite
 * non-negative E4M3 values (codes 0x00..0x7E), found by exhaustive search;
 * on a tie the code with an even mantissa wins; values above 448 give 448. */
unsigned orc_e4m3_round(float s)
{
    const double x = (double)s;
    unsigned best = 0;
    double best_d = INFINITY;
    if (!(x >= 0.0)) return 0u;          /* negative or NaN: out of contract */
    if (x >= 448.0) return 0x7Eu;        /* satfinite */
    for (unsigned c = 0; c <= 0x7Eu; ++c) {
        double d = fabs(E4M3_VAL[c] - x);   /* exact in binary64 */
        if (d < best_d || (d == best_d && (c & 1u) == 0u)) {
            best_d = d;
            best = c;
        }
    }
    return best;
}

/* Pi_FP4 magnitude for m >= 0: index 0..7 of the nearest E2M1 magnitude by
 * exhaustive search, ties to the even index (even mantissa), clipped at 6. */
unsigned orc_e2m1_round(float m)
{
    const double x = (double)m;
    unsigned best = 0;
    double best_d = INFINITY;
    if (!(x >= 0.0)) return 0u;
    if (x >= 6.0) return 7u;             /* clipping */
    for (unsigned i = 0; i < 8u; ++i) {
        double d = fabs(E2M1_MAG[i] - x);
        if (d < best_d || (d == best_d && (i & 1u) == 0u)) {
            best_d = d;
            best = i;
        }
    }
    return best;
}

float orc_bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary64 value to the nearest bfloat16 (8 exponent bits, 7
 * mantissa bits), ties to even.  Done on the binary64 value directly so
 * there is no double rounding through binary32. */
uint16_t orc_double_to_bf16(double v)
{
    if (isnan(v)) return (uint16_t)0x7FC0u;
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    uint16_t sign = (uint16_t)(neg ? 0x8000u : 0u);
    if (a == 0.0) return sign;
    /* Largest finite bf16 is (2 - 2^-7) * 2^127; the rounding boundary to
     * infinity is (2 - 2^-8) * 2^127. */
    if (a >= ldexp(2.0 - ldexp(1.0, -8), 127)) return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(a, &e);                        /* a = f * 2^e, f in [0.5, 1) */
    int exp_unb = e - 1;                 /* a in [2^exp_unb, 2^(exp_unb+1)) */
    if (exp_unb < -126) exp_unb = -126;  /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, exp_unb - 7);
    double q = a / quantum;              /* exact: power-of-two division */
    double fl = floor(q);
    double r = q - fl;
    double n = fl;
    if (r > 0.5 || (r == 0.5 && fmod(fl, 2.0) != 0.0)) n = fl + 1.0;
    double rounded = n * quantum;        /* exact */
    float f = (float)rounded;            /* exact: rounded has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFFu));
}

/* ------------------------------------------------------------------------ */
/* Tensor scale                                                             */
/* ------------------------------------------------------------------------ */

/* amax over a BF16 tensor and the tensor-level scale alpha derived from it.
 * Returns 1 (and still fills *amax_out / *alpha_out from the finite values)
 * if any element is NaN or infinite, else 0. */
int orc_tensor_alpha(const uint16_t* x, int64_t n, float* amax_out, float* alpha_out)
{
    float amax = 0.0f;
    int nonfinite = 0;
    for (int64_t i = 0; i < n; ++i) {
        float v = fabsf(orc_bf16_to_float(x[i]));
        if (!isfinite(v)) { nonfinite = 1; continue; }
        if (v > amax) amax = v;
    }
    const float qmax_times_e4m3max = 6.0f * 448.0f;   /* 2688, exact */
    float alpha = (amax == 0.0f) ? 1.0f : amax / qmax_times_e4m3max;
    if (amax_out) *amax_out = amax;
    if (alpha_out) *alpha_out = alpha;
    return nonfinite;
}

/* ------------------------------------------------------------------------ */
/* Quantization (Eq. 2 and Eq. 3)                                           */
/* ------------------------------------------------------------------------ */

/* Quantize one block of 16 BF16 values with tensor scale alpha.
 * Writes 16 four-bit codes (one per byte, not packed) and returns the E4M3
 * code of the block scale sigma_b. */
static unsigned quantize_block(const uint16_t* xb, float alpha, unsigned char codes16[16])
{
    float amax_b = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float v = fabsf(orc_bf16_to_float(xb[i]));
        if (v > amax_b) amax_b = v;
    }
    /* Eq. 3: sigma_b = Pi_E4M3( amax_b / (alpha * q_max) ) */
    float alpha_qmax = alpha * 6.0f;
    float s = amax_b / alpha_qmax;
    unsigned sigma_code = orc_e4m3_round(s);
    float sigma = (float)orc_e4m3_value(sigma_code);   /* exact in binary32 */
    /* Eq. 2: q_i = Pi_FP4( x_i / (alpha * sigma_b) ) */
    float d = alpha * sigma;
    float enc = (d == 0.0f) ? 0.0f : 1.0f / d;
    for (int i = 0; i < 16; ++i) {
        float v = orc_bf16_to_float(xb[i]);
        unsigned sign = signbit(v) ? 8u : 0u;
        float a = fabsf(v);
        unsigned mag = (a == 0.0f) ? 0u : orc_e2m1_round(a * enc);
        codes16[i] = (unsigned char)(sign | mag);
    }
    return sigma_code;
}

/* ------------------------------------------------------------------------ */
/* Optional scale search (the paper's "scale optimization", read as a       */
/* per-block choice among the E4M3 neighbours of the Eq. 3 scale)          */
/* ------------------------------------------------------------------------ */

/* Eq. 2 codes of one block for a given block-scale code. */
static void encode_block(const uint16_t* xb, float alpha, unsigned sigma_code, unsigned char codes16[16])
{
    float d = alpha * (float)orc_e4m3_value(sigma_code);
    float enc = (d == 0.0f) ? 0.0f : 1.0f / d;
    for (int i = 0; i < 16; ++i) {
        float v = orc_bf16_to_float(xb[i]);
        unsigned sign = signbit(v) ? 8u : 0u;
        float a = fabsf(v);
        unsigned mag = (a == 0.0f) ? 0u : orc_e2m1_round(a * enc);
        codes16[i] = (unsigned char)(sign | mag);
    }
}

/* Squared error of a coded block, in binary32 and in element order:
 * y_i = fl(d * v_i) with d = fl(alpha * sigma) and v_i the signed E2M1
 * value; r_i = fl(x_i - y_i); e = fl(e + fl(r_i * r_i)). */
static float block_sq_error(const uint16_t* xb, float alpha, unsigned sigma_code, const unsigned char codes16[16])
{
    float d = alpha * (float)orc_e4m3_value(sigma_code);
    float e = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float v = (float)orc_e2m1_value(codes16[i]);
        float y = d * v;
        float r = orc_bf16_to_float(xb[i]) - y;
        float rr = r * r;
        e = e + rr;
    }
    return e;
}

/* Block quantization with scale search: candidates are the Eq. 3 code c0
 * and its E4M3 neighbours c0 - 1 and c0 + 1 (within 0 .. 0x7E), tried in the
 * order c0, c0 - 1, c0 + 1; the first candidate with the smallest squared
 * error (block_sq_error) wins, so ties keep the Eq. 3 scale. */
static unsigned quantize_block_search(const uint16_t* xb, float alpha, unsigned char codes16[16])
{
    unsigned c0 = quantize_block(xb, alpha, codes16);
    float best = block_sq_error(xb, alpha, c0, codes16);
    unsigned best_c = c0;
    unsigned cand[2] = {c0 - 1u, c0 + 1u};
    int valid[2] = {c0 >= 1u, c0 <= 0x7Du};
    for (int j = 0; j < 2; ++j) {
        if (!valid[j]) continue;
        unsigned char q[16];
        encode_block(xb, alpha, cand[j], q);
        float e = block_sq_error(xb, alpha, cand[j], q);
        if (e < best) {
            best = e;
            best_c = cand[j];
            memcpy(codes16, q, 16);
        }
    }
    return best_c;
}

/* Quantize rows x[rows][K] (BF16, row-major; K a multiple of 16).
 * codes: [rows][K/2] bytes, element k in byte k/2, even k in the low nibble.
 * scales: [rows][K/16] E4M3 codes, row-major (the plain layout). */
void orc_quantize_rows(const uint16_t* x, int64_t rows, int64_t K, float alpha,
                       uint8_t* codes, uint8_t* scales)
{
    const int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            unsigned char q[16];
            unsigned sc = quantize_block(x + r * K + b * 16, alpha, q);
            scales[r * nb + b] = (uint8_t)sc;
            for (int i = 0; i < 16; i += 2)
                codes[r * (K / 2) + b * 8 + i / 2] = (uint8_t)(q[i] | (q[i + 1] << 4));
        }
    }
}

/* As orc_quantize_rows, with the per-block scale search. */
void orc_quantize_rows_search(const uint16_t* x, int64_t rows, int64_t K, float alpha,
                              uint8_t* codes, uint8_t* scales)
{
    const int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            unsigned char q[16];
            unsigned sc = quantize_block_search(x + r * K + b * 16, alpha, q);
            scales[r * nb + b] = (uint8_t)sc;
            for (int i = 0; i < 16; i += 2)
                codes[r * (K / 2) + b * 8 + i / 2] = (uint8_t)(q[i] | (q[i + 1] << 4));
        }
    }
}

/* ------------------------------------------------------------------------ */
/* RMSNorm producing the tensor that the prefill linear quantizes           */
/* ------------------------------------------------------------------------ */

/* h[r][k] = bf16( fl32( fl32(x[r][k] * rstd_r) * gamma[k] ) ) with
 *   ms_r   = fl32( (sum_k x^2, in binary64, k ascending) / K ),
 *   rstd_r = fl32( 1 / sqrt( (double)ms_r + (double)eps ) )  (binary64, one rounding).
 * x, gamma, h: BF16 bit patterns; rstd (optional): the per-row FP32 factors. */
void orc_rmsnorm_rows(const uint16_t* x, int64_t rows, int64_t K, const uint16_t* gamma, float eps,
                      uint16_t* h, float* rstd)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + r * K;
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double v = (double)orc_bf16_to_float(xr[k]);
            ss += v * v;
        }
        float ms = (float)(ss / (double)K);
        float rs = (float)(1.0 / sqrt((double)ms + (double)eps));
        if (rstd) rstd[r] = rs;
        for (int64_t k = 0; k < K; ++k) {
            float t = orc_bf16_to_float(xr[k]) * rs;
            float u = t * orc_bf16_to_float(gamma[k]);
            h[r * K + k] = orc_double_to_bf16((double)u);
        }
    }
}

/* Dequantize (Eq. 2 right-hand side): xhat = alpha * sigma_b * q_i, in
 * binary64.  With alpha = 1 this gives sigma_b * q_i, the operand the
 * block-scaled matmul multiplies before the tensor scales are applied. */
void orc_dequantize_rows(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                         int64_t K, float alpha, double* out)
{
    double e2m1[16];
    const double* e4m3 = E4M3_VAL;
    for (unsigned c = 0; c < 16u; ++c) e2m1[c] = orc_e2m1_value(c);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[r * (K / 2) + k / 2];
            unsigned code = (k & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 15u);
            double sigma = e4m3[scales[r * (K / 16) + k / 16]];
            out[r * K + k] = (double)alpha * sigma * e2m1[code];
        }
    }
}

/* Round binary64 values to bfloat16 (RNE). */
void orc_round_bf16(const double* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_double_to_bf16(v[i]);
}

/* Gated MLP activation between the gate/up and down projections:
 *   h = bf16( fl32( silu(g) ) * u ),  g = fl32(gate), u = fl32(up),
 *   silu(g) = g / (1 + exp(-g)).
 * The intermediate is rounded to BF16 before it is requantized, as an
 * unfused BF16 pipeline would store it. */
void orc_silu_mul(const double* gate, const double* up, int64_t n, uint16_t* h)
{
    for (int64_t i = 0; i < n; ++i) {
        float g = (float)gate[i];
        float u = (float)up[i];
        float sg = (float)((double)g / (1.0 + exp(-(double)g)));
        float p = sg * u;
        h[i] = orc_double_to_bf16((double)p);
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
