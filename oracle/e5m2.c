/*
 * E5M2 (FP8) codec for the ARKV oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * The ARKV page stores mid-importance tokens in "low precision, e.g. FP8"
 * ("ARKV: Adaptive and Resource-Efficient KV Cache Management ...", 기술요약 §2.다,
 * Quantization tier).  E4M3 is the default; E5M2, the other FP8 format, is the
 * second choice offered for that tier.  This file writes the format out from its
 * public definition (OCP 8-bit Floating Point Specification, E5M2):
 *   1 sign bit, 5 exponent bits (bias 15), 2 mantissa bits;
 *   exponent field 0 -> subnormal, value = m * 2^-16;
 *   exponent field 1..30 -> normal, value = (1 + m/4) * 2^(e-15);
 *   exponent field 31 -> infinity (m = 0) or NaN (m != 0); the largest finite
 *   value is 57344.
 * Encoding rounds to nearest, ties to even, and saturates to +-57344 (the
 * "satfinite" convention, infinities included), keeping the sign of zero.  NaN
 * encodes to S.11111.11.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may load
 * this library.  Built with -ffp-contract=off; every double operation below is
 * exact (power-of-two scalings of values with at most 24 significant bits).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static uint8_t encode_one(float x)
{
    uint32_t bits;
    memcpy(&bits, &x, sizeof bits);
    const uint8_t sign = (uint8_t)((bits >> 31) << 7);
    if (isnan(x))
        return (uint8_t)(sign | 0x7F);
    const double a = fabs((double)x);
    if (a >= 57344.0)                     /* saturate (infinities too) */
        return (uint8_t)(sign | 0x7B);
    if (a == 0.0)
        return sign;

    /* spacing of E5M2 values around a: 2^(max(floor(log2 a), -14) - 2) */
    int e2;
    frexp(a, &e2);                        /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                       /* floor(log2 a) */
    if (E < -14)
        E = -14;                          /* subnormal range shares the 2^-16 spacing */
    const double ulp = ldexp(1.0, E - 2);
    const double q = a / ulp;             /* exact */
    double k = floor(q);
    const double rem = q - k;
    if (rem > 0.5 || (rem == 0.5 && fmod(k, 2.0) == 1.0))
        k += 1.0;                         /* round to nearest, ties to even */
    const double val = k * ulp;           /* <= 57344 because a < 57344 */
    if (val == 0.0)
        return sign;

    frexp(val, &e2);
    E = e2 - 1;
    if (E < -14)                          /* subnormal: val = m * 2^-16, m in 1..3 */
        return (uint8_t)(sign | (uint8_t)ldexp(val, 16));
    const int mant = (int)(ldexp(val, -E) * 4.0) - 4;   /* 0..3 */
    return (uint8_t)(sign | ((E + 15) << 2) | mant);
}

static double decode_one(uint8_t c)
{
    const int e = (c >> 2) & 0x1F, m = c & 3;
    const double s = (c & 0x80) ? -1.0 : 1.0;
    if (e == 31)
        return m == 0 ? s * INFINITY : NAN;
    if (e == 0)
        return s * ldexp((double)m, -16);
    return s * ldexp(1.0 + m / 4.0, e - 15);
}

void arkv_oracle_e5m2_encode(const float *x, uint8_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = encode_one(x[i]);
}

void arkv_oracle_e5m2_decode(const uint8_t *c, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = decode_one(c[i]);
}

/* Encode the float32 values whose bit patterns are start, start+1, ...,
 * start+n-1 (exhaustive sweeps over the float32 space). */
void arkv_oracle_e5m2_encode_bits_range(uint32_t start, int64_t n, uint8_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const uint32_t b = start + (uint32_t)i;
        float x;
        memcpy(&x, &b, sizeof x);
        out[i] = encode_one(x);
    }
}
