/*
 * Number formats, written out from their public definitions. TEST INFRASTRUCTURE:
 * only tests/, the smoke check and the benchmark's CPU baseline use the oracle.
 *
 * bf16  : the upper 16 bits of an IEEE binary32 ([v4_mtp.rs], argmax_grammar_masked,
 *         which widens a bf16 logit by shifting it into the top half of an f32).
 *         Narrowing rounds to nearest, ties to even.
 * E4M3  : OCP 8-bit float E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits,
 *         no infinities, S.1111.111 is NaN, largest finite 448, subnormal step 2^-9.
 *         The pages never define the encoder; the reading used is round to nearest,
 *         ties to even mantissa, saturating to +-448 ("satfinite"), sign kept.
 * E2M1  : OCP FP4: 1 sign, 2 exponent (bias 1), 1 mantissa bit; magnitudes
 *         {0, .5, 1, 1.5, 2, 3, 4, 6}. Same rounding reading, saturating to +-6.
 *
 * Pins (tests/test_oracle.py): every encoder is checked against a linear search
 * over all codes on every bf16 bit pattern and on every midpoint +-1 ulp, and the
 * E4M3 decode/encode against torch.float8_e4m3fn.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "oracle.h"

double orc_bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Nearest bf16 to the real value x (single rounding, ties to even). */
uint16_t orc_f64_to_bf16(double x) {
    if (isnan(x)) return 0x7FC0;
    double a = fabs(x);
    double v;
    if (a == 0.0) {
        v = 0.0;
    } else {
        int ex;
        frexp(a, &ex);           /* a = f * 2^ex, f in [0.5, 1) */
        int e = ex - 1;          /* a in [2^e, 2^(e+1)) */
        if (e < -126) e = -126;  /* subnormal range: fixed quantum */
        double quantum = ldexp(1.0, e - 7);
        v = rint(a / quantum) * quantum; /* rint: current mode = nearest-even */
    }
    float f = (float)v; /* exact: v is a bf16 value (or overflows to inf) */
    if (signbit(x)) f = -f;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

void orc_f64_to_bf16_vec(const double* v, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f64_to_bf16(v[i]);
}

double orc_e4m3_value(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

uint8_t orc_e4m3_encode(double v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormals: integer multiples of 2^-9; q == 8 is the smallest normal */
        double q = rint(a / ldexp(1.0, -9));
        return sign | (uint8_t)q;
    }
    int ex;
    frexp(a, &ex);
    int e = ex - 1;                           /* a in [2^e, 2^(e+1)), e in [-6, 8] */
    double q = rint(a / ldexp(1.0, e - 3));   /* in [8, 16]; spacing 2^(e-3) */
    if (q == 16.0) {
        e += 1;
        q = 8.0;
    }
    return sign | (uint8_t)(((e + 7) << 3) | ((int)q - 8));
}

void orc_e4m3_encode_vec(const double* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

double orc_e2m1_value(uint8_t code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

uint8_t orc_e2m1_encode(double v) {
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs(v);
    if (isnan(v)) return 0x7;
    if (a >= 6.0) return sign | 0x7;
    if (a < 1.0) {
        double q = rint(a / 0.5); /* 0, 1 or 2 (2 is the code of 1.0) */
        return sign | (uint8_t)q;
    }
    int ex;
    frexp(a, &ex);
    int e = ex - 1;                          /* 0, 1 or 2 */
    double q = rint(a / ldexp(1.0, e - 1));  /* in [2, 4] */
    if (q == 4.0) {
        e += 1;
        q = 2.0;
    }
    return sign | (uint8_t)(((e + 1) << 1) | ((int)q - 2));
}

void orc_e2m1_encode_vec(const double* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}
