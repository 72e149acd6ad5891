/*
 * Weight quantizers and dequantizers. TEST INFRASTRUCTURE (see oracle.h).
 *
 * The pages name the two load-time quantizers of the draft head -- a BF16 -> FP8
 * weight quantizer and a two-pass BF16 -> NVFP4 quantizer (a global |w| max pass,
 * then the block encode) -- in [new.rs] (the kernel lookups at the top of
 * MtpHead::new) and [mtp_head.rs] (quantize_proj), but not their arithmetic.
 * The readings below are stated as fp32 operations, each rounded to nearest even,
 * because the quantized codes are integers that both sides must decide alike:
 *
 * FP8 per-row (fp32 row scale = absmax/448):
 *   a = max_k |W[n,k]|;  s = a / 448.0f;  q = e4m3(W[n,k] / s);  a == 0 -> s = 0, q = 0.
 * NVFP4 (E2M1 codes, one E4M3 scale per 16 consecutive k, one fp32 global scale):
 *   A = max |W|;  g = A / 2688.0f (2688 = 6 * 448), g = 1 when A == 0;
 *   per block: B = max |W_b|;  sb = e4m3((B / 6.0f) / g);  S = e4m3val(sb) * g;
 *   q_i = e2m1(W_i / S), or 0 when S == 0.  Dequant: e2m1val(q) * e4m3val(sb) * g.
 *   Codes pack two per byte, element 2j in the low nibble of byte j.
 *
 * Pins (tests/test_oracle.py): per-element round-trip bounds, the absmax element
 * mapping to +-448, a hand-worked NVFP4 block (tests/golden/nvfp4_block.txt), and an
 * independent torch implementation built on torch's own float8 cast.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#include "oracle.h"

static float bf16_to_f32(uint16_t b) { return (float)orc_bf16_to_f64(b); }

void orc_quantize_fp8_rows(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                           float* row_scale) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        const uint16_t* row = w + r * k;
        float a = 0.0f;
        for (int64_t j = 0; j < k; ++j) {
            float v = fabsf(bf16_to_f32(row[j]));
            if (v > a) a = v;
        }
        float s = a / 448.0f;
        row_scale[r] = s;
        for (int64_t j = 0; j < k; ++j) {
            if (a == 0.0f) {
                codes[r * k + j] = 0x00;
            } else {
                float q = bf16_to_f32(row[j]) / s;
                codes[r * k + j] = orc_e4m3_encode((double)q);
            }
        }
    }
}

void orc_quantize_nvfp4(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                        uint8_t* block_scale, float* global_scale) {
    /* pass 1: global |w| max (exact in fp32) */
    float A = 0.0f;
    for (int64_t i = 0; i < n * k; ++i) {
        float v = fabsf(bf16_to_f32(w[i]));
        if (v > A) A = v;
    }
    float g = (A == 0.0f) ? 1.0f : A / 2688.0f;
    *global_scale = g;
    const int64_t nb = k / 16;
    /* pass 2: per-16 block scale, then the E2M1 codes */
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const uint16_t* blk = w + r * k + b * 16;
            float B = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float v = fabsf(bf16_to_f32(blk[i]));
                if (v > B) B = v;
            }
            float t = B / 6.0f;
            float u = t / g;
            uint8_t sb = orc_e4m3_encode((double)u);
            block_scale[r * nb + b] = sb;
            float S = (float)orc_e4m3_value(sb) * g;
            for (int i = 0; i < 16; i += 2) {
                uint8_t lo = 0, hi = 0;
                if (S != 0.0f) {
                    float q0 = bf16_to_f32(blk[i]) / S;
                    float q1 = bf16_to_f32(blk[i + 1]) / S;
                    lo = orc_e2m1_encode((double)q0);
                    hi = orc_e2m1_encode((double)q1);
                }
                codes[r * (k / 2) + (b * 16 + i) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

/* Dequantized row `row` of a [*, k] table in fp64. fmt: 0 bf16, 1 fp8 per-row,
 * 2 nvfp4 ([mtp_head.rs] ProjectionWeight variants Bf16, Fp8, Nvfp4). */
void orc_dequant_row(int32_t fmt, const void* data, const float* row_scale,
                     const uint8_t* block_scale, float global_scale, int64_t k,
                     int64_t row, double* out) {
    if (fmt == 0) {
        const uint16_t* p = (const uint16_t*)data + row * k;
        for (int64_t j = 0; j < k; ++j) out[j] = orc_bf16_to_f64(p[j]);
    } else if (fmt == 1) {
        const uint8_t* p = (const uint8_t*)data + row * k;
        double s = (double)row_scale[row];
        for (int64_t j = 0; j < k; ++j) out[j] = orc_e4m3_value(p[j]) * s;
    } else {
        const uint8_t* p = (const uint8_t*)data + row * (k / 2);
        const uint8_t* sc = block_scale + row * (k / 16);
        double g = (double)global_scale;
        for (int64_t j = 0; j < k; ++j) {
            uint8_t byte = p[j / 2];
            uint8_t code = (j & 1) ? (byte >> 4) : (byte & 0xF);
            out[j] = orc_e2m1_value(code) * orc_e4m3_value(sc[j / 16]) * g;
        }
    }
}
