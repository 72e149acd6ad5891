/*
 * Drafter-context prefill, row by row. TEST INFRASTRUCTURE (see oracle.h).
 *
 * [mtp_head.rs] (the drafter-prefill docs and MtpPrefillScratch) states that the
 * drafter's K/V for prompt row i depend only on the pair (embed(token_{i+1}),
 * target_hidden_i), so the prefill is: the combiner, the fc projection, the k/v
 * projections, RoPE on K, and the KV-cache write -- no attention. Every buffer in
 * that scratch is bf16, so each stage's output is rounded to bf16 here:
 *   y   = bf16(fc . [bf16(rms(e) w_e) || bf16(rms(x) w_h)])
 *   k   = bf16(Wk . y),  v = bf16(Wv . y)        (nkv heads of hd each)
 *   k'  = bf16(RoPE(k, pos))        NeoX half rotation over the whole head:
 *         theta_j = pos * base^(-2j/hd), j < hd/2,
 *         k'_j = k_j cos - k_{j+hd/2} sin,  k'_{j+hd/2} = k_{j+hd/2} cos + k_j sin
 *   codes = e4m3(fp32(k') / k_scale), e4m3(fp32(v) / v_scale)  (fp32 division, RNE)
 *   cache row p = cache_start + r;  slot = block_table[p / bs] * bs + p % bs
 *   ([v4_mtp.rs] forward_one step 4 computes the slot this way; block size 16 in
 *   [new.rs] and [init.rs] KV configs). Element (slot, head, d) of a cache laid out
 *   [num_blocks, bs, nkv, hd] is at ((slot * nkv + head) * hd + d).
 * A row whose block-table entry is missing or out of range is not written and
 * raises ORC_FLAG_BAD_SLOT.
 *
 * Readings (the pages are silent): by default no norm sits between fc and the k/v
 * projections and no per-head k norm is applied (the benchmark's step list has neither,
 * though the reference scratch has a `normed2` buffer and the head a `k_norm` weight);
 * with `in_norm` given (orc_prefill_rows_ext), k and v are projected from
 * bf16(rms(y) in_norm) -- the decoder layer's input norm, the scratch's `normed2`
 * buffer -- instead of y (same eps and weight mode as the combiner's norms);
 * with `k_norm` given, each bf16 k head is RMS-normalized over hd
 * with those weights (same eps and weight mode as the combiner's norms) and rounded to
 * bf16 before RoPE, the usual order of a per-head k norm; RoPE style, rotary dim and theta come from the
 * benchmark configuration (NeoX, full head, base given); the RoPE position of each
 * row is an explicit input because a forward_one at RoPE position p writes pair key
 * p - 1 ([mtp_head.rs] MtpProposerState docs), i.e. position and cache row differ.
 *
 * Pins (tests/test_oracle.py): RoPE at pos 0 is the identity, preserves each pair's
 * norm, turns pair 0 by exactly 1 rad at pos 1 and composes additively; the slot
 * formula on hand-worked cases from the V4 page; stage-by-stage agreement with the
 * combiner and a numpy matmul.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include "oracle.h"

void orc_rope_neox(const double* k, int32_t hd, double pos, double base, double* out) {
    int32_t half = hd / 2;
    for (int32_t j = 0; j < half; ++j) {
        double inv_freq = pow(base, -2.0 * (double)j / (double)hd);
        double th = pos * inv_freq;
        double c = cos(th), s = sin(th);
        out[j] = k[j] * c - k[j + half] * s;
        out[j + half] = k[j + half] * c + k[j] * s;
    }
}

int64_t orc_slot(const int32_t* block_table, int64_t n_table, int32_t block_size,
                 int64_t num_blocks, int64_t p) {
    if (p < 0) return -1;
    int64_t bi = p / block_size;
    if (bi >= n_table) return -1;
    int64_t blk = block_table[bi];
    if (blk < 0 || blk >= num_blocks) return -1;
    return blk * block_size + p % block_size;
}

void orc_kv_encode(const uint16_t* vals, int64_t n, float scale, uint8_t* codes) {
    for (int64_t i = 0; i < n; ++i) {
        float v = (float)orc_bf16_to_f64(vals[i]);
        float q = v / scale;
        codes[i] = orc_e4m3_encode((double)q);
    }
}

static void matvec_bf16(const uint16_t* W, int64_t n, int64_t k, const uint16_t* x,
                        uint16_t* y) {
    for (int64_t i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < k; ++j)
            acc += orc_bf16_to_f64(W[i * k + j]) * orc_bf16_to_f64(x[j]);
        y[i] = orc_f64_to_bf16(acc);
    }
}

int32_t orc_prefill_rows_ext(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                         const uint16_t* hidden, int32_t h,
                         const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                         double eps, const uint16_t* fc, const uint16_t* wk,
                         const uint16_t* wv, int32_t nkv, int32_t hd, double rope_base,
                         const int32_t* rope_pos, int64_t cache_start,
                         const int32_t* block_table, int64_t n_table,
                         int32_t block_size, int64_t num_blocks, float k_scale,
                         float v_scale, int32_t mode, const uint16_t* k_norm,
                         const uint16_t* in_norm, const int64_t* rows, int64_t nrows,
                         uint16_t* out_y, uint16_t* out_k_rot, uint16_t* out_v,
                         uint8_t* out_k_codes, uint8_t* out_v_codes, int64_t* out_slot) {
    int32_t flags = 0;
    const int64_t kvd = (int64_t)nkv * hd;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : flags)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t r = rows[i];
        uint16_t* y = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)h);
        uint16_t* n2 = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)h);
        uint16_t* kb = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)kvd);
        uint16_t* vb = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)kvd);
        double* kd = (double*)malloc(sizeof(double) * (size_t)hd);
        double* kr = (double*)malloc(sizeof(double) * (size_t)hd);
        int32_t tok = tokens[r];
        flags |= orc_combine_mode(embed, vocab, &tok, hidden + r * (int64_t)h, 1, h,
                                  w_norm_embed, w_norm_hidden, eps, mode, fc, NULL, y);
        /* the decoder layer's input norm (the scratch's normed2), when given, feeds k and v */
        const uint16_t* a = y;
        if (in_norm) {
            orc_rmsnorm_row_mode(y, in_norm, h, eps, mode, n2);
            a = n2;
        }
        matvec_bf16(wk, kvd, h, a, kb);
        matvec_bf16(wv, kvd, h, a, vb);
        for (int32_t hh = 0; hh < nkv; ++hh) {
            if (k_norm)  /* per-head RMSNorm of k over hd, before RoPE */
                orc_rmsnorm_row_mode(kb + hh * hd, k_norm, hd, eps, mode, kb + hh * hd);
            for (int32_t d = 0; d < hd; ++d) kd[d] = orc_bf16_to_f64(kb[hh * hd + d]);
            orc_rope_neox(kd, hd, (double)rope_pos[r], rope_base, kr);
            for (int32_t d = 0; d < hd; ++d) kb[hh * hd + d] = orc_f64_to_bf16(kr[d]);
        }
        if (out_y)
            for (int32_t j = 0; j < h; ++j) out_y[i * h + j] = y[j];
        if (out_k_rot)
            for (int64_t j = 0; j < kvd; ++j) out_k_rot[i * kvd + j] = kb[j];
        if (out_v)
            for (int64_t j = 0; j < kvd; ++j) out_v[i * kvd + j] = vb[j];
        orc_kv_encode(kb, kvd, k_scale, out_k_codes + i * kvd);
        orc_kv_encode(vb, kvd, v_scale, out_v_codes + i * kvd);
        int64_t s = orc_slot(block_table, n_table, block_size, num_blocks, cache_start + r);
        if (s < 0) flags |= ORC_FLAG_BAD_SLOT;
        out_slot[i] = s;
        free(y);
        free(n2);
        free(kb);
        free(vb);
        free(kd);
        free(kr);
    }
    return flags;
}

int32_t orc_prefill_rows(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                         const uint16_t* hidden, int32_t h,
                         const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                         double eps, const uint16_t* fc, const uint16_t* wk,
                         const uint16_t* wv, int32_t nkv, int32_t hd, double rope_base,
                         const int32_t* rope_pos, int64_t cache_start,
                         const int32_t* block_table, int64_t n_table,
                         int32_t block_size, int64_t num_blocks, float k_scale,
                         float v_scale, const int64_t* rows, int64_t nrows,
                         uint16_t* out_y, uint16_t* out_k_rot, uint16_t* out_v,
                         uint8_t* out_k_codes, uint8_t* out_v_codes, int64_t* out_slot) {
    return orc_prefill_rows_ext(embed, vocab, tokens, hidden, h, w_norm_embed, w_norm_hidden, eps,
                                fc, wk, wv, nkv, hd, rope_base, rope_pos, cache_start, block_table,
                                n_table, block_size, num_blocks, k_scale, v_scale, 0, NULL, NULL,
                                rows,
                                nrows, out_y, out_k_rot, out_v, out_k_codes, out_v_codes, out_slot);
}
