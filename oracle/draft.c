/*
 * One draft step's weight-streaming part: combiner, lm_head sweep, argmax.
 * TEST INFRASTRUCTURE (see oracle.h). fp64 accumulation throughout; values are
 * rounded to bf16 only where the reference stores a bf16 activation buffer.
 *
 * Combiner ([v4_mtp.rs] module docs "One draft" and forward_one steps 1-2;
 * [mtp_head.rs] module docs: embed+hidden concat -> fc):
 *   e  = embed_tokens[token]                      (a row copy)
 *   ne = bf16(rms(e) * w_enorm),  nh = bf16(rms(hidden) * w_hnorm),
 *        rms(v)_i = v_i / sqrt(sum_j v_j^2 / h + eps)  (plain weights: the V4 page
 *        notes its norm weights multiply as w * x_normed, not (1 + w))
 *   c  = [ne || nh]   (embedding half first)
 *   y  = bf16(fc . c) with fc [h, 2h] (MtpHead::new quantizes fc as n = h, k = 2h)
 * A token id outside [0, vocab) reads as a zero row and raises ORC_FLAG_BAD_TOKEN.
 *
 * lm_head sweep + argmax ([v4_mtp.rs] forward_one steps 6-7, argmax_grammar_masked;
 * [init.rs] the draft-head sweep over rows packed at K):
 *   l[m, n] = sum_k deq(W)[n, k] * x[m, k]  for n < n_eff
 *   token t is allowed iff no mask, or word t/32 exists and bit t%32 of it is set;
 *   idx = the lowest allowed n whose logit equals the allowed maximum (an upward
 *   scan from -inf with a strict '>'); no allowed token -> idx 0, value -inf and
 *   ORC_FLAG_EMPTY_MASK (the page returns token 0 as a pad draft).
 * Reading (where the page rounds logits to bf16 before its argmax): the argmax here
 * is taken on the unrounded logit, so that a top-2 gap larger than one bf16 ulp of
 * the logit decides the winner.
 *
 * Top-1 log-probability ([mtp_head.rs] MtpHead fields: argmax_bf16_batch_lp emits
 * each row's top-1 log-probability; the chain confidence is the smallest top-1
 * softmax probability across drafts): the log-softmax of the logits over the allowed
 * tokens, taken at the argmax,
 *   lp = l[idx] - log(sum over allowed n of exp(l[n])),
 * evaluated as -log(sum over allowed n of exp(l[n] - l[idx])) since l[idx] is the
 * allowed maximum. Reading: no temperature, the same unrounded logits and mask as
 * the argmax; no allowed token -> -inf.
 *
 * Pins (tests/test_oracle.py): one-hot inputs select exact table entries, numpy's
 * float64 matmul on the dequantized table, planted maxima, masked decoys,
 * duplicate rows (lowest index), the all-masked row, closed forms of RMSNorm; for
 * the log-probability: equal logits give -log(allowed count), a single allowed token
 * gives 0, two tied maxima far above the rest give -log 2, and adding a constant to
 * every logit changes nothing.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#include "oracle.h"

int32_t orc_num_threads(void) {
#ifdef _OPENMP
    return (int32_t)omp_get_max_threads();
#else
    return 1;
#endif
}

/* RMSNorm of one row, y_i = bf16(x_i / sqrt(mean(x^2) + eps) * w'_i), with w' = w (mode 0,
 * the plain weights of the V4 page) or w' = 1 + w (mode 1: the V4 page notes that the
 * shared rms_norm kernel applies 1 + w). */
void orc_rmsnorm_row_mode(const uint16_t* x, const uint16_t* w, int64_t h, double eps,
                          int32_t mode, uint16_t* y) {
    double ss = 0.0;
    for (int64_t i = 0; i < h; ++i) {
        double v = orc_bf16_to_f64(x[i]);
        ss += v * v;
    }
    double inv = 1.0 / sqrt(ss / (double)h + eps);
    for (int64_t i = 0; i < h; ++i) {
        double wi = orc_bf16_to_f64(w[i]) + (mode == 1 ? 1.0 : 0.0);
        y[i] = orc_f64_to_bf16(orc_bf16_to_f64(x[i]) * inv * wi);
    }
}

void orc_rmsnorm_row(const uint16_t* x, const uint16_t* w, int64_t h, double eps,
                     uint16_t* y) {
    orc_rmsnorm_row_mode(x, w, h, eps, 0, y);
}

int32_t orc_combine(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                    const uint16_t* hidden, int32_t M, int32_t h,
                    const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                    double eps, const uint16_t* fc, uint16_t* out_concat,
                    uint16_t* out_y) {
    return orc_combine_mode(embed, vocab, tokens, hidden, M, h, w_norm_embed, w_norm_hidden,
                            eps, 0, fc, out_concat, out_y);
}

int32_t orc_combine_mode(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                         const uint16_t* hidden, int32_t M, int32_t h,
                         const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                         double eps, int32_t mode, const uint16_t* fc, uint16_t* out_concat,
                         uint16_t* out_y) {
    int32_t flags = 0;
    uint16_t* c = (uint16_t*)malloc(sizeof(uint16_t) * 2 * (size_t)h);
    uint16_t* zero = (uint16_t*)calloc((size_t)h, sizeof(uint16_t));
    for (int32_t m = 0; m < M; ++m) {
        int64_t tok = tokens[m];
        const uint16_t* e = zero;
        if (tok >= 0 && tok < vocab)
            e = embed + tok * (int64_t)h;
        else
            flags |= ORC_FLAG_BAD_TOKEN;
        orc_rmsnorm_row_mode(e, w_norm_embed, h, eps, mode, c);
        orc_rmsnorm_row_mode(hidden + (int64_t)m * h, w_norm_hidden, h, eps, mode, c + h);
        if (out_concat)
            for (int64_t j = 0; j < 2 * h; ++j) out_concat[(int64_t)m * 2 * h + j] = c[j];
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < h; ++i) {
            double acc = 0.0;
            for (int64_t j = 0; j < 2 * (int64_t)h; ++j)
                acc += orc_bf16_to_f64(fc[i * 2 * h + j]) * orc_bf16_to_f64(c[j]);
            out_y[(int64_t)m * h + i] = orc_f64_to_bf16(acc);
        }
    }
    free(c);
    free(zero);
    return flags;
}

static int allowed(const int32_t* mask, int64_t mask_words, int64_t t) {
    if (!mask) return 1;
    int64_t word = t / 32;
    if (word >= mask_words) return 0;
    return (int)(((uint32_t)mask[word] >> (t % 32)) & 1u);
}

int32_t orc_argmax_masked(const double* logits, int64_t n, const int32_t* mask,
                          int64_t mask_words, int32_t* out_idx, double* out_val) {
    int32_t best = 0;
    double best_val = -INFINITY;
    int any = 0;
    for (int64_t t = 0; t < n; ++t) {
        if (!allowed(mask, mask_words, t)) continue;
        any = 1;
        if (logits[t] > best_val) {
            best_val = logits[t];
            best = (int32_t)t;
        }
    }
    if (!any) {
        *out_idx = 0;
        *out_val = -INFINITY;
        return ORC_FLAG_EMPTY_MASK;
    }
    *out_idx = best;
    *out_val = best_val;
    return 0;
}

double orc_top1_logprob(const double* logits, int64_t n, const int32_t* mask,
                        int64_t mask_words) {
    int32_t idx = 0;
    double top = 0.0;
    if (orc_argmax_masked(logits, n, mask, mask_words, &idx, &top) != 0) return -INFINITY;
    double sum = 0.0;
    for (int64_t t = 0; t < n; ++t)
        if (allowed(mask, mask_words, t)) sum += exp(logits[t] - top);
    return -log(sum);
}

int32_t orc_lm_head_argmax(int32_t fmt, const void* data, const float* row_scale,
                           const uint8_t* block_scale, float global_scale,
                           int64_t n_eff, int64_t k, const uint16_t* x, int32_t M,
                           const int32_t* mask, int64_t mask_words,
                           int64_t mask_stride_words, double* logits,
                           int32_t* out_idx, double* out_val) {
    double* L = logits ? logits : (double*)malloc(sizeof(double) * (size_t)M * (size_t)n_eff);
    double* xd = (double*)malloc(sizeof(double) * (size_t)M * (size_t)k);
    for (int64_t i = 0; i < (int64_t)M * k; ++i) xd[i] = orc_bf16_to_f64(x[i]);
#pragma omp parallel
    {
        double* row = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(static)
        for (int64_t n = 0; n < n_eff; ++n) {
            orc_dequant_row(fmt, data, row_scale, block_scale, global_scale, k, n, row);
            for (int32_t m = 0; m < M; ++m) {
                const double* xm = xd + (int64_t)m * k;
                double acc = 0.0;
                for (int64_t j = 0; j < k; ++j) acc += row[j] * xm[j];
                L[(int64_t)m * n_eff + n] = acc;
            }
        }
        free(row);
    }
    int32_t flags = 0;
    for (int32_t m = 0; m < M; ++m) {
        const int32_t* mrow = mask ? mask + (int64_t)m * mask_stride_words : NULL;
        flags |= orc_argmax_masked(L + (int64_t)m * n_eff, n_eff, mrow, mask_words,
                                   out_idx + m, out_val + m);
    }
    free(xd);
    if (!logits) free(L);
    return flags;
}
