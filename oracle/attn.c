/*
 * Single-token paged decode attention over the drafter's FP8 KV cache. TEST
 * INFRASTRUCTURE (see oracle.h): plain loops, fp64.
 *
 * [new.rs] MtpHead::new gives the drafter one attention layer with its own paged KV cache
 * (block size 16; FP8 for NVFP4 heads, fed unit K/V scales by default) and looks up a
 * single-token decode-attention kernel for that FP8 cache next to its BF16 twin;
 * [mtp_head.rs] module docs put the attention after fc in the draft's forward order;
 * [v4_mtp.rs] forward_one step 4: cache row p lives at slot
 * block_table[p / bs] * bs + p % bs. The pages print no attention formula; the reading
 * here is the standard one for one query token over the rows 0 .. seq_len - 1 of its
 * sequence, with grouped kv heads (query head i reads kv head i / (nq / nkv)):
 *   s_p = scale * sum_d q[i, d] * (k_scale * e4m3(K[slot(p), g, d]))
 *   w_p = exp(s_p - max_p' s_p') / sum_p' exp(s_p' - max)
 *   out[i, d] = sum_p w_p * (v_scale * e4m3(V[slot(p), g, d]))
 * q is bf16 (as every activation buffer of the pages), the sums and the softmax are fp64,
 * out is returned in fp64. A row whose block is missing or out of range is skipped and
 * raises ORC_FLAG_BAD_SLOT; with no readable row the output is zero.
 *
 * Pins (tests/test_oracle.py): one row gives that row's values exactly; a zero scale or
 * identical keys give the mean of the values; one planted key whose score exceeds the
 * others' by ~800 gives that row's values (no overflow); permuting physical blocks (with
 * their data) changes nothing; query heads of one group see the same kv head.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include "oracle.h"

int32_t orc_paged_decode_attn(const uint16_t* q, int32_t nq, int32_t nkv, int32_t hd,
                              const uint8_t* k_cache, const uint8_t* v_cache,
                              const int32_t* block_table, int64_t n_table, int32_t block_size,
                              int64_t num_blocks, int64_t seq_len, double k_scale, double v_scale,
                              double scale, double* out) {
    int32_t flags = 0;
    const int32_t group = nq / nkv;
    double* s = (double*)malloc(sizeof(double) * (size_t)(seq_len > 0 ? seq_len : 1));
    int64_t* slot = (int64_t*)malloc(sizeof(int64_t) * (size_t)(seq_len > 0 ? seq_len : 1));
    for (int64_t p = 0; p < seq_len; ++p) {
        slot[p] = orc_slot(block_table, n_table, block_size, num_blocks, p);
        if (slot[p] < 0) flags |= ORC_FLAG_BAD_SLOT;
    }
    for (int32_t i = 0; i < nq; ++i) {
        const int32_t g = i / group;
        double mx = -INFINITY;
        for (int64_t p = 0; p < seq_len; ++p) {
            if (slot[p] < 0) continue;
            const uint8_t* kr = k_cache + (slot[p] * nkv + g) * (int64_t)hd;
            double acc = 0.0;
            for (int32_t d = 0; d < hd; ++d)
                acc += orc_bf16_to_f64(q[(int64_t)i * hd + d]) * (k_scale * orc_e4m3_value(kr[d]));
            s[p] = scale * acc;
            if (s[p] > mx) mx = s[p];
        }
        double den = 0.0;
        for (int64_t p = 0; p < seq_len; ++p)
            if (slot[p] >= 0) den += exp(s[p] - mx);
        for (int32_t d = 0; d < hd; ++d) out[(int64_t)i * hd + d] = 0.0;
        if (den == 0.0) continue;
        for (int64_t p = 0; p < seq_len; ++p) {
            if (slot[p] < 0) continue;
            const double w = exp(s[p] - mx) / den;
            const uint8_t* vr = v_cache + (slot[p] * nkv + g) * (int64_t)hd;
            for (int32_t d = 0; d < hd; ++d)
                out[(int64_t)i * hd + d] += w * (v_scale * orc_e4m3_value(vr[d]));
        }
    }
    free(s);
    free(slot);
    return flags;
}
