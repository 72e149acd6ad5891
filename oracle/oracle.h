/*
 * CPU oracle for the MTP draft-head hot path -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously-correct C: scalar loops, fp64 accumulation, no SIMD,
 * no blocking or fusion. Only tests/, the smoke check and the benchmark's CPU
 * baseline leg may load it. It shares no code, header or constant with the
 * CUDA library; the two meet only through seeded input arrays.
 *
 * Sources (web pages on one subject: the single-layer multi-token-prediction
 * draft head):
 *   [mtp_head.rs]   spark_model/layers/mtp_head.rs (MtpHead docs, MtpQuantization,
 *                   ProjectionWeight, the gemv dispatch, quantize_proj)
 *   [new.rs]        metrale_model_layers/layers/mtp_head/new.rs (MtpHead::new:
 *                   quantizer kernels, KV pool, prefill scratch)
 *   [init.rs]       metrale_model_arch/glm5next_mtp_head/init.rs (vocab-sharded
 *                   draft lm_head, FP8 shard, the head-skip timing)
 *   [v4_mtp.rs]     metrale_model_arch/deepseek_v4_mtp.rs (module docs "One
 *                   draft", forward_one steps 1-7, argmax_grammar_masked)
 * Public format definitions where the pages are silent: OCP 8-bit floating
 * point (E4M3FN) and OCP microscaling FP4 (E2M1) with the NVFP4 two-level
 * scale recipe.
 *
 * Pinning: every function here is pinned in tests/test_oracle.py against
 * brute force, closed forms, invariants or an independent library routine.
 */
#ifndef MTP_ORACLE_H
#define MTP_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* formats.c */
double   orc_bf16_to_f64(uint16_t b);
uint16_t orc_f64_to_bf16(double x);
double   orc_e4m3_value(uint8_t code);
uint8_t  orc_e4m3_encode(double v);
double   orc_e2m1_value(uint8_t code);
uint8_t  orc_e2m1_encode(double v);
void     orc_e4m3_encode_vec(const double* v, int64_t n, uint8_t* out);
void     orc_e2m1_encode_vec(const double* v, int64_t n, uint8_t* out);
void     orc_f64_to_bf16_vec(const double* v, int64_t n, uint16_t* out);

/* quant.c */
void orc_quantize_fp8_rows(const uint16_t* w, int64_t n, int64_t k,
                           uint8_t* codes, float* row_scale);
void orc_quantize_nvfp4(const uint16_t* w, int64_t n, int64_t k,
                        uint8_t* codes, uint8_t* block_scale, float* global_scale);
void orc_dequant_row(int32_t fmt, const void* data, const float* row_scale,
                     const uint8_t* block_scale, float global_scale,
                     int64_t k, int64_t row, double* out);

/* draft.c */
void orc_rmsnorm_row(const uint16_t* x, const uint16_t* w, int64_t h, double eps,
                     uint16_t* y);
void orc_rmsnorm_row_mode(const uint16_t* x, const uint16_t* w, int64_t h, double eps,
                          int32_t mode, uint16_t* y);
int32_t orc_combine_mode(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                         const uint16_t* hidden, int32_t M, int32_t h,
                         const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                         double eps, int32_t mode, const uint16_t* fc, uint16_t* out_concat,
                         uint16_t* out_y);
int32_t orc_prefill_rows_ext(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                             const uint16_t* hidden, int32_t h,
                             const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                             double eps, const uint16_t* fc, const uint16_t* wk,
                             const uint16_t* wv, int32_t nkv, int32_t hd, double rope_base,
                             const int32_t* rope_pos, int64_t cache_start,
                             const int32_t* block_table, int64_t n_table,
                             int32_t block_size, int64_t num_blocks, float k_scale,
                             float v_scale, int32_t mode, const uint16_t* k_norm,
                             const uint16_t* in_norm,
                             const int64_t* rows, int64_t nrows,
                             uint16_t* out_y, uint16_t* out_k_rot, uint16_t* out_v,
                             uint8_t* out_k_codes, uint8_t* out_v_codes, int64_t* out_slot);
int32_t orc_combine(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                    const uint16_t* hidden, int32_t M, int32_t h,
                    const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                    double eps, const uint16_t* fc, uint16_t* out_concat,
                    uint16_t* out_y);
int32_t orc_lm_head_argmax(int32_t fmt, const void* data, const float* row_scale,
                           const uint8_t* block_scale, float global_scale,
                           int64_t n_eff, int64_t k, const uint16_t* x, int32_t M,
                           const int32_t* mask, int64_t mask_words,
                           int64_t mask_stride_words, double* logits,
                           int32_t* out_idx, double* out_val);
int32_t orc_argmax_masked(const double* logits, int64_t n, const int32_t* mask,
                          int64_t mask_words, int32_t* out_idx, double* out_val);
double  orc_top1_logprob(const double* logits, int64_t n, const int32_t* mask,
                         int64_t mask_words);

/* prefill.c */
void    orc_rope_neox(const double* k, int32_t hd, double pos, double base, double* out);
int64_t orc_slot(const int32_t* block_table, int64_t n_table, int32_t block_size,
                 int64_t num_blocks, int64_t p);
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
                         uint8_t* out_k_codes, uint8_t* out_v_codes, int64_t* out_slot);
void orc_kv_encode(const uint16_t* vals, int64_t n, float scale, uint8_t* codes);

/* attn.c: single-token paged decode attention over an E4M3 cache [num_blocks, bs, nkv, hd] */
int32_t orc_paged_decode_attn(const uint16_t* q, int32_t nq, int32_t nkv, int32_t hd,
                              const uint8_t* k_cache, const uint8_t* v_cache,
                              const int32_t* block_table, int64_t n_table, int32_t block_size,
                              int64_t num_blocks, int64_t seq_len, double k_scale, double v_scale,
                              double scale, double* out);

/* threads the OpenMP loops use */
int32_t orc_num_threads(void);

/* status flags returned by the oracle (bit set) */
#define ORC_FLAG_BAD_TOKEN   1
#define ORC_FLAG_EMPTY_MASK  2
#define ORC_FLAG_BAD_SLOT    4

#ifdef __cplusplus
}
#endif
#endif
