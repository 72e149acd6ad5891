/*
 * mtp.h -- C ABI of the B200 (sm_100a) multi-token-prediction draft-head library.
 *
 * The library implements the weight-streaming hot path of a single-layer MTP draft
 * head, as described by these pages (cited below by title and section):
 *   [mtp_head.rs] spark_model/layers/mtp_head.rs -- MtpHead docs, MtpQuantization,
 *                 ProjectionWeight, the gemv dispatch, quantize_proj, the drafter-
 *                 prefill docs and MtpPrefillScratch;
 *   [new.rs]      metrale_model_layers/layers/mtp_head/new.rs -- MtpHead::new (the
 *                 quantizer kernels, the KV-pool config, the prefill scratch);
 *   [init.rs]     metrale_model_arch/glm5next_mtp_head/init.rs -- the vocab-sharded
 *                 draft lm_head over [vocab, hidden] rows packed at K, FP8 shard;
 *   [v4_mtp.rs]   metrale_model_arch/deepseek_v4_mtp.rs -- module docs "One draft",
 *                 forward_one steps 1-7, argmax_grammar_masked.
 *
 * Conventions for every entry point:
 *  - Pointers marked (device) are CUDA device memory owned by the caller; the
 *    library never allocates, frees or retains them and keeps no state between
 *    calls (except the workspace contract of the functions that take one).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *    All work is enqueued asynchronously on it; results are valid once the stream
 *    reaches that point.
 *  - bf16 values are passed as their uint16_t bit patterns.
 *  - Arguments are validated on the host before anything is launched. A call that
 *    returns non-zero has enqueued nothing (MTP_ERR_CUDA: a launch failed; earlier
 *    kernels of the same call may have been enqueued).
 *  - Data-dependent problems found on the device (a token id outside the table, a
 *    cache row with no block, a mask that allows nothing) never trap: the kernel
 *    ORs an MTP_DEVFLAG_* bit into *dev_err (when dev_err is not NULL) and carries
 *    on with the documented fallback. Read it after the stream synchronises.
 *  - Functions are re-entrant; calls that share a workspace must not overlap in time.
 */
#ifndef MTP_H
#define MTP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 2: mtp_combine, mtp_draft_step and mtp_prefill_kv take norm_mode; mtp_prefill_kv takes
 * k_norm and in_norm. */
#define MTP_ABI_VERSION 2

typedef enum {
    MTP_OK = 0,
    MTP_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or stride */
    MTP_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels handle (shape, M) */
    MTP_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the *_ws_bytes size */
    MTP_ERR_CUDA = 4,        /* a CUDA launch or API call failed */
    MTP_WARN_EMPTY_MASK = 5  /* mtp_devflags_status(): a mask allowed no token */
} mtp_status;

/* RMSNorm weight modes (every norm of a call): the plain w * x_normed of the V4 head
 * ([v4_mtp.rs] DeepseekV4MtpHead::new: "the norm weights are plain"), or (1 + w) * x_normed,
 * what that page says the shared rms_norm kernel applies. */
#define MTP_NORM_W 0
#define MTP_NORM_ONE_PLUS_W 1

/* Bits a kernel ORs into the caller's device error word. */
#define MTP_DEVFLAG_BAD_TOKEN 1  /* token id outside [0, vocab): its row read as zeros */
#define MTP_DEVFLAG_EMPTY_MASK 2 /* a row's mask allowed nothing: idx 0, value -inf */
#define MTP_DEVFLAG_BAD_SLOT 4   /* a cache row had no valid block: row not written */
#define MTP_DEVFLAG_TIMEOUT 8    /* an internal pipeline wait ran out (about 1 s): the
                                    call's outputs are not valid */

/* Weight formats ([mtp_head.rs] MtpQuantization and ProjectionWeight: Bf16, Fp8,
 * Nvfp4). */
typedef enum {
    MTP_FMT_BF16 = 0,    /* data: bf16 [n, k] */
    MTP_FMT_FP8_ROW = 1, /* data: E4M3FN codes [n, k]; row_scale: f32 [n] */
    MTP_FMT_NVFP4 = 2    /* data: E2M1 codes [n, k/2] (element 2j = low nibble of byte
                            j); block_scale: E4M3FN [n, pitch] with
                            pitch = mtp_nvfp4_scale_pitch(k) (k/16 rounded up to a
                            multiple of 16; padding bytes zero); global_scale: f32[1] */
} mtp_format;

/* A [n, k] weight table in one of the formats, rows packed at k (no row stride:
 * [init.rs] notes the draft-head GEMV assumes rows packed at K). All pointers are
 * device pointers (data and block_scale 16-byte aligned); the unused ones must be
 * NULL. dequant(W)[r, j] is the bf16 value, e4m3(code) * row_scale[r], or
 * e2m1(code) * e4m3(block_scale[r * pitch + j/16]) * global_scale[0]. */
typedef struct {
    int32_t fmt;
    int32_t reserved; /* must be 0 */
    int64_t n;
    int64_t k;
    const void* data;
    const float* row_scale;
    const uint8_t* block_scale;
    const float* global_scale;
} mtp_weight;

/* Row pitch in bytes of an NVFP4 block-scale table: k/16 rounded up to a multiple
 * of 16, so that every row starts 16-byte aligned. */
int64_t mtp_nvfp4_scale_pitch(int64_t k);

/* ---------------------------------------------------------------------------------
 * mtp_quantize_fp8 -- BF16 -> FP8 E4M3 with one fp32 scale per row.
 * Source: [new.rs] MtpHead::new looks up the BF16 -> FP8 quantizer; [mtp_head.rs]
 * quantize_proj calls it for MtpQuantization::Fp8; [init.rs] quantizes the draft
 * head's rows to FP8. Rule (fp32, round to nearest even): a = max_j |w[r, j]|,
 * row_scale[r] = a / 448, codes[r, j] = e4m3_satfinite(w[r, j] / row_scale[r]); an
 * all-zero row gets scale 0 and codes 0.
 *   w          (device) bf16 [n, k], 16-byte aligned
 *   codes      (device) u8 [n, k], 16-byte aligned, written
 *   row_scale  (device) f32 [n], written
 * Requires n >= 1, k >= 16, k % 16 == 0.
 * ------------------------------------------------------------------------------ */
mtp_status mtp_quantize_fp8(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                            float* row_scale, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_quantize_nvfp4 -- BF16 -> NVFP4 in two passes.
 * Source: [new.rs] MtpHead::new looks up the global-absmax pass and the BF16 -> NVFP4
 * pass; [mtp_head.rs] quantize_proj uses them for MtpQuantization::Nvfp4; the
 * per-row size is k/2 code bytes (the MtpHead::new lm-head size log). Rule (fp32,
 * round to nearest even): A = max|w|, g = A / 2688 (1 if A == 0); per block b of
 * 16 consecutive k: B = max|w_b|, sb = e4m3_satfinite((B / 6) / g),
 * S = e4m3(sb) * g, code = e2m1_satfinite(w / S) (0 when S == 0).
 *   w            (device) bf16 [n, k], 16-byte aligned
 *   codes        (device) u8 [n, k/2] written (two codes per byte, element 2j low)
 *   block_scale  (device) u8 [n, mtp_nvfp4_scale_pitch(k)] written (16-byte aligned;
 *                the padding after the k/16 scales of each row is written as 0)
 *   global_scale (device) f32 [1] written (g)
 *   ws           (device) >= mtp_quantize_nvfp4_ws_bytes(n, k) bytes, 16-byte
 *                aligned, ALL ZERO before the first call; each call leaves it zero.
 * Requires n >= 1, k >= 32, k % 32 == 0.
 * ------------------------------------------------------------------------------ */
size_t mtp_quantize_nvfp4_ws_bytes(int64_t n, int64_t k);
mtp_status mtp_quantize_nvfp4(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                              uint8_t* block_scale, float* global_scale, void* ws,
                              size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_combine -- the draft's embed+hidden combiner for M rows.
 * Source: [v4_mtp.rs] forward_one steps 1-2 (embedding row copy; two RMSNorms with
 * plain weights w * x_normed; e_proj / h_proj combiner) and [mtp_head.rs] module
 * docs (embed+hidden concat -> fc), with fc [h, 2h] as quantized in [new.rs].
 *   e = embed[token_ids[m]];  ne = bf16(e / sqrt(mean(e^2) + eps) * w_norm_embed)
 *   nh = bf16(x / sqrt(mean(x^2) + eps) * w_norm_hidden),  x = hidden[m]
 *   out[m] = bf16(fc . [ne || nh])           (embedding half first)
 *   (with norm_mode MTP_NORM_ONE_PLUS_W the weights are 1 + w_norm_*; any other value
 *   than the two MTP_NORM_* is MTP_ERR_INVALID_ARG)
 *   embed         (device) bf16 [vocab, h]
 *   token_ids     (device) i32 [M]; an id outside [0, vocab) reads as a zero row and
 *                 sets MTP_DEVFLAG_BAD_TOKEN
 *   hidden        (device) bf16 [M, h]
 *   w_norm_embed, w_norm_hidden (device) bf16 [h]
 *   fc            weight with n == h, k == 2h (MTP_FMT_BF16, MTP_FMT_FP8_ROW or
 *                 MTP_FMT_NVFP4)
 *   out           (device) bf16 [M, h], written
 *   dev_err       (device) i32 [1] or NULL
 * Requires 1 <= M <= 16, h % 16 == 0, fc rows a multiple of 128 bytes (2h % 64 for
 * BF16, % 128 for FP8, % 256 for NVFP4), all device pointers 16-byte aligned except
 * token_ids / dev_err (4-byte).
 * ------------------------------------------------------------------------------ */
mtp_status mtp_combine(const uint16_t* embed, int64_t vocab, const int32_t* token_ids,
                       const uint16_t* hidden, int32_t M, int32_t h,
                       const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                       float eps, int32_t norm_mode, const mtp_weight* fc, uint16_t* out,
                       int32_t* dev_err, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_lm_head_argmax -- the draft lm_head sweep fused with a (masked) argmax.
 * Source: [v4_mtp.rs] forward_one steps 6-7 (lm_head GEMV over the first v rows,
 * v = the effective vocab, then argmax, grammar-masked when a bitmask is given) and
 * argmax_grammar_masked (token t allowed iff word t/32 exists and bit t%32 is set;
 * lowest index wins ties; nothing allowed -> token 0); [init.rs] the sweep over
 * [vocab, hidden] rows, "most of the drafter's time".
 *   l[m, r] = sum_j dequant(head)[r, j] * x[m, j]   (fp32 accumulation), r < n_eff
 *   out_idx[m] = lowest allowed r with the largest l[m, r]; the argmax is taken on
 *   the fp32 logit. No token allowed -> out_idx 0, out_val -inf, MTP_DEVFLAG_EMPTY_MASK.
 *   head          weight [n, k]; n_eff <= n rows are swept (the effective vocab)
 *   x             (device) bf16 [M, k], 16-byte aligned
 *   mask          (device) i32 words or NULL; row m's mask starts at
 *                 mask + m * mask_stride_words (stride 0: one mask for all rows) and
 *                 has mask_words words (tokens past 32 * mask_words are disallowed)
 *   out_idx       (device) i32 [M], written
 *   out_val       (device) f32 [M] or NULL: the winning logit
 *   out_logits    (device) bf16 [M, n_eff] or NULL: bf16(l), masked tokens -inf
 *   dev_err       (device) i32 [1] or NULL
 *   ws            (device) >= mtp_lm_head_ws_bytes(head, n_eff, M) bytes, 16-byte
 *                 aligned, ALL ZERO before the first call; each call leaves its
 *                 counter zero again. It also holds x as the quantized tables' sweeps
 *                 read it, rewritten by each call: for FP8 tables with M >= 7 two E4M3
 *                 planes of 16 or 32 rows (2 * 16 * k or 2 * 32 * k bytes), for NVFP4
 *                 with M >= 3 six E2M1 terms per input (N = 32, 48, 96 or 192 rows of
 *                 k / 2 code bytes and k / 16 scale bytes).
 * Requires 1 <= M <= 32, 1 <= n_eff <= n; table rows a multiple of 128 bytes (k % 64
 * for BF16, % 128 for FP8, % 256 for NVFP4; the sweep streams 128-byte segments); for
 * M <= 8 (FP8: M <= 6) the staged inputs (M * k * 2 bytes) must leave shared memory for
 * the stream (MTP_ERR_UNSUPPORTED otherwise; more inputs stream x per K chunk instead).
 * Results are bit-identical for every M within BF16 1-8, 9-16, 17-32; FP8 1-6, 7-16,
 * 17-32; NVFP4 1-2, 3-16, 17-32, whose sweeps sum the same products in different fixed
 * orders. BF16 tables from 9 inputs, FP8 from 7 and NVFP4 from 3 run on the tcgen05
 * tensor cores. There x enters FP8 products as two E4M3 terms whose sum is x exactly
 * except for elements below 2^-9 of the input's largest |x|, which keep an absolute error
 * of at most 2^-17 of that largest |x|; NVFP4 products take the table's E2M1 codes and
 * E4M3 block scales as stored (block-scaled FP4 MMAs) and x as six E2M1 terms per
 * 16-element block with a power-of-two scale, whose sum is x exactly for every element
 * within 9 binades of its block's largest |x| and within 2^-17 of that largest |x|
 * otherwise. With a grammar mask and up to 8 inputs only the table rows that some
 * input's mask allows are read.
 * ------------------------------------------------------------------------------ */
size_t mtp_lm_head_ws_bytes(const mtp_weight* head, int64_t n_eff, int32_t M);
mtp_status mtp_lm_head_argmax(const mtp_weight* head, int64_t n_eff, const uint16_t* x,
                              int32_t M, const int32_t* mask, int64_t mask_words,
                              int64_t mask_stride_words, int32_t* out_idx, float* out_val,
                              uint16_t* out_logits, int32_t* dev_err, void* ws,
                              size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_lm_head_argmax_host -- mtp_lm_head_argmax with the input and the result in pinned
 * host memory: the whole draft step (host -> device input, sweep, device -> host result)
 * in one call on `stream`, with no separate copy operations in the stream.
 * The pages' draft step reads the argmax back to the host every draft ([init.rs] /
 * [v4_mtp.rs] argmax then a 4-byte device-to-host read); this entry point is that step.
 *   x_host    pinned host bf16 [M, k] (cudaHostAlloc / cudaHostRegister; torch
 *             pin_memory), 16-byte aligned; read by the device during the call
 *   out_host  pinned host i32 [2M]: out_host[m] = index, then M f32 values (the winning
 *             logits) at out_host + M; written by the device; valid after the stream
 *             has synchronised
 *   ws        (device) >= mtp_lm_head_host_ws_bytes(head, n_eff, M) bytes: the sweep's
 *             workspace followed by the device copy of x
 * A small kernel copies x into the workspace (it reads before and writes after waiting
 * for the previous kernel in the stream, so the host-link latency overlaps that kernel's
 * tail); the sweep then writes its results straight into out_host. Because x_host is
 * read before earlier work in the stream has finished, its contents must be final when
 * the call is made: work queued earlier on the stream must not write x_host. Returns
 * MTP_ERR_INVALID_ARG if x_host or out_host is not pinned host memory; otherwise the
 * requirements and results of mtp_lm_head_argmax (no logits output).
 * ------------------------------------------------------------------------------ */
size_t mtp_lm_head_host_ws_bytes(const mtp_weight* head, int64_t n_eff, int32_t M);
mtp_status mtp_lm_head_argmax_host(const mtp_weight* head, int64_t n_eff, const uint16_t* x_host,
                                   int32_t M, const int32_t* mask, int64_t mask_words,
                                   int64_t mask_stride_words, int32_t* out_host, int32_t* dev_err,
                                   void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_lm_head_argmax_lp -- mtp_lm_head_argmax that also writes each input's top-1
 * log-probability from the same sweep (no extra table bytes).
 * Source: [mtp_head.rs] MtpHead fields: argmax_bf16_batch_lp, the batched argmax that
 * also emits each row's top-1 log-probability, and the chain confidence (the smallest
 * top-1 softmax probability across drafts).
 *   out_logprob[m] = l[m, idx] - log(sum over allowed r < n_eff of exp(l[m, r]))
 * over the same fp32 logits and mask as the argmax (no temperature); -inf when no
 * token is allowed. The sum of exponentials is accumulated in fp32 in an order that
 * follows the run-time split of the table over SMs, so its last bits can differ from
 * one call to the next; the argmax, out_val and out_logits do not.
 *   out_logprob   (device) f32 [M], written; must not be NULL (MTP_ERR_INVALID_ARG)
 * Every other argument, the workspace and the requirements are mtp_lm_head_argmax's.
 * ------------------------------------------------------------------------------ */
mtp_status mtp_lm_head_argmax_lp(const mtp_weight* head, int64_t n_eff, const uint16_t* x,
                                 int32_t M, const int32_t* mask, int64_t mask_words,
                                 int64_t mask_stride_words, int32_t* out_idx, float* out_val,
                                 float* out_logprob, uint16_t* out_logits, int32_t* dev_err,
                                 void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_draft_step -- one whole draft step for a small BF16 draft head in ONE launch:
 * mtp_combine (BF16 fc) followed by mtp_lm_head_argmax (BF16 head, no logits), fused.
 * Source: [v4_mtp.rs] forward_one steps 1-2 and 6-7 (embedding row, two RMSNorms with plain
 * weights, e_proj / h_proj combiner, lm_head GEMV over the first n_eff rows, argmax,
 * grammar-masked when a bitmask is given) and [mtp_head.rs] module docs (concat -> fc).
 *   c[m] = [bf16(rms(embed[token_ids[m]]) w_norm_embed) || bf16(rms(hidden[m]) w_norm_hidden)]
 *   (weights 1 + w_norm_* with norm_mode MTP_NORM_ONE_PLUS_W, as mtp_combine)
 *   y[m] = bf16(fc . c[m]);  l[m, r] = sum_j head[r, j] y[m, j] (fp32), r < n_eff
 *   out_idx[m] = lowest allowed r with the largest l[m, r] (mask as mtp_lm_head_argmax;
 *   nothing allowed -> 0, -inf and MTP_DEVFLAG_EMPTY_MASK)
 *   embed (device) bf16 [vocab, h]; token_ids (device) i32 [M] (a bad id reads as a zero row
 *   and sets MTP_DEVFLAG_BAD_TOKEN); hidden (device) bf16 [M, h]; w_norm_* (device) bf16 [h];
 *   fc (device) bf16 [h, 2h]; head (device) bf16 [>= n_eff, h], rows packed at h;
 *   out_y (device) bf16 [M, h] or NULL: y, for instance the next step's hidden rows (it
 *   must not overlap hidden: MTP_ERR_INVALID_ARG);
 *   out_idx (device) i32 [M]; out_val (device) f32 [M] or NULL; dev_err i32 [1] or NULL.
 * One thread-block cluster does the whole step (no workspace), so it suits heads that sit
 * in L2 (a few MB, as the tiny draft head's 2 MB); a large head belongs to
 * mtp_lm_head_argmax, which spreads over every SM. The launch allows programmatic
 * dependent launch: a chain of steps, each reading the previous one's out_idx and out_y
 * as its token_ids and hidden, overlaps each launch with the previous step's end.
 * Requires 1 <= M <= 4, 8 <= h <= 1024, h % 8 == 0; embed, hidden, fc, head 16-byte
 * aligned. fc products are summed in fp32 in a fixed order, so y can differ from
 * mtp_combine's in the last bit.
 * ------------------------------------------------------------------------------ */
mtp_status mtp_draft_step(const uint16_t* embed, int64_t vocab, const int32_t* token_ids,
                          const uint16_t* hidden, int32_t M, int32_t h,
                          const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden, float eps,
                          int32_t norm_mode, const uint16_t* fc, const uint16_t* head, int64_t n_eff,
                          const int32_t* mask, int64_t mask_words, int64_t mask_stride_words,
                          uint16_t* out_y, int32_t* out_idx, float* out_val, int32_t* dev_err,
                          void* stream);

/* ---------------------------------------------------------------------------------
 * Vocab-sharded sweep: each of G GPUs sweeps a contiguous range of the table's rows,
 * writes a 16-byte partial per input, the partials are gathered (G x M x 16 bytes, one
 * collective, the caller's: NCCL all-gather over NVLink), and every rank merges them.
 * Source: [init.rs] the draft head split by vocab across tensor-parallel ranks, each
 * rank sweeping its own rows, followed by one small (max, argmax) exchange.
 *
 * mtp_lm_head_shard_partial -- mtp_lm_head_argmax over one shard.
 *   shard         the shard's rows as a weight [n, k]; n_eff <= n are swept
 *   row_offset    global index of the shard's first row; row_offset + n_eff < 2^31
 *   mask          the GLOBAL mask (token t = row_offset + local row; same layout as
 *                 mtp_lm_head_argmax's)
 *   out_partial   (device) 16-byte aligned [M] x {f32 max logit, i32 global row of the
 *                 maximum (lowest on ties; INT32_MAX when no row of the shard is
 *                 allowed), f32 sum over allowed rows of exp(l - max), 4 bytes unused}
 *   out_logits    (device) bf16 [M, n_eff] of the shard, or NULL
 * An empty shard is not an error (no MTP_DEVFLAG_EMPTY_MASK here). Workspace and the
 * other requirements are mtp_lm_head_argmax's.
 *
 * mtp_argmax_merge_partials -- folds n_parts partials per input, laid out
 * [n_parts][M] (rank-major, as an all-gather leaves them), into out_idx (i32 [M]),
 * out_val (f32 [M] or NULL) and out_logprob (f32 [M] or NULL, the log-softmax at the
 * argmax over all shards). Nothing allowed in any shard -> index 0, -inf, -inf and
 * MTP_DEVFLAG_EMPTY_MASK in dev_err (i32 [1] or NULL). The fold order is fixed, so every
 * rank that merges the same partials gets the same bits. 1 <= n_parts <= 65536.
 * ------------------------------------------------------------------------------ */
mtp_status mtp_lm_head_shard_partial(const mtp_weight* shard, int64_t n_eff, int64_t row_offset,
                                     const uint16_t* x, int32_t M, const int32_t* mask,
                                     int64_t mask_words, int64_t mask_stride_words,
                                     void* out_partial, uint16_t* out_logits, int32_t* dev_err,
                                     void* ws, size_t ws_bytes, void* stream);
mtp_status mtp_argmax_merge_partials(const void* partials, int32_t n_parts, int32_t M,
                                     int32_t* out_idx, float* out_val, float* out_logprob,
                                     int32_t* dev_err, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_prefill_kv -- the drafter-context prefill: the drafter's K/V cache rows for R
 * prompt rows, written as E4M3 codes into a paged cache.
 * Source: [mtp_head.rs] drafter-prefill docs (the drafter's K/V for prompt row i are a
 * pure function of (embed(token_{i+1}), target_hidden_i): fc + k/v projections + norms +
 * RoPE + cache write, no attention) and MtpPrefillScratch (chunked rows, bf16 buffers);
 * [new.rs] KV config (block size 16, FP8 cache with unit K/V scales); [v4_mtp.rs]
 * forward_one step 4 (block = block_table[pos / bs], slot = block * bs + pos % bs).
 * Per row r (all intermediate activations rounded to bf16):
 *   c = [rms(embed[token_ids[r]]) w_norm_embed || rms(hidden[r]) w_norm_hidden]
 *   y = fc . c;  a = y, or, when in_norm is given, a = rms(y) in_norm (the decoder
 *   layer's input norm, the scratch's normed2 buffer);
 *   k = wk . a;  v = wv . a;  k' = NeoX RoPE over each head of hd at
 *   position rope_pos[r] (theta_j = pos * rope_base^(-2j/hd)) of k, or, when k_norm is
 *   given, of bf16(k_head / sqrt(mean(k_head^2) + eps) * k_norm) per head ([new.rs] and
 *   [mtp_head.rs] list the head's per-head k_norm weight; the norm precedes RoPE here);
 *   norm_mode MTP_NORM_ONE_PLUS_W makes every norm weight of the call 1 + w;
 *   p = cache_start + r;  slot = block_table[p / block_size] * block_size + p % block_size
 *   k_cache[(slot * nkv + head) * hd + d] = e4m3_satfinite(k'[head, d] / k_scale), same
 *   for v with v_scale. A row whose block is missing (p / block_size >= n_table) or out of
 *   range is not written and sets MTP_DEVFLAG_BAD_SLOT; a bad token id reads as a zero
 *   embedding row and sets MTP_DEVFLAG_BAD_TOKEN.
 *   embed (device) bf16 [vocab, h]; token_ids, rope_pos (device) i32 [R];
 *   hidden (device) bf16 [R, h]; w_norm_* (device) bf16 [h]; fc (device) bf16 [h, 2h];
 *   wk, wv (device) bf16 [nkv * hd, h]; k_norm (device) bf16 [hd] or NULL;
 *   in_norm (device) bf16 [h] or NULL (16-byte aligned);
 *   block_table (device) i32 [n_table];
 *   k_cache, v_cache (device) u8 [num_blocks, block_size, nkv, hd], written in place;
 *   ws (device) mtp_prefill_ws_bytes(min(chunk_rows, R), h, nkv, hd) bytes, 1 KB
 *   aligned, no initial contents required: a small counter header (zeroed by the call
 *   itself with a memset on `stream`), then two lanes of a chunk's concat rows and fc
 *   output and three RoPE tables. Half of that size (one lane, two RoPE tables) is the
 *   minimum (MTP_ERR_WORKSPACE below it); with one lane consecutive chunks take turns on
 *   the same buffers, with two they overlap. The whole call is one kernel on `stream`
 *   (after the memset): every SM takes the chunks' prologue, fc and k/v tiles in one fixed
 *   order from a counter in the header, waiting (bounded) on per-chunk completion counters
 *   there, so the next chunk's tiles fill the SMs the current one leaves idle. The library
 *   creates no streams or events; the call can be captured in a CUDA graph. Calls that
 *   share a workspace must not overlap.
 * Rows run in chunks of chunk_rows (the GEMMs' M). Requires h % 256 == 0, h <= 12288,
 * hd in {64, 128, 256}, nkv * hd % 256 == 0, k_scale, v_scale > 0.
 * ------------------------------------------------------------------------------ */
size_t mtp_prefill_ws_bytes(int64_t chunk_rows, int32_t h, int32_t nkv, int32_t hd);
mtp_status mtp_prefill_kv(const uint16_t* embed, int64_t vocab, const int32_t* token_ids,
                          const uint16_t* hidden, int64_t R, int32_t h,
                          const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden, float eps,
                          int32_t norm_mode, const uint16_t* fc, const uint16_t* wk,
                          const uint16_t* wv, const uint16_t* k_norm, const uint16_t* in_norm,
                          int32_t nkv, int32_t hd, float rope_base, const int32_t* rope_pos,
                          int64_t cache_start, const int32_t* block_table, int64_t n_table,
                          int32_t block_size, uint8_t* k_cache, uint8_t* v_cache,
                          int64_t num_blocks, float k_scale, float v_scale, int64_t chunk_rows,
                          void* ws, size_t ws_bytes, int32_t* dev_err, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_paged_decode_attn -- single-token decode attention of the drafter over its paged
 * E4M3 KV cache (the cache mtp_prefill_kv writes).
 * Source: [new.rs] MtpHead::new (one attention layer with its own paged KV cache, block
 * size 16, FP8 cache fed unit K/V scales by default, a single-token decode-attention
 * kernel for that FP8 cache); [mtp_head.rs] module docs (attention follows fc);
 * [v4_mtp.rs] forward_one step 4 (cache row p at block_table[p / bs] * bs + p % bs).
 * The pages print no formula; this is the standard one, per query head i with kv head
 * g = i / (nq / nkv), over the sequence's cache rows p = 0 .. seq_len - 1:
 *   s_p = scale * sum_d q[i, d] k_scale e4m3(k_cache[(slot(p) * nkv + g) * hd + d])
 *   out[i, d] = bf16(sum_p softmax(s)_p v_scale e4m3(v_cache[(slot(p) * nkv + g) * hd + d]))
 * (fp32 sums and softmax; the tensor cores take q as f16 scaled per head by a power of two
 * -- exact -- and the weights exp(s_p - max) in (0, 1] rounded to f16, the same rounded
 * weights in the denominator). A row whose block is missing (p / block_size >= n_table) or
 * out of range is skipped and sets MTP_DEVFLAG_BAD_SLOT; no readable row -> zeros.
 *   q (device) bf16 [nq, hd]; k_cache, v_cache (device) u8 [num_blocks, block_size, nkv,
 *   hd], 16-byte aligned; block_table (device) i32 [n_table]; out (device) bf16 [nq, hd];
 *   dev_err i32 [1] or NULL; ws (device) >= mtp_paged_decode_attn_ws_bytes(nq, hd,
 *   seq_len) bytes, 16-byte aligned (per-piece partial sums; no initial contents).
 * Requires hd in {64, 128, 256}, nq % nkv == 0, nq / nkv <= 16, seq_len <= 2,097,152
 * (MTP_ERR_UNSUPPORTED otherwise), scale >= 0 (the usual choice is 1 / sqrt(hd)),
 * k_scale, v_scale > 0. Two kernels on `stream`: CTAs of one kv head over a contiguous
 * range of cache rows (as many as the SMs hold at once; every K and V row read once),
 * then a merge per query head in a fixed order.
 * ------------------------------------------------------------------------------ */
size_t mtp_paged_decode_attn_ws_bytes(int32_t nq, int32_t hd, int64_t seq_len);
mtp_status mtp_paged_decode_attn(const uint16_t* q, int32_t nq, int32_t nkv, int32_t hd,
                                 const uint8_t* k_cache, const uint8_t* v_cache,
                                 const int32_t* block_table, int64_t n_table, int32_t block_size,
                                 int64_t num_blocks, int64_t seq_len, float k_scale, float v_scale,
                                 float scale, uint16_t* out, int32_t* dev_err, void* ws,
                                 size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * Stage checks of the prefill, each through the code the prefill itself runs:
 * mtp_debug_gemm_bf16: C = bf16(A . B^T), A bf16 [M, K], B bf16 [N, K], C bf16 [M, N]
 *   (the tcgen05 GEMM); requires N % 256 == 0, K % 64 == 0, 16-byte aligned pointers.
 * mtp_debug_kv_write: already-rotated bf16 k'[R, nkv*hd] and v[R, nkv*hd] -> E4M3 codes
 *   at the paged slots of cache rows cache_start + r (the GEMM epilogue's encode and
 *   slot code).
 * ------------------------------------------------------------------------------ */
mtp_status mtp_debug_gemm_bf16(const uint16_t* A, const uint16_t* B, uint16_t* C, int32_t M,
                               int32_t N, int32_t K, void* stream);
mtp_status mtp_debug_kv_write(const uint16_t* k_rot, const uint16_t* v, int64_t R, int32_t nkv,
                              int32_t hd, int64_t cache_start, const int32_t* block_table,
                              int64_t n_table, int32_t block_size, int64_t num_blocks,
                              uint8_t* k_cache, uint8_t* v_cache, float k_scale, float v_scale,
                              int32_t* dev_err, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_lm_head_argmax_noalloc -- mtp_lm_head_argmax without a workspace argument.
 * The pages have no counterpart: this entry point exists for callers that cannot
 * allocate device memory when they run a draft (a plugin inside another framework's
 * memory pool, an engine that reserves all free memory for its KV cache at start-up,
 * code that must not risk the device synchronisation cudaMalloc/cudaFree can cause).
 * Inputs and outputs are the caller's, exactly as for mtp_lm_head_argmax; the scratch
 * is a static device array inside the library, mtp_noalloc_scratch_bytes() bytes
 * (983,296: a 256-byte header, 16-byte partials of up to 1,024 CTAs x 32 input rows and
 * 448 KB for x in the form the quantized tables' sweeps read it) held on every GPU that
 * loads the library until the process exits. Calls whose mtp_lm_head_ws_bytes exceeds
 * it return MTP_ERR_WORKSPACE: BF16 tables run at every M up to 32; FP8 tables at every
 * M up to 32 with k <= 7,152; NVFP4 tables with up to 16 inputs and k <= 8,448, with
 * 17-32 inputs and k <= 4,096.
 *  - The first call made with a device current looks up that array's device address.
 *    Under the CUDA runtime's lazy module loading (the default since CUDA 12.2) that
 *    look-up is also when the array is committed on the device, so make the first call
 *    on each device before reserving the device's free memory, and before any stream
 *    capture; later calls change no device memory outside their inputs and outputs.
 *  - The array is zero when its module loads, and each call leaves its counter zero
 *    again. All calls on a device share the array: calls that overlap on the GPU race
 *    and must be serialised by the caller.
 *  - Arguments are checked as mtp_lm_head_argmax checks them, before anything else;
 *    then MTP_ERR_WORKSPACE if the call would need more scratch than the array holds.
 *    It never allocates.
 * ------------------------------------------------------------------------------ */
size_t mtp_noalloc_scratch_bytes(void);
mtp_status mtp_lm_head_argmax_noalloc(const mtp_weight* head, int64_t n_eff, const uint16_t* x,
                                      int32_t M, const int32_t* mask, int64_t mask_words,
                                      int64_t mask_stride_words, int32_t* out_idx, float* out_val,
                                      uint16_t* out_logits, int32_t* dev_err, void* stream);

/* ---------------------------------------------------------------------------------
 * mtp_debug_wait_timeout -- self-check of the bounded waits every pipelined kernel here
 * uses (the pages have no counterpart: it tests this library's failure handling). One
 * small kernel waits, through the same helpers, on something that never happens --
 * which 0: an mbarrier phase no thread completes; which 1: the device u32 *counter
 * reaching 1 (the caller keeps it 0) -- gives up after limit_cycles SM clock cycles
 * (1 .. 4e9; the pipelines use about one second), ORs MTP_DEVFLAG_TIMEOUT into *dev_err
 * (device i32, required) and ends; the context stays usable.
 * ------------------------------------------------------------------------------ */
mtp_status mtp_debug_wait_timeout(int32_t which, int64_t limit_cycles, const uint32_t* counter,
                                  int32_t* dev_err, void* stream);

/* Maps a device error word read back by the caller to a status: MTP_OK, or
 * MTP_WARN_EMPTY_MASK when only the empty-mask bit is set, else MTP_ERR_INVALID_ARG. */
mtp_status mtp_devflags_status(int32_t dev_err_value);

/* ---------------------------------------------------------------------------------
 * Exhaustive-check entry points: the device E4M3 / E2M1 encoders used by the
 * quantizers and the KV write, one f32 in -> one code out (E2M1 in the low nibble).
 *   in (device) f32 [n]; out (device) u8 [n]
 * ------------------------------------------------------------------------------ */
mtp_status mtp_debug_encode_e4m3(const float* in, int64_t n, uint8_t* out, void* stream);
mtp_status mtp_debug_encode_e2m1(const float* in, int64_t n, uint8_t* out, void* stream);

const char* mtp_status_str(mtp_status s);
int32_t mtp_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MTP_H */
