// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mtp {

// One draft-head GEMV sweep over rows [0, n) of a [*, k] table, with x staged per CTA.
// mode 0: fused argmax (+ optional logits); mode 1: combiner (x built from the
// embedding row and target hidden, output y = bf16(W . c)).
struct SweepParams {
    const uint8_t* w;            // table bytes, rows packed at `row_bytes`
    const float* row_scale;      // FP8: f32[n]
    const uint8_t* block_scale;  // NVFP4: e4m3[n, k/16]
    const float* global_scale;   // NVFP4: f32[1] on the device
    int64_t n;                   // rows swept
    int64_t k;                   // reduction length (table columns)
    int64_t row_bytes;
    int32_t M;                   // input rows (1..16)
    int32_t kpad;                // staged-x row stride in elements
    // mode 0 input
    const uint16_t* x;           // bf16 [M, k]
    // mode 1 inputs (k == 2h)
    const uint16_t* embed;
    int64_t vocab;
    const int32_t* tokens;       // [M]
    const uint16_t* hidden;      // bf16 [M, h]
    const uint16_t* w_norm_embed;
    const uint16_t* w_norm_hidden;
    float eps;
    int32_t h;
    int32_t norm_mode;           // 0: weights w, 1: weights 1 + w
    // grammar mask (mode 0)
    const int32_t* mask;
    int64_t mask_words;
    int64_t mask_stride;
    // outputs
    int32_t* out_idx;
    float* out_val;
    uint16_t* out_logits;        // bf16 [M, n] or null
    float* out_logprob;          // f32 [M] top-1 log-probability, or null
    void* out_partial;           // vocab shard: 16-byte (max, row, sum exp) per input, or null
    int64_t row_offset;          // vocab shard: global index of the table's first row
    uint16_t* x16;               // many inputs, quantized tables: x as those sweeps read it
                                 // (FP8: E4M3 hi / lo planes; NVFP4: f16 [M, k]), scaled per row
    int32_t* xexp;               // its per-row power of two [M]
    uint16_t* out_y;             // mode 1: bf16 [M, n]
    int32_t* dev_err;
    // workspace (mode 0)
    uint32_t* ticket;
    void* partials;
    int64_t num_tiles;
    int64_t scale_pitch;         // NVFP4: bytes between block-scale rows
    int32_t stages;              // ring depth (set by the launcher)
    int32_t stage_bytes;
    int32_t segs;                // 128-byte row segments per stage
    int32_t stages_per_tile;
};

struct SweepLaunch {
    int grid;
    int smem_bytes;
};

// Folds n_parts 16-byte shard partials per input (rank-major [n_parts][M]) into the
// argmax, its value and the top-1 log-probability; one warp per input.
cudaError_t merge_partials_launch(const void* parts, int n_parts, int M, int32_t* out_idx,
                                  float* out_val, float* out_logprob, int32_t* dev_err,
                                  cudaStream_t s);

// Picks the kernel instance and grid; returns cudaErrorInvalidValue if the staged
// input does not fit in shared memory.
cudaError_t sweep_launch(const SweepParams& p, int fmt, int mode, cudaStream_t s,
                         SweepLaunch* info);
// Shared memory the sweep for these inputs needs (masked: the gathered sweep, M <= 8).
size_t sweep_smem_bytes(int M, int64_t k, int fmt, int* kpad_out, int mode, bool masked = false);
// Workspace bytes the many-input argmax sweeps need for x in their own form (FP8 tables
// from 7 inputs: two E4M3 planes; NVFP4 from 9: an f16 copy) plus 1 KB of per-input
// exponents: 0 for BF16 and for fewer inputs.
size_t sweep_x16_bytes(int M, int64_t k, int fmt);
int sweep_max_grid();

// Copies `bytes` (a multiple of 16) from device-reachable host memory into device memory
// with a programmatic-dependent-launch kernel (loads before, stores after waiting for the
// previous grid).
cudaError_t fetch_x_launch(const void* src, void* dst, size_t bytes, cudaStream_t s);

// Quantizers.
cudaError_t quant_fp8_launch(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                             float* row_scale, cudaStream_t s);
cudaError_t quant_nvfp4_launch(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                               uint8_t* block_scale, float* global_scale, uint32_t* ws,
                               cudaStream_t s);
int quant_nvfp4_max_grid();
int64_t nvfp4_scale_pitch(int64_t k);

// Drafter-context prefill (prefill.cu).
struct PrefillArgs {
    const uint16_t* embed;
    int64_t vocab;
    const int32_t* tokens;
    const uint16_t* hidden;
    int64_t R;
    int32_t h;
    const uint16_t* w_norm_embed;
    const uint16_t* w_norm_hidden;
    float eps;
    int32_t norm_mode;
    const uint16_t* fc;
    const uint16_t* wk;
    const uint16_t* wv;
    const uint16_t* k_norm;  // [hd] or null: per-head RMSNorm of k before RoPE
    const uint16_t* in_norm;  // [h] or null: RMSNorm of the fc output before k and v
    int32_t nkv, hd;
    double rope_base;
    const int32_t* rope_pos;
    int64_t cache_start;
    const int32_t* block_table;
    int64_t n_table;
    int32_t block_size;
    uint8_t* k_cache;
    uint8_t* v_cache;
    int64_t num_blocks;
    float k_scale, v_scale;
    int64_t chunk_rows;
    void* ws;
    size_t ws_bytes;
    int32_t* dev_err;
};
// Workspace of the prefill: a counter header, then one or two lanes of a chunk's concat
// rows and fc output rows, and one more RoPE table than lanes. prefill_lane_bytes is the
// one-lane minimum, prefill_ws_bytes the two-lane size (consecutive chunks overlap).
size_t prefill_lane_bytes(int64_t chunk_rows, int32_t h, int32_t nkv, int32_t hd);
size_t prefill_ws_bytes(int64_t chunk_rows, int32_t h, int32_t nkv, int32_t hd);
int prefill_max_hidden();
cudaError_t prefill_launch(const PrefillArgs& a, cudaStream_t s);
cudaError_t gemm_bf16_launch(const uint16_t* A, const uint16_t* B, uint16_t* C, int M, int N,
                             int K, int32_t* dev_err, cudaStream_t s);
cudaError_t kv_write_launch(const uint16_t* k_rot, const uint16_t* v, int64_t R, int nkv, int hd,
                            int64_t cache_start, const int32_t* block_table, int64_t n_table,
                            int block_size, int64_t num_blocks, uint8_t* k_cache, uint8_t* v_cache,
                            float k_scale, float v_scale, int32_t* dev_err, cudaStream_t s);
int gemm_tile_n();
int gemm_tile_k();

// One whole draft step for a small BF16 head in one cluster launch (draft.cu).
int draft_step_max_m();
int draft_step_max_h();
cudaError_t draft_step_launch(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                              const uint16_t* hidden, int M, int h, const uint16_t* w_ne,
                              const uint16_t* w_nh, float eps, int norm_mode, const uint16_t* fc,
                              const uint16_t* head, int64_t n, const int32_t* mask,
                              int64_t mask_words, int64_t mask_stride, uint16_t* out_y,
                              int32_t* out_idx, float* out_val, int32_t* dev_err, cudaStream_t s);

// Single-token paged decode attention over the E4M3 KV cache (attn.cu).
int attn_max_group();
size_t attn_ws_bytes(int nq, int hd, int64_t seq_len);
cudaError_t attn_launch(const uint16_t* q, int nq, int nkv, int hd, const uint8_t* k_cache,
                        const uint8_t* v_cache, const int32_t* block_table, int64_t n_table,
                        int block_size, int64_t num_blocks, int64_t seq_len, float k_scale,
                        float v_scale, float scale, uint16_t* out, int32_t* dev_err, void* ws,
                        cudaStream_t s);

// Self-check of the bounded waits (selfcheck.cu): which 0 waits on an mbarrier phase that
// nothing completes, 1 on a global counter (device u32, kept at 0 by the caller) that
// nothing increments; either gives up after limit_cycles and sets DEVFLAG_TIMEOUT.
cudaError_t wait_timeout_launch(int which, long long limit_cycles, const uint32_t* counter,
                                int32_t* dev_err, cudaStream_t s);

// Encoders exposed for exhaustive checks.
cudaError_t debug_encode_launch(const float* in, int64_t n, uint8_t* out, int which,
                                cudaStream_t s);

}  // namespace mtp
