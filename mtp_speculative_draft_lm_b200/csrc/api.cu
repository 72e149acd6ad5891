// C ABI (include/mtp.h): host-side argument validation, then the kernel launches.
// Nothing here computes the method; every arithmetic step runs in the kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mtp.h"
#include "kernels.h"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool finite_pos(float v) { return v > 0.f && v < 3.0e38f; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

mtp_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MTP_OK;
    if (e == cudaErrorInvalidValue) return MTP_ERR_UNSUPPORTED;
    return MTP_ERR_CUDA;
}

// Checks a weight descriptor: format, sizes, pointer presence and alignment.
mtp_status check_weight(const mtp_weight* w) {
    if (!w || w->reserved != 0 || w->n < 1 || w->k < 1 || !w->data) return MTP_ERR_INVALID_ARG;
    if (!aligned(w->data, 16)) return MTP_ERR_INVALID_ARG;
    switch (w->fmt) {
        case MTP_FMT_BF16:
            if (w->k % 8 || w->row_scale || w->block_scale || w->global_scale)
                return MTP_ERR_INVALID_ARG;
            return MTP_OK;
        case MTP_FMT_FP8_ROW:
            if (w->k % 16 || !w->row_scale || w->block_scale || w->global_scale)
                return MTP_ERR_INVALID_ARG;
            if (!aligned(w->row_scale, 4)) return MTP_ERR_INVALID_ARG;
            return MTP_OK;
        case MTP_FMT_NVFP4:
            if (w->k % 32 || w->row_scale || !w->block_scale || !w->global_scale)
                return MTP_ERR_INVALID_ARG;
            if (!aligned(w->block_scale, 16) || !aligned(w->global_scale, 4))
                return MTP_ERR_INVALID_ARG;
            return MTP_OK;
        default:
            return MTP_ERR_INVALID_ARG;
    }
}

}  // namespace

extern "C" int64_t mtp_nvfp4_scale_pitch(int64_t k) { return mtp::nvfp4_scale_pitch(k); }

namespace {

int64_t row_bytes(const mtp_weight* w) {
    return w->fmt == MTP_FMT_BF16 ? w->k * 2 : w->fmt == MTP_FMT_FP8_ROW ? w->k : w->k / 2;
}

constexpr size_t kTicketBytes = 256;
constexpr size_t kPartialBytes = 16;  // {float value, int32 index, float sum of exp, pad}
constexpr int kMaxM = 32;       // inputs per sweep
constexpr int kMaxMCombine = 16;
constexpr int kPartSlots = 32;   // partials per CTA

}  // namespace

extern "C" {

int32_t mtp_abi_version(void) { return MTP_ABI_VERSION; }

const char* mtp_status_str(mtp_status s) {
    switch (s) {
        case MTP_OK: return "ok";
        case MTP_ERR_INVALID_ARG: return "invalid argument";
        case MTP_ERR_UNSUPPORTED: return "unsupported shape or size";
        case MTP_ERR_WORKSPACE: return "workspace missing or too small";
        case MTP_ERR_CUDA: return "CUDA error";
        case MTP_WARN_EMPTY_MASK: return "a grammar mask allowed no token";
    }
    return "unknown status";
}

mtp_status mtp_devflags_status(int32_t v) {
    if (v == 0) return MTP_OK;
    if (v == MTP_DEVFLAG_EMPTY_MASK) return MTP_WARN_EMPTY_MASK;
    return MTP_ERR_INVALID_ARG;
}

mtp_status mtp_quantize_fp8(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                            float* row_scale, void* stream) {
    if (!w || !codes || !row_scale || n < 1 || k < 16 || k % 16) return MTP_ERR_INVALID_ARG;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(row_scale, 4))
        return MTP_ERR_INVALID_ARG;
    return from_cuda(mtp::quant_fp8_launch(w, n, k, codes, row_scale, as_stream(stream)));
}

size_t mtp_quantize_nvfp4_ws_bytes(int64_t n, int64_t k) {
    (void)n;
    (void)k;
    return kTicketBytes + sizeof(float) * (size_t)mtp::quant_nvfp4_max_grid();
}

mtp_status mtp_quantize_nvfp4(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                              uint8_t* block_scale, float* global_scale, void* ws,
                              size_t ws_bytes, void* stream) {
    if (!w || !codes || !block_scale || !global_scale || n < 1 || k < 32 || k % 32)
        return MTP_ERR_INVALID_ARG;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(block_scale, 16) ||
        !aligned(global_scale, 4))
        return MTP_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, 16) || ws_bytes < mtp_quantize_nvfp4_ws_bytes(n, k))
        return MTP_ERR_WORKSPACE;
    return from_cuda(mtp::quant_nvfp4_launch(w, n, k, codes, block_scale, global_scale,
                                             static_cast<uint32_t*>(ws), as_stream(stream)));
}

mtp_status mtp_combine(const uint16_t* embed, int64_t vocab, const int32_t* token_ids,
                       const uint16_t* hidden, int32_t M, int32_t h,
                       const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden,
                       float eps, int32_t norm_mode, const mtp_weight* fc, uint16_t* out,
                       int32_t* dev_err, void* stream) {
    if (!embed || !token_ids || !hidden || !w_norm_embed || !w_norm_hidden || !out)
        return MTP_ERR_INVALID_ARG;
    if (vocab < 1 || h < 16 || h % 16 || !(eps >= 0.f) ||
        (norm_mode != MTP_NORM_W && norm_mode != MTP_NORM_ONE_PLUS_W))
        return MTP_ERR_INVALID_ARG;
    if (M < 1 || M > kMaxMCombine) return MTP_ERR_UNSUPPORTED;
    mtp_status st = check_weight(fc);
    if (st != MTP_OK) return st;
    if (fc->n != h || fc->k != 2 * (int64_t)h) return MTP_ERR_INVALID_ARG;
    if (row_bytes(fc) % 128) return MTP_ERR_UNSUPPORTED;
    if (!aligned(embed, 16) || !aligned(hidden, 16) || !aligned(out, 16) ||
        !aligned(w_norm_embed, 4) || !aligned(w_norm_hidden, 4) || !aligned(token_ids, 4) ||
        !aligned(dev_err, 4))
        return MTP_ERR_INVALID_ARG;
    if (mtp::sweep_smem_bytes(M, fc->k, fc->fmt, nullptr, 1) > 227 * 1024) return MTP_ERR_UNSUPPORTED;
    mtp::SweepParams p{};
    p.w = static_cast<const uint8_t*>(fc->data);
    p.row_scale = fc->row_scale;
    p.block_scale = fc->block_scale;
    p.global_scale = fc->global_scale;
    p.n = fc->n;
    p.k = fc->k;
    p.row_bytes = row_bytes(fc);
    p.M = M;
    p.embed = embed;
    p.vocab = vocab;
    p.tokens = token_ids;
    p.hidden = hidden;
    p.w_norm_embed = w_norm_embed;
    p.w_norm_hidden = w_norm_hidden;
    p.eps = eps;
    p.h = h;
    p.norm_mode = norm_mode;
    p.out_y = out;
    p.dev_err = dev_err;
    p.num_tiles = (fc->n + 15) / 16;
    p.scale_pitch = mtp::nvfp4_scale_pitch(fc->k);
    return from_cuda(mtp::sweep_launch(p, fc->fmt, 1, as_stream(stream), nullptr));
}

size_t mtp_lm_head_ws_bytes(const mtp_weight* head, int64_t n_eff, int32_t M) {
    (void)n_eff;
    const size_t base = kTicketBytes + kPartialBytes * kPartSlots * (size_t)mtp::sweep_max_grid();
    if (!head || M < 1 || M > kMaxM) return base;
    return base + mtp::sweep_x16_bytes(M, head->k, head->fmt);
}

namespace {

mtp_status lm_head_impl(const mtp_weight* head, int64_t n_eff, const uint16_t* x, int32_t M,
                        const int32_t* mask, int64_t mask_words, int64_t mask_stride_words,
                        int32_t* out_idx, float* out_val, float* out_logprob,
                        uint16_t* out_logits, int32_t* dev_err, void* ws, size_t ws_bytes,
                        void* stream, void* out_partial = nullptr, int64_t row_offset = 0) {
    mtp_status st = check_weight(head);
    if (st != MTP_OK) return st;
    if (!x || (!out_idx && !out_partial) || n_eff < 1 || n_eff > head->n) return MTP_ERR_INVALID_ARG;
    if (row_offset < 0 || row_offset + n_eff > (int64_t)INT32_MAX) return MTP_ERR_INVALID_ARG;
    if (!aligned(out_partial, 16)) return MTP_ERR_INVALID_ARG;
    if (n_eff > (int64_t)INT32_MAX || row_bytes(head) % 128) return MTP_ERR_UNSUPPORTED;
    if (M < 1 || M > kMaxM) return MTP_ERR_UNSUPPORTED;
    if (mask && (mask_words < 1 || mask_stride_words < 0)) return MTP_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out_idx, 4) || !aligned(out_val, 4) ||
        !aligned(out_logprob, 4) ||
        !aligned(out_logits, 2) || !aligned(dev_err, 4) || !aligned(mask, 4))
        return MTP_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, 16) || ws_bytes < mtp_lm_head_ws_bytes(head, n_eff, M))
        return MTP_ERR_WORKSPACE;
    if (mtp::sweep_smem_bytes(M, head->k, head->fmt, nullptr, 0, mask != nullptr) > 227 * 1024)
        return MTP_ERR_UNSUPPORTED;
    mtp::SweepParams p{};
    p.w = static_cast<const uint8_t*>(head->data);
    p.row_scale = head->row_scale;
    p.block_scale = head->block_scale;
    p.global_scale = head->global_scale;
    p.n = n_eff;
    p.k = head->k;
    p.row_bytes = row_bytes(head);
    p.M = M;
    p.x = x;
    p.mask = mask;
    p.mask_words = mask ? mask_words : 0;
    p.mask_stride = mask ? mask_stride_words : 0;
    p.out_idx = out_idx;
    p.out_val = out_val;
    p.out_logits = out_logits;
    p.out_logprob = out_logprob;
    p.out_partial = out_partial;
    p.row_offset = row_offset;
    p.dev_err = dev_err;
    p.ticket = static_cast<uint32_t*>(ws);
    p.partials = static_cast<uint8_t*>(ws) + kTicketBytes;
    if (mtp::sweep_x16_bytes(M, head->k, head->fmt)) {  // x as the many-input sweeps read it
        uint8_t* xb = static_cast<uint8_t*>(ws) + kTicketBytes + kPartialBytes * kPartSlots *
                                                                   (size_t)mtp::sweep_max_grid();
        p.x16 = reinterpret_cast<uint16_t*>(xb);
        p.xexp = reinterpret_cast<int32_t*>(xb + mtp::sweep_x16_bytes(M, head->k, head->fmt) - 1024);
    }
    p.num_tiles = (n_eff + 15) / 16;
    p.scale_pitch = mtp::nvfp4_scale_pitch(head->k);
    return from_cuda(mtp::sweep_launch(p, head->fmt, 0, as_stream(stream), nullptr));
}

}  // namespace

mtp_status mtp_lm_head_argmax(const mtp_weight* head, int64_t n_eff, const uint16_t* x,
                              int32_t M, const int32_t* mask, int64_t mask_words,
                              int64_t mask_stride_words, int32_t* out_idx, float* out_val,
                              uint16_t* out_logits, int32_t* dev_err, void* ws,
                              size_t ws_bytes, void* stream) {
    return lm_head_impl(head, n_eff, x, M, mask, mask_words, mask_stride_words, out_idx, out_val,
                        nullptr, out_logits, dev_err, ws, ws_bytes, stream);
}

size_t mtp_lm_head_host_ws_bytes(const mtp_weight* head, int64_t n_eff, int32_t M) {
    const size_t base = mtp_lm_head_ws_bytes(head, n_eff, M);
    if (!head || M < 1 || M > kMaxM || head->k < 1) return base;
    return base + (((size_t)M * (size_t)head->k * 2 + 15) & ~(size_t)15);
}

namespace {

// The device address of pinned (page-locked) host memory, or null if `p` is not pinned.
void* pinned_device_ptr(const void* p) {
    cudaPointerAttributes a{};
    if (!p || cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // clear the error a non-registered pointer leaves behind
        return nullptr;
    }
    if (a.type != cudaMemoryTypeHost || !a.devicePointer) return nullptr;
    return a.devicePointer;
}

}  // namespace

mtp_status mtp_lm_head_argmax_host(const mtp_weight* head, int64_t n_eff, const uint16_t* x_host,
                                   int32_t M, const int32_t* mask, int64_t mask_words,
                                   int64_t mask_stride_words, int32_t* out_host, int32_t* dev_err,
                                   void* ws, size_t ws_bytes, void* stream) {
    mtp_status st = check_weight(head);
    if (st != MTP_OK) return st;
    if (!x_host || !out_host) return MTP_ERR_INVALID_ARG;
    if (M < 1 || M > kMaxM) return MTP_ERR_UNSUPPORTED;
    if (!aligned(x_host, 16) || !aligned(out_host, 4) || (head->k * 2) % 16)
        return MTP_ERR_INVALID_ARG;
    const size_t base = mtp_lm_head_ws_bytes(head, n_eff, M);
    if (!ws || !aligned(ws, 16) || ws_bytes < mtp_lm_head_host_ws_bytes(head, n_eff, M))
        return MTP_ERR_WORKSPACE;
    void* xd = pinned_device_ptr(x_host);
    void* od = pinned_device_ptr(out_host);
    if (!xd || !od) return MTP_ERR_INVALID_ARG;  // both must be pinned host memory
    uint16_t* x_dev = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + base);
    const size_t xbytes = (size_t)M * (size_t)head->k * 2;
    cudaError_t e = mtp::fetch_x_launch(xd, x_dev, xbytes, as_stream(stream));
    if (e != cudaSuccess) return from_cuda(e);
    int32_t* idx = static_cast<int32_t*>(od);
    float* val = reinterpret_cast<float*>(idx + M);
    return lm_head_impl(head, n_eff, x_dev, M, mask, mask_words, mask_stride_words, idx, val,
                        nullptr, nullptr, dev_err, ws, base, stream);
}

mtp_status mtp_lm_head_shard_partial(const mtp_weight* shard, int64_t n_eff, int64_t row_offset,
                                     const uint16_t* x, int32_t M, const int32_t* mask,
                                     int64_t mask_words, int64_t mask_stride_words,
                                     void* out_partial, uint16_t* out_logits, int32_t* dev_err,
                                     void* ws, size_t ws_bytes, void* stream) {
    if (!out_partial) return MTP_ERR_INVALID_ARG;
    return lm_head_impl(shard, n_eff, x, M, mask, mask_words, mask_stride_words, nullptr, nullptr,
                        nullptr, out_logits, dev_err, ws, ws_bytes, stream, out_partial,
                        row_offset);
}

mtp_status mtp_argmax_merge_partials(const void* partials, int32_t n_parts, int32_t M,
                                     int32_t* out_idx, float* out_val, float* out_logprob,
                                     int32_t* dev_err, void* stream) {
    if (!partials || !out_idx || n_parts < 1 || n_parts > 65536) return MTP_ERR_INVALID_ARG;
    if (M < 1 || M > kMaxM) return MTP_ERR_UNSUPPORTED;
    if (!aligned(partials, 16) || !aligned(out_idx, 4) || !aligned(out_val, 4) ||
        !aligned(out_logprob, 4) || !aligned(dev_err, 4))
        return MTP_ERR_INVALID_ARG;
    return from_cuda(mtp::merge_partials_launch(partials, n_parts, M, out_idx, out_val, out_logprob,
                                                dev_err, as_stream(stream)));
}

mtp_status mtp_lm_head_argmax_lp(const mtp_weight* head, int64_t n_eff, const uint16_t* x,
                                 int32_t M, const int32_t* mask, int64_t mask_words,
                                 int64_t mask_stride_words, int32_t* out_idx, float* out_val,
                                 float* out_logprob, uint16_t* out_logits, int32_t* dev_err,
                                 void* ws, size_t ws_bytes, void* stream) {
    if (!out_logprob) return MTP_ERR_INVALID_ARG;
    return lm_head_impl(head, n_eff, x, M, mask, mask_words, mask_stride_words, out_idx, out_val,
                        out_logprob, out_logits, dev_err, ws, ws_bytes, stream);
}

mtp_status mtp_draft_step(const uint16_t* embed, int64_t vocab, const int32_t* token_ids,
                          const uint16_t* hidden, int32_t M, int32_t h,
                          const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden, float eps,
                          int32_t norm_mode, const uint16_t* fc, const uint16_t* head, int64_t n_eff,
                          const int32_t* mask, int64_t mask_words, int64_t mask_stride_words,
                          uint16_t* out_y, int32_t* out_idx, float* out_val, int32_t* dev_err,
                          void* stream) {
    if (!embed || !token_ids || !hidden || !w_norm_embed || !w_norm_hidden || !fc || !head ||
        !out_idx)
        return MTP_ERR_INVALID_ARG;
    if (vocab < 1 || n_eff < 1 || n_eff > (int64_t)INT32_MAX || h < 8 || h % 8 || !(eps >= 0.f) ||
        (norm_mode != MTP_NORM_W && norm_mode != MTP_NORM_ONE_PLUS_W))
        return MTP_ERR_INVALID_ARG;
    if (mask && (mask_words < 1 || mask_stride_words < 0)) return MTP_ERR_INVALID_ARG;
    if (M < 1 || M > mtp::draft_step_max_m() || h > mtp::draft_step_max_h()) return MTP_ERR_UNSUPPORTED;
    if (!aligned(embed, 16) || !aligned(hidden, 16) || !aligned(fc, 16) || !aligned(head, 16) ||
        !aligned(w_norm_embed, 2) || !aligned(w_norm_hidden, 2) || !aligned(token_ids, 4) ||
        !aligned(out_y, 2) || !aligned(out_idx, 4) || !aligned(out_val, 4) || !aligned(mask, 4) ||
        !aligned(dev_err, 4))
        return MTP_ERR_INVALID_ARG;
    if (out_y) {  // each CTA writes its slice of y while others may still read hidden
        const uintptr_t y0 = reinterpret_cast<uintptr_t>(out_y), x0 = reinterpret_cast<uintptr_t>(hidden);
        const uintptr_t bytes = (uintptr_t)M * (uintptr_t)h * 2u;
        if (y0 < x0 + bytes && x0 < y0 + bytes) return MTP_ERR_INVALID_ARG;
    }
    return from_cuda(mtp::draft_step_launch(embed, vocab, token_ids, hidden, M, h, w_norm_embed,
                                            w_norm_hidden, eps, norm_mode, fc, head, n_eff, mask,
                                            mask_words,
                                            mask_stride_words, out_y, out_idx, out_val, dev_err,
                                            as_stream(stream)));
}

size_t mtp_paged_decode_attn_ws_bytes(int32_t nq, int32_t hd, int64_t seq_len) {
    if (nq < 1 || hd < 1 || seq_len < 1) return 0;
    return mtp::attn_ws_bytes(nq, hd, seq_len);
}

mtp_status mtp_paged_decode_attn(const uint16_t* q, int32_t nq, int32_t nkv, int32_t hd,
                                 const uint8_t* k_cache, const uint8_t* v_cache,
                                 const int32_t* block_table, int64_t n_table, int32_t block_size,
                                 int64_t num_blocks, int64_t seq_len, float k_scale, float v_scale,
                                 float scale, uint16_t* out, int32_t* dev_err, void* ws,
                                 size_t ws_bytes, void* stream) {
    if (!q || !k_cache || !v_cache || !block_table || !out) return MTP_ERR_INVALID_ARG;
    if (nq < 1 || nkv < 1 || nq % nkv || n_table < 1 || block_size < 1 || num_blocks < 1 ||
        seq_len < 1 || !finite_pos(k_scale) || !finite_pos(v_scale) || !(scale >= 0.f) ||
        !(scale < 3.0e38f))
        return MTP_ERR_INVALID_ARG;
    if ((hd != 64 && hd != 128 && hd != 256) || nq / nkv > mtp::attn_max_group() ||
        seq_len > (int64_t)8192 * 256)
        return MTP_ERR_UNSUPPORTED;
    if (!aligned(q, 2) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_table, 4) || !aligned(out, 2) || !aligned(dev_err, 4))
        return MTP_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, 16) || ws_bytes < mtp::attn_ws_bytes(nq, hd, seq_len))
        return MTP_ERR_WORKSPACE;
    return from_cuda(mtp::attn_launch(q, nq, nkv, hd, k_cache, v_cache, block_table, n_table,
                                      block_size, num_blocks, seq_len, k_scale, v_scale, scale,
                                      out, dev_err, ws, as_stream(stream)));
}

size_t mtp_prefill_ws_bytes(int64_t chunk_rows, int32_t h, int32_t nkv, int32_t hd) {
    if (chunk_rows < 1 || h < 1 || nkv < 1 || hd < 2) return 0;
    return mtp::prefill_ws_bytes(chunk_rows, h, nkv, hd);
}

mtp_status mtp_prefill_kv(const uint16_t* embed, int64_t vocab, const int32_t* token_ids,
                          const uint16_t* hidden, int64_t R, int32_t h,
                          const uint16_t* w_norm_embed, const uint16_t* w_norm_hidden, float eps,
                          int32_t norm_mode, const uint16_t* fc, const uint16_t* wk,
                          const uint16_t* wv, const uint16_t* k_norm, const uint16_t* in_norm,
                          int32_t nkv, int32_t hd, float rope_base, const int32_t* rope_pos,
                          int64_t cache_start, const int32_t* block_table, int64_t n_table,
                          int32_t block_size, uint8_t* k_cache, uint8_t* v_cache,
                          int64_t num_blocks, float k_scale, float v_scale, int64_t chunk_rows,
                          void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
    if (!embed || !token_ids || !hidden || !w_norm_embed || !w_norm_hidden || !fc || !wk ||
        !wv || !rope_pos || !block_table || !k_cache || !v_cache)
        return MTP_ERR_INVALID_ARG;
    if (vocab < 1 || R < 1 || h < 1 || nkv < 1 || hd < 2 || block_size < 1 || n_table < 1 ||
        num_blocks < 1 || chunk_rows < 1 || !(eps >= 0.f) || !finite_pos(k_scale) ||
        !finite_pos(v_scale) || !(rope_base > 0.f) || cache_start < 0 ||
        (norm_mode != MTP_NORM_W && norm_mode != MTP_NORM_ONE_PLUS_W) || !aligned(k_norm, 2) ||
        !aligned(in_norm, 16))
        return MTP_ERR_INVALID_ARG;
    const int tn = mtp::gemm_tile_n();
    if (h % tn || h > mtp::prefill_max_hidden() || (hd != 64 && hd != 128 && hd != 256) ||
        ((int64_t)nkv * hd) % tn || chunk_rows > (int64_t)1 << 30)
        return MTP_ERR_UNSUPPORTED;
    if (!aligned(embed, 16) || !aligned(hidden, 16) || !aligned(fc, 16) || !aligned(wk, 16) ||
        !aligned(wv, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(w_norm_embed, 2) || !aligned(w_norm_hidden, 2) || !aligned(token_ids, 4) ||
        !aligned(rope_pos, 4) || !aligned(block_table, 4) || !aligned(dev_err, 4))
        return MTP_ERR_INVALID_ARG;
    const int64_t chunk = chunk_rows < R ? chunk_rows : R;
    if (!ws || !aligned(ws, 1024) || ws_bytes < mtp::prefill_lane_bytes(chunk, h, nkv, hd))
        return MTP_ERR_WORKSPACE;
    mtp::PrefillArgs a{};
    a.embed = embed;
    a.vocab = vocab;
    a.tokens = token_ids;
    a.hidden = hidden;
    a.R = R;
    a.h = h;
    a.w_norm_embed = w_norm_embed;
    a.w_norm_hidden = w_norm_hidden;
    a.eps = eps;
    a.norm_mode = norm_mode;
    a.fc = fc;
    a.wk = wk;
    a.wv = wv;
    a.k_norm = k_norm;
    a.in_norm = in_norm;
    a.nkv = nkv;
    a.hd = hd;
    a.rope_base = (double)rope_base;
    a.rope_pos = rope_pos;
    a.cache_start = cache_start;
    a.block_table = block_table;
    a.n_table = n_table;
    a.block_size = block_size;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.num_blocks = num_blocks;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.chunk_rows = chunk;
    a.ws = ws;
    a.ws_bytes = ws_bytes;
    a.dev_err = dev_err;
    return from_cuda(mtp::prefill_launch(a, as_stream(stream)));
}

mtp_status mtp_debug_gemm_bf16(const uint16_t* A, const uint16_t* B, uint16_t* C, int32_t M,
                               int32_t N, int32_t K, void* stream) {
    if (!A || !B || !C || M < 1 || N < 1 || K < 1) return MTP_ERR_INVALID_ARG;
    if (N % mtp::gemm_tile_n() || K % mtp::gemm_tile_k()) return MTP_ERR_UNSUPPORTED;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16)) return MTP_ERR_INVALID_ARG;
    return from_cuda(mtp::gemm_bf16_launch(A, B, C, M, N, K, nullptr, as_stream(stream)));
}

mtp_status mtp_debug_kv_write(const uint16_t* k_rot, const uint16_t* v, int64_t R, int32_t nkv,
                              int32_t hd, int64_t cache_start, const int32_t* block_table,
                              int64_t n_table, int32_t block_size, int64_t num_blocks,
                              uint8_t* k_cache, uint8_t* v_cache, float k_scale, float v_scale,
                              int32_t* dev_err, void* stream) {
    if (!k_rot || !v || !block_table || !k_cache || !v_cache || R < 1 || nkv < 1 || hd < 32 ||
        hd % 32 || block_size < 1 || n_table < 1 || num_blocks < 1 || cache_start < 0 ||
        !finite_pos(k_scale) || !finite_pos(v_scale))
        return MTP_ERR_INVALID_ARG;
    if (!aligned(k_rot, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_table, 4) || !aligned(dev_err, 4))
        return MTP_ERR_INVALID_ARG;
    return from_cuda(mtp::kv_write_launch(k_rot, v, R, nkv, hd, cache_start, block_table, n_table,
                                          block_size, num_blocks, k_cache, v_cache, k_scale,
                                          v_scale, dev_err, as_stream(stream)));
}

mtp_status mtp_debug_wait_timeout(int32_t which, int64_t limit_cycles, const uint32_t* counter,
                                  int32_t* dev_err, void* stream) {
    if ((which != 0 && which != 1) || limit_cycles < 1 || limit_cycles > 4000000000LL || !dev_err ||
        !aligned(dev_err, 4) || (which == 1 && (!counter || !aligned(counter, 4))))
        return MTP_ERR_INVALID_ARG;
    return from_cuda(mtp::wait_timeout_launch(which, (long long)limit_cycles, counter, dev_err,
                                              as_stream(stream)));
}

mtp_status mtp_debug_encode_e4m3(const float* in, int64_t n, uint8_t* out, void* stream) {
    if (!in || !out || n < 1 || !aligned(in, 4)) return MTP_ERR_INVALID_ARG;
    return from_cuda(mtp::debug_encode_launch(in, n, out, 0, as_stream(stream)));
}

mtp_status mtp_debug_encode_e2m1(const float* in, int64_t n, uint8_t* out, void* stream) {
    if (!in || !out || n < 1 || !aligned(in, 4)) return MTP_ERR_INVALID_ARG;
    return from_cuda(mtp::debug_encode_launch(in, n, out, 1, as_stream(stream)));
}

}  // extern "C"
