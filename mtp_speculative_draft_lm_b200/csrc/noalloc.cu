// mtp_lm_head_argmax_noalloc: the fused lm_head sweep + argmax without a caller
// workspace, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run a draft: a plugin
// that lives inside another framework's memory pool and may not allocate behind its
// back, an engine that reserves all free device memory for its KV cache at start-up
// and treats any later allocation as an error, or code that must not risk the device
// synchronisation that cudaMalloc/cudaFree can cause. They still pass their own
// inputs and outputs; only the sweep's scratch (the CTA partials, the last-CTA counter
// and x in the form the quantized tables' sweeps read it) comes from here.
//
// The scratch is the file-scope device array below: every GPU that loads this library
// holds it (kScratchBytes) until the process exits, and every call on that GPU shares
// it. In host code `g_sweep_scratch` names a host-side stand-in, not device memory, so
// the kernel is given the address that cudaGetSymbolAddress returns for the current
// device. That look-up runs on the first call made with each device current. With the
// CUDA runtime's lazy module loading (the default since CUDA 12.2) it is also the moment
// the array is committed on that device, so make the first call before reserving the
// device's free memory, and before any stream capture. A __device__ array without an
// initialiser is zero when its module loads, so the counter starts at zero; each call
// leaves it at zero again. Calls that overlap on the GPU (two streams, or two host
// threads) share the array and race: serialise them. Nothing here allocates: no
// cudaMalloc, no cudaFree, no memset.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/mtp.h"
#include "kernels.h"

namespace {

constexpr size_t kTicketBytes = 256;
// header + 1024 CTAs x 32 partials + 448 KB for x in the form the quantized tables' sweeps
// read it (NVFP4: its E2M1 terms and their scales; FP8 from 7 inputs: two E4M3 planes)
constexpr size_t kXBytes = 448 * 1024;
constexpr size_t kScratchBytes = kTicketBytes + 16 * 32 * 1024 + kXBytes;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_sweep_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// The device address of g_sweep_scratch on the current device (set up once per device).
mtp_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MTP_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_sweep_scratch) != cudaSuccess || !ptr) return MTP_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return MTP_OK;
}

}  // namespace

extern "C" size_t mtp_noalloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" mtp_status mtp_lm_head_argmax_noalloc(const mtp_weight* head, int64_t n_eff,
                                                 const uint16_t* x, int32_t M,
                                                 const int32_t* mask, int64_t mask_words,
                                                 int64_t mask_stride_words, int32_t* out_idx,
                                                 float* out_val, uint16_t* out_logits,
                                                 int32_t* dev_err, void* stream) {
    // Argument checks first (a null workspace is the one thing left to reject), so that a
    // rejected call never reads an unchecked table descriptor nor triggers the set-up;
    // then the scratch size this call needs.
    mtp_status st = mtp_lm_head_argmax(head, n_eff, x, M, mask, mask_words, mask_stride_words,
                                       out_idx, out_val, out_logits, dev_err, nullptr,
                                       kScratchBytes, nullptr);
    if (st != MTP_ERR_WORKSPACE) return st == MTP_OK ? MTP_ERR_CUDA : st;
    if (mtp_lm_head_ws_bytes(head, n_eff, M) > kScratchBytes) return MTP_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((st = scratch_for_current_device(&scratch)) != MTP_OK) return st;
    return mtp_lm_head_argmax(head, n_eff, x, M, mask, mask_words, mask_stride_words, out_idx,
                              out_val, out_logits, dev_err, scratch, kScratchBytes, stream);
}
