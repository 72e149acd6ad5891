// Load-time weight quantizers (the draft-head pages name a BF16 -> FP8 weight
// quantizer and a two-pass BF16 -> NVFP4 quantizer -- a global |w| max pass and a
// block-encode pass -- in metrale_model_layers/layers/mtp_head/new.rs (MtpHead::new,
// kernel lookups) and spark_model/layers/mtp_head.rs (quantize_proj); their
// arithmetic is not on the pages). Every step is an fp32 operation rounded to
// nearest even, so the codes are bit-identical to any implementation of the rule:
//
//   FP8 per row:  a = max|W[n,:]|, s = a / 448, q = e4m3(W / s); a == 0 -> s = 0, q = 0.
//   NVFP4:        A = max|W|, g = A / 2688 (1 when A == 0); per 16-block:
//                 B = max|W_b|, sb = e4m3((B / 6) / g), S = e4m3(sb) * g,
//                 q = e2m1(W / S) (0 when S == 0); element 2j in the low nibble.
//                 Block-scale rows are padded with zeros to a multiple of 16 bytes so that
//                 every row starts 16-byte aligned (the sweep streams them with TMA).
//
// E4M3/E2M1 encodes use the hardware satfinite converts (round to nearest even,
// saturating); the exhaustive checks compare them with the CPU oracle.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace mtp {
namespace {

constexpr int kQThreads = 256;
constexpr int kAbsmaxMaxGrid = 1024;

__device__ __forceinline__ float absmax8(const uint4& v) {
    float a = fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x)));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w))));
    return a;
}

__device__ __forceinline__ uint32_t enc_e4m3x4(float a, float b, float c, float d) {
    return (uint32_t)f32x2_to_e4m3x2(a, b) | ((uint32_t)f32x2_to_e4m3x2(c, d) << 16);
}

// One warp per row.
__global__ void __launch_bounds__(kQThreads) quant_fp8_kernel(const uint16_t* __restrict__ w,
                                                              int64_t n, int64_t k,
                                                              uint8_t* __restrict__ codes,
                                                              float* __restrict__ row_scale) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kQThreads / 32);
    for (int64_t r = (int64_t)blockIdx.x * (kQThreads / 32) + (threadIdx.x >> 5); r < n;
         r += warps) {
        const uint16_t* row = w + r * k;
        float a = 0.f;
        for (int64_t j = (int64_t)lane * 8; j < k; j += 256)
            a = fmaxf(a, absmax8(*reinterpret_cast<const uint4*>(row + j)));
        for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const float s = __fdiv_rn(a, 448.0f);
        if (lane == 0) row_scale[r] = s;
        uint8_t* out = codes + r * k;
        for (int64_t j = (int64_t)lane * 8; j < k; j += 256) {
            uint2 q = make_uint2(0u, 0u);
            if (a != 0.f) {
                uint4 v = *reinterpret_cast<const uint4*>(row + j);
                q.x = enc_e4m3x4(__fdiv_rn(bf16_lo(v.x), s), __fdiv_rn(bf16_hi(v.x), s),
                                 __fdiv_rn(bf16_lo(v.y), s), __fdiv_rn(bf16_hi(v.y), s));
                q.y = enc_e4m3x4(__fdiv_rn(bf16_lo(v.z), s), __fdiv_rn(bf16_hi(v.z), s),
                                 __fdiv_rn(bf16_lo(v.w), s), __fdiv_rn(bf16_hi(v.w), s));
            }
            *reinterpret_cast<uint2*>(out + j) = q;
        }
    }
}

// Pass 1: global |w| max. Partials per CTA; the last CTA (atomic ticket) reduces,
// writes g and re-zeroes the ticket.
__global__ void __launch_bounds__(kQThreads) nvfp4_absmax_kernel(const uint16_t* __restrict__ w,
                                                                 int64_t count8,
                                                                 uint32_t* ws,
                                                                 float* global_scale) {
    __shared__ float red[kQThreads / 32];
    __shared__ int last;
    float a = 0.f;
    for (int64_t i = (int64_t)blockIdx.x * kQThreads + threadIdx.x; i < count8;
         i += (int64_t)gridDim.x * kQThreads)
        a = fmaxf(a, absmax8(ldg_stream(w + i * 8)));
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.f;
        for (int i = 0; i < kQThreads / 32; ++i) b = fmaxf(b, red[i]);
        float* part = reinterpret_cast<float*>(ws + 64);
        part[blockIdx.x] = b;
        __threadfence();
        last = (atomicAdd(ws, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    if (threadIdx.x == 0) {
        const float* part = reinterpret_cast<const float*>(ws + 64);
        float A = 0.f;
        for (int i = 0; i < (int)gridDim.x; ++i) A = fmaxf(A, __ldcg(part + i));
        *global_scale = (A == 0.f) ? 1.0f : __fdiv_rn(A, 2688.0f);
        *ws = 0u;
    }
}

// Pass 2: one thread per 16-element block. Block-scale rows are `pitch` bytes long
// (k/16 rounded up to 16); the padding bytes are written as zero.
__global__ void __launch_bounds__(kQThreads) nvfp4_encode_kernel(const uint16_t* __restrict__ w,
                                                                 int64_t n, int64_t nb,
                                                                 int64_t pitch,
                                                                 uint8_t* __restrict__ codes,
                                                                 uint8_t* __restrict__ bscale,
                                                                 const float* global_scale) {
    const float g = *global_scale;
    const int64_t blocks = n * nb;
    const int64_t stride = (int64_t)gridDim.x * kQThreads;
    for (int64_t b = (int64_t)blockIdx.x * kQThreads + threadIdx.x; b < blocks; b += stride) {
        const uint4 v0 = ldg_stream(w + b * 16);
        const uint4 v1 = ldg_stream(w + b * 16 + 8);
        const float B = fmaxf(absmax8(v0), absmax8(v1));
        const float u = __fdiv_rn(__fdiv_rn(B, 6.0f), g);
        const uint32_t sb = f32x2_to_e4m3x2(u, 0.f) & 0xFFu;
        const float S = e4m3_to_f32(sb) * g;
        uint2 q = make_uint2(0u, 0u);
        if (S != 0.f) {
            const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            uint32_t bytes[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                bytes[i] = f32x2_to_e2m1x2(__fdiv_rn(bf16_lo(wv[i]), S),
                                           __fdiv_rn(bf16_hi(wv[i]), S));
            q.x = bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24);
            q.y = bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24);
        }
        *reinterpret_cast<uint2*>(codes + b * 8) = q;
        const int64_t r = b / nb;
        bscale[r * pitch + (b - r * nb)] = (uint8_t)sb;
    }
    const int64_t pad = pitch - nb;
    if (pad > 0) {
        for (int64_t i = (int64_t)blockIdx.x * kQThreads + threadIdx.x; i < n * pad; i += stride) {
            const int64_t r = i / pad;
            bscale[r * pitch + nb + (i - r * pad)] = 0;
        }
    }
}

__global__ void debug_encode_kernel(const float* in, int64_t n, uint8_t* out, int which) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float v = in[i];
        out[i] = which == 0 ? (uint8_t)(f32x2_to_e4m3x2(v, 0.f) & 0xFF)
                            : (uint8_t)(f32x2_to_e2m1x2(v, 0.f) & 0xF);
    }
}

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

int quant_nvfp4_max_grid() { return kAbsmaxMaxGrid; }

int64_t nvfp4_scale_pitch(int64_t k) { return ((k / 16 + 15) / 16) * 16; }

cudaError_t quant_fp8_launch(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                             float* row_scale, cudaStream_t s) {
    int64_t grid = (n + 7) / 8;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (grid > cap) grid = cap;
    quant_fp8_kernel<<<(int)grid, kQThreads, 0, s>>>(w, n, k, codes, row_scale);
    return cudaGetLastError();
}

cudaError_t quant_nvfp4_launch(const uint16_t* w, int64_t n, int64_t k, uint8_t* codes,
                               uint8_t* block_scale, float* global_scale, uint32_t* ws,
                               cudaStream_t s) {
    const int64_t count8 = n * k / 8;
    int64_t g1 = (count8 + kQThreads - 1) / kQThreads;
    int64_t cap = (int64_t)sm_count() * 4;
    if (cap > kAbsmaxMaxGrid) cap = kAbsmaxMaxGrid;
    if (g1 > cap) g1 = cap;
    nvfp4_absmax_kernel<<<(int)g1, kQThreads, 0, s>>>(w, count8, ws, global_scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t blocks = n * k / 16;
    int64_t g2 = (blocks + kQThreads - 1) / kQThreads;
    const int64_t cap2 = (int64_t)sm_count() * 8;
    if (g2 > cap2) g2 = cap2;
    nvfp4_encode_kernel<<<(int)g2, kQThreads, 0, s>>>(w, n, k / 16, nvfp4_scale_pitch(k), codes,
                                                        block_scale, global_scale);
    return cudaGetLastError();
}

cudaError_t debug_encode_launch(const float* in, int64_t n, uint8_t* out, int which,
                                cudaStream_t s) {
    int64_t grid = (n + 255) / 256;
    if (grid > 4096) grid = 4096;
    if (grid < 1) grid = 1;
    debug_encode_kernel<<<(int)grid, 256, 0, s>>>(in, n, out, which);
    return cudaGetLastError();
}

}  // namespace mtp
