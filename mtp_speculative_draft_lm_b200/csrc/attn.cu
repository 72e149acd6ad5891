// Single-token decode attention of the MTP drafter over its paged E4M3 KV cache (the
// cache mtp_prefill_kv writes).
//
// What it computes (metrale_model_layers/layers/mtp_head/new.rs: one attention layer with
// its own paged cache, block size 16, FP8 cache with unit K/V scales by default, and a
// single-token decode kernel for that FP8 cache; spark_model/layers/mtp_head.rs: attention
// follows fc in the draft's forward order; metrale_model_arch/deepseek_v4_mtp.rs
// forward_one step 4: cache row p at slot block_table[p / bs] * bs + p % bs). The pages
// print no formula; the standard one, for query head i and kv head g = i / (nq / nkv):
//   s_p = scale * sum_d q[i, d] k_scale e4m3(K[slot(p), g, d]),  p < seq_len
//   out[i, d] = sum_p softmax(s)_p v_scale e4m3(V[slot(p), g, d])
//
// Design (B200, HBM-bound: every cached K and V byte is read once): the positions are split
// into pieces of kAPos; CTA (g, piece) loads its positions' K and V rows for kv head g with
// 16-byte loads (many in flight per thread), keeps V in shared memory, computes the scores
// of every query head of the group with fp32 sums, then per head the piece's maximum, its
// sum of exp(s - max) and the exp-weighted sum of V rows; a second kernel merges the pieces
// of each head in a fixed order (deterministic) and writes bf16. Rows whose block is
// missing or out of range are skipped and set MTP_DEVFLAG_BAD_SLOT.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace mtp {
namespace {

constexpr int kAPos = 256;      // positions per CTA
constexpr int kAThreads = 128;
constexpr int kAMaxGroup = 16;  // query heads per kv head
constexpr int kAMaxHd = 256;
constexpr int kAMaxPieces = 8192;  // cache rows up to 2M (the merge keeps a factor per piece)

struct AttnParams {
    const uint16_t* q;  // [nq, hd] bf16
    int nq, nkv, hd, group;
    const uint8_t* k_cache;
    const uint8_t* v_cache;
    const int32_t* block_table;
    int64_t n_table;
    int block_size;
    int64_t num_blocks;
    int64_t seq_len;
    float qk_scale;  // scale * k_scale
    float v_scale;
    float* part;     // [pieces][nq][hd + 2]: (max, sum of exp, weighted V sum)
    int pieces;
    uint16_t* out;
    int32_t* dev_err;
};

// 16-byte asynchronous copy global -> shared (L2 only), and the wait for this thread's.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// 16 E4M3 codes -> 16 floats (exact).
__device__ __forceinline__ void e4m3x16(uint4 c, float (&f)[16]) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)(w[i] & 0xFFFFu)));
        const float2 b = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)(w[i] >> 16)));
        f[4 * i] = a.x;
        f[4 * i + 1] = a.y;
        f[4 * i + 2] = b.x;
        f[4 * i + 3] = b.y;
    }
}

template <int HD>
__global__ void __launch_bounds__(kAThreads) attn_piece_kernel(const __grid_constant__ AttnParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int hd = HD;
    const int G = p.group;
    float* qs = reinterpret_cast<float*>(smem);              // [G][hd]
    float* sc = qs + G * hd;                                  // [G][kAPos] scores, then weights
    float* stat = sc + G * kAPos;                             // [G][2] max, sum
    uint8_t* vs = reinterpret_cast<uint8_t*>(stat + 2 * kAMaxGroup);  // [kAPos][hd] V codes
    const int g = blockIdx.x, piece = blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t p0 = (int64_t)piece * kAPos;
    const int npos = (int)min((int64_t)kAPos, p.seq_len - p0);
    pdl_launch_dependents();

    for (int i = tid; i < G * hd; i += kAThreads)
        qs[i] = bf16_to_f32(p.q[(int64_t)(g * G) * hd + i]) * p.qk_scale;
    __syncthreads();

    // scores: a thread per position; its K row in 16-byte pieces, V row into shared memory
    constexpr int pieces16 = HD / 16;
    for (int t = tid; t < kAPos; t += kAThreads) {
        float s[kAMaxGroup];
#pragma unroll
        for (int i = 0; i < kAMaxGroup; ++i) s[i] = -INFINITY;
        int64_t slot = -1;
        if (t < npos) {
            const int64_t pos = p0 + t;
            const int64_t b = pos / p.block_size;
            if (b < p.n_table) {
                const int64_t blk = p.block_table[b];
                if (blk >= 0 && blk < p.num_blocks) slot = blk * p.block_size + pos % p.block_size;
            }
            if (slot < 0) raise_flag(p.dev_err, DEVFLAG_BAD_SLOT);
        }
        if (slot >= 0) {
            const uint8_t* krow = p.k_cache + (slot * p.nkv + g) * (int64_t)hd;
            const uint8_t* vrow = p.v_cache + (slot * p.nkv + g) * (int64_t)hd;
#pragma unroll
            for (int i = 0; i < kAMaxGroup; ++i) s[i] = 0.f;
            // every 16-byte piece of both rows in flight before any is used: V straight
            // into shared memory (asynchronous copies), K into registers
#pragma unroll
            for (int c = 0; c < pieces16; ++c) cp_async16(vs + (size_t)t * hd + 16 * c, vrow + 16 * c);
            uint4 kr[pieces16];
#pragma unroll
            for (int c = 0; c < pieces16; ++c) kr[c] = ldg_stream(krow + 16 * c);
#pragma unroll
            for (int c = 0; c < pieces16; ++c) {
                float kf[16];
                e4m3x16(kr[c], kf);
#pragma unroll
                for (int i = 0; i < kAMaxGroup; ++i) {
                    if (i >= G) break;
                    const float* qr = qs + i * hd + 16 * c;
                    float a = s[i];
#pragma unroll
                    for (int j = 0; j < 16; ++j) a = fmaf(qr[j], kf[j], a);
                    s[i] = a;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kAMaxGroup; ++i)
            if (i < G) sc[i * kAPos + t] = s[i];
    }
    cp_async_wait_all();
    __syncthreads();

    // per head: the piece's maximum and sum of exp(s - max); scores become weights
    for (int i = warp; i < G; i += kAThreads / 32) {
        float m = -INFINITY;
        for (int t = lane; t < kAPos; t += 32) m = fmaxf(m, sc[i * kAPos + t]);
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int t = lane; t < kAPos; t += 32) {
            const float s = sc[i * kAPos + t];
            const float w = (m == -INFINITY || s == -INFINITY) ? 0.f : expf(s - m);
            sc[i * kAPos + t] = w;
            l += w;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) {
            stat[2 * i] = m;
            stat[2 * i + 1] = l;
        }
    }
    __syncthreads();

    // weighted V sums: a thread per (head, 8 dims), positions in order
    const int dch = hd / 8;
    for (int u = tid; u < G * dch; u += kAThreads) {
        const int i = u / dch, d0 = 8 * (u - i * dch);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int t = 0; t < npos; ++t) {
            const float w = sc[i * kAPos + t];
            if (w == 0.f) continue;
            const uint2 c = *reinterpret_cast<const uint2*>(vs + (size_t)t * hd + d0);
            const uint32_t cw[2] = {c.x, c.y};
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const float2 a = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)(cw[h2] & 0xFFFFu)));
                const float2 b = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)(cw[h2] >> 16)));
                acc[4 * h2] = fmaf(w, a.x, acc[4 * h2]);
                acc[4 * h2 + 1] = fmaf(w, a.y, acc[4 * h2 + 1]);
                acc[4 * h2 + 2] = fmaf(w, b.x, acc[4 * h2 + 2]);
                acc[4 * h2 + 3] = fmaf(w, b.y, acc[4 * h2 + 3]);
            }
        }
        float* dst = p.part + ((int64_t)piece * p.nq + g * G + i) * (hd + 2);
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[2 + d0 + j] = acc[j];
        if (d0 == 0) {
            dst[0] = stat[2 * i];
            dst[1] = stat[2 * i + 1];
        }
    }
}

// One CTA per query head: out = sum_s e^(m_s - M) acc_s / sum_s e^(m_s - M) l_s (zero
// when no row was readable), as bf16. The pieces' (max, sum) pairs are loaded in parallel
// and their factors folded in a fixed order; each thread then sums its dimension over the
// pieces with many loads in flight.
__global__ void __launch_bounds__(kAMaxHd) attn_merge_kernel(const __grid_constant__ AttnParams p) {
    __shared__ float fac[kAMaxPieces];
    __shared__ float red[kAMaxHd / 32];
    __shared__ float tot[2];
    const int i = blockIdx.x, d = threadIdx.x, hd = p.hd;
    const int lane = d & 31, warp = d >> 5;
    pdl_wait();
    const int64_t rs = (int64_t)p.nq * (hd + 2);  // floats between a head's pieces
    const float* base = p.part + (int64_t)i * (hd + 2);
    float mloc = -INFINITY;
    for (int s = d; s < p.pieces; s += kAMaxHd) mloc = fmaxf(mloc, base[s * rs]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
    if (lane == 0) red[warp] = mloc;
    __syncthreads();
    if (d == 0) {
        float M = -INFINITY;
        for (int w = 0; w < kAMaxHd / 32; ++w) M = fmaxf(M, red[w]);
        tot[0] = M;
    }
    __syncthreads();
    const float M = tot[0];
    for (int s = d; s < p.pieces; s += kAMaxHd) {
        const float m = base[s * rs];
        fac[s] = (M == -INFINITY || m == -INFINITY) ? 0.f : expf(m - M);
    }
    __syncthreads();
    if (d == 0) {  // the denominator in piece order
        float L = 0.f;
        for (int s = 0; s < p.pieces; ++s) L = fmaf(fac[s], base[s * rs + 1], L);
        tot[1] = L;
    }
    float a = 0.f;
    if (d < hd) {
        int s = 0;
        for (; s + 8 <= p.pieces; s += 8) {  // eight independent loads in flight
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = base[(s + j) * rs + 2 + d];
#pragma unroll
            for (int j = 0; j < 8; ++j) a = fmaf(fac[s + j], v[j], a);
        }
        for (; s < p.pieces; ++s) a = fmaf(fac[s], base[s * rs + 2 + d], a);
    }
    __syncthreads();
    const float L = tot[1];
    if (d < hd) p.out[(int64_t)i * hd + d] = f32_to_bf16(L > 0.f ? a / L * p.v_scale : 0.f);
}

}  // namespace

int attn_max_group() { return kAMaxGroup; }

size_t attn_ws_bytes(int nq, int hd, int64_t seq_len) {
    const int64_t pieces = (seq_len + kAPos - 1) / kAPos;
    return (size_t)(pieces < 1 ? 1 : pieces) * (size_t)nq * (size_t)(hd + 2) * sizeof(float);
}

cudaError_t attn_launch(const uint16_t* q, int nq, int nkv, int hd, const uint8_t* k_cache,
                        const uint8_t* v_cache, const int32_t* block_table, int64_t n_table,
                        int block_size, int64_t num_blocks, int64_t seq_len, float k_scale,
                        float v_scale, float scale, uint16_t* out, int32_t* dev_err, void* ws,
                        cudaStream_t s) {
    AttnParams p{};
    p.q = q;
    p.nq = nq;
    p.nkv = nkv;
    p.hd = hd;
    p.group = nq / nkv;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_table = block_table;
    p.n_table = n_table;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    p.seq_len = seq_len;
    p.qk_scale = scale * k_scale;
    p.v_scale = v_scale;
    p.part = static_cast<float*>(ws);
    p.pieces = (int)((seq_len + kAPos - 1) / kAPos);
    p.out = out;
    p.dev_err = dev_err;
    const size_t smem = (size_t)p.group * hd * 4 + (size_t)p.group * kAPos * 4 +
                        2 * kAMaxGroup * 4 + (size_t)kAPos * hd;
    cudaError_t e = cudaSuccess;
    auto kern = hd == 64 ? attn_piece_kernel<64> : hd == 128 ? attn_piece_kernel<128> : attn_piece_kernel<256>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)nkv, (unsigned)p.pieces), kAThreads, smem, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)nq);
    cfg.blockDim = dim3(kAMaxHd);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, attn_merge_kernel, p)) != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace mtp
