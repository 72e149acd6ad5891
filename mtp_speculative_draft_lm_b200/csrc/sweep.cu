// The draft lm_head sweep fused with argmax, and the combiner's fc projection.
//
// What it computes (the MTP draft-head pages: metrale_model_arch/deepseek_v4_mtp.rs,
// forward_one steps 1-2 and 6-7 and argmax_grammar_masked; glm5next_mtp_head/init.rs,
// the draft-head sweep over [vocab, hidden] rows packed at K):
//   l[m, n] = s_n * sum_k deq(W)[n, k] * x[m, k]   for n < n_eff, m < M
//   idx[m]  = the lowest allowed n with the largest l[m, n]  (mask bit n%32 of word n/32)
// with deq(W) the BF16 value, an E4M3 code (row scale s_n) or an E2M1 code times its
// E4M3 block scale (global scale s_n = g).
//
// Design (B200): the sweep is HBM-bound, so the whole table is streamed exactly once
// with 16-byte non-allocating loads, many in flight per thread. A CTA of 8 warps owns
// a contiguous range of 16-row tiles; the 8 warps split K (slab s of 4 lanes x 16 B
// goes to warp s % 8). Each warp turns its slab into tensor-core MMAs with the table
// rows as the 16-row A operand and the inputs as the 8-column B operand (swap-AB),
// so dequantization needs one convert per 2 codes and no FP32 FMA work; codes are
// decoded exactly into f16 (E4M3, and E2M1 times the E4M3 block scale, are exact in
// f16) and x is staged once per CTA in shared memory (bf16 for BF16 tables; f16
// scaled by a per-row power of two for quantized tables, undone in fp32 at the end).
// Per tile the 8 warp partials are summed in a fixed order (deterministic, the same
// for every M), scaled, masked and folded into a running (max, lowest index) per
// input row. Each CTA writes its partial; the last CTA to finish (an atomic ticket,
// no waiting) reduces them in CTA order and resets the ticket to zero.
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace mtp {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTileRows = 16;
constexpr int kMaxGrid = 1024;

struct Partial {
    float v;
    int32_t i;
};

template <int FMT> struct FmtTraits;
template <> struct FmtTraits<0> { static constexpr int V = 8;  static constexpr int D = 8; };
template <> struct FmtTraits<1> { static constexpr int V = 16; static constexpr int D = 6; };
template <> struct FmtTraits<2> { static constexpr int V = 32; static constexpr int D = 4; };

__device__ __forceinline__ bool mask_allows(const SweepParams& p, int m, int64_t row) {
    if (!p.mask) return true;
    int64_t word = row >> 5;
    if (word >= p.mask_words) return false;
    uint32_t bits = (uint32_t)__ldg(p.mask + (int64_t)m * p.mask_stride + word);
    return (bits >> (row & 31)) & 1u;
}

__device__ __forceinline__ bool row_needed(const SweepParams& p, int64_t row) {
    if (row >= p.n) return false;
    if (!p.mask) return true;
    for (int m = 0; m < p.M; ++m)
        if (mask_allows(p, m, row)) return true;
    return false;
}

__device__ __forceinline__ float block_sum(float v, float* scratch) {
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += scratch[w];
    return t;
}

__device__ __forceinline__ float block_max(float v, float* scratch) {
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t = fmaxf(t, scratch[w]);
    return t;
}

// Stage x (bf16) into xs[m][0..Kp): a copy (mode 0) or the combiner's concat
// [bf16(rms(e) w_e) || bf16(rms(hidden) w_h)] (mode 1). Columns K..Kp are zero.
template <int MODE>
__device__ void stage_bf16(const SweepParams& p, uint16_t* xs, int Kp, float* scratch) {
    const int tid = threadIdx.x;
    const int64_t K = p.k;
    if (MODE == 0) {
        const int vecs = Kp / 8;
        for (int i = tid; i < p.M * vecs; i += kThreads) {
            int m = i / vecs, v = i - m * vecs;
            int64_t k0 = (int64_t)v * 8;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (k0 < K) val = *reinterpret_cast<const uint4*>(p.x + (int64_t)m * K + k0);
            *reinterpret_cast<uint4*>(xs + (int64_t)m * p.kpad + k0) = val;
        }
    } else {
        const int h = p.h;
        for (int m = 0; m < p.M; ++m) {
            int64_t tok = p.tokens[m];
            bool bad = tok < 0 || tok >= p.vocab;
            if (bad && tid == 0) raise_flag(p.dev_err, DEVFLAG_BAD_TOKEN);
            const uint16_t* e = bad ? nullptr : p.embed + tok * h;
            const uint16_t* hx = p.hidden + (int64_t)m * h;
            float se = 0.f, sx = 0.f;
            for (int j = tid; j < h; j += kThreads) {
                float ev = e ? bf16_to_f32(e[j]) : 0.f;
                float xv = bf16_to_f32(hx[j]);
                se += ev * ev;
                sx += xv * xv;
            }
            se = block_sum(se, scratch);
            sx = block_sum(sx, scratch + kWarps);
            float inv_e = 1.0f / sqrtf(se / (float)h + p.eps);
            float inv_x = 1.0f / sqrtf(sx / (float)h + p.eps);
            uint16_t* row = xs + (int64_t)m * p.kpad;
            for (int j = tid; j < h; j += kThreads) {
                float ev = e ? bf16_to_f32(e[j]) : 0.f;
                row[j] = f32_to_bf16(ev * inv_e * bf16_to_f32(p.w_norm_embed[j]));
                row[h + j] = f32_to_bf16(bf16_to_f32(hx[j]) * inv_x *
                                         bf16_to_f32(p.w_norm_hidden[j]));
            }
            for (int j = (int)K + tid; j < Kp; j += kThreads) row[j] = 0;
        }
    }
    __syncthreads();
}

// Quantized tables: rescale each staged row by 2^e_m (largest |x| lands in
// [2^14, 2^15)) and convert it in place to f16. Exact for every element within
// 2^29 of the row maximum; the power of two is undone on the fp32 logit.
__device__ void stage_to_f16(const SweepParams& p, uint16_t* xs, int Kp, int* xexp,
                             float* scratch) {
    const int tid = threadIdx.x;
    for (int m = 0; m < p.M; ++m) {
        uint16_t* row = xs + (int64_t)m * p.kpad;
        float a = 0.f;
        for (int j = tid; j < Kp; j += kThreads) a = fmaxf(a, fabsf(bf16_to_f32(row[j])));
        a = block_max(a, scratch);
        int ex = 0;
        if (a > 0.f) frexpf(a, &ex);
        int e = (a > 0.f) ? 15 - ex : 0;
        if (tid == 0) xexp[m] = e;
        for (int j = tid; j < Kp; j += kThreads)
            row[j] = f32_to_f16(ldexpf(bf16_to_f32(row[j]), e));
        __syncthreads();
    }
}

template <int FMT, int NT, int MODE>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 2 : 1) sweep_kernel(const SweepParams p) {
    constexpr int V = FmtTraits<FMT>::V;
    constexpr int D = FmtTraits<FMT>::D;
    constexpr int SLAB = 4 * V;           // elements of one row covered by one slab
    constexpr int RED_COLS = 8 * NT;

    extern __shared__ __align__(16) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int64_t K = p.k;
    const int S = (int)((K + SLAB - 1) / SLAB);
    const int Kp = S * SLAB;

    uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
    size_t xs_bytes = ((size_t)p.M * p.kpad * 2 + 15) & ~(size_t)15;
    float* red = reinterpret_cast<float*>(smem + xs_bytes);          // [2][8][16][RED_COLS]
    float* scratch = red + 2 * kWarps * kTileRows * RED_COLS;        // [2*8]
    int* xexp = reinterpret_cast<int*>(scratch + 2 * kWarps);        // [16]
    int* last_flag = xexp + 16;

    const int64_t T = p.num_tiles;
    const int64_t t_begin = (T * blockIdx.x) / gridDim.x;
    const int64_t t_end = (T * (blockIdx.x + 1)) / gridDim.x;

    stage_bf16<MODE>(p, xs, Kp, scratch);
    if (FMT != 0) stage_to_f16(p, xs, Kp, xexp, scratch);

    const int Sw = (S > warp) ? (S - warp + kWarps - 1) / kWarps : 0;
    const int64_t total = (t_end - t_begin) * (int64_t)Sw;

    // rows of this lane inside a tile
    const int M = p.M;
    const bool xg0 = g < M;                 // B column g of n-tile 0 is a real input row
    const bool xg1 = NT > 1 && (8 + g) < M; // ... of n-tile 1

    // load stream
    int64_t lt = t_begin;
    int ls = warp;
    bool need0 = false, need1 = false;
    if (total > 0) {
        need0 = row_needed(p, lt * kTileRows + g);
        need1 = row_needed(p, lt * kTileRows + g + 8);
    }
    uint4 ra[D], rb[D];
    uint32_t rsc[D];

    auto issue = [&](int d) {
        const int64_t r0 = lt * kTileRows + g;
        const int64_t e0 = (int64_t)ls * SLAB + c * V;
        const bool kin = e0 < K;
        const uint8_t* base = p.w + (int64_t)ls * 64 + c * 16;
        ra[d] = (need0 && kin) ? ldg_stream(base + r0 * p.row_bytes) : make_uint4(0, 0, 0, 0);
        rb[d] = (need1 && kin) ? ldg_stream(base + (r0 + 8) * p.row_bytes) : make_uint4(0, 0, 0, 0);
        if (FMT == 2) {
            const int64_t kb = K >> 4;
            const uint8_t* sb = p.block_scale + (int64_t)ls * 8 + 2 * c;
            uint32_t s0 = (need0 && kin) ? ldg_u16(sb + r0 * kb) : 0u;
            uint32_t s1 = (need1 && kin) ? ldg_u16(sb + (r0 + 8) * kb) : 0u;
            rsc[d] = s0 | (s1 << 16);
        }
        ls += kWarps;
        if (ls >= S) {
            ls = warp;
            ++lt;
            if (lt < t_end) {
                need0 = row_needed(p, lt * kTileRows + g);
                need1 = row_needed(p, lt * kTileRows + g + 8);
            }
        }
    };

    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;

    // running best (reducer threads with row 0)
    float best_v = -INFINITY;
    int32_t best_i = INT_MAX;
    const int red_threads = kTileRows * RED_COLS;
    const int rrow = tid & 15, rcol = tid >> 4;

    int buf = 0;
    int64_t ct = t_begin;
    int cs = warp;

    auto reduce_tile = [&](int64_t tile, int b) {
        if (tid < red_threads) {
            const float* rp = red + (size_t)b * kWarps * kTileRows * RED_COLS;
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) a += rp[(w * kTileRows + rrow) * RED_COLS + rcol];
            const int64_t row = tile * kTileRows + rrow;
            const bool valid = row < p.n && rcol < M;
            float l = a;
            if (FMT != 0 && valid) l = ldexpf(a, -xexp[rcol]);
            if (FMT == 1 && valid) l *= __ldg(p.row_scale + row);
            if (FMT == 2 && valid) l *= __ldg(p.global_scale);
            if (MODE == 1) {
                if (valid) p.out_y[(int64_t)rcol * p.n + row] = f32_to_bf16(l);
            } else {
                const bool ok = valid && mask_allows(p, rcol, row);
                if (valid && p.out_logits)
                    p.out_logits[(int64_t)rcol * p.n + row] = ok ? f32_to_bf16(l) : (uint16_t)0xFF80u;
                float v = ok ? l : -INFINITY;
                int32_t i = ok ? (int32_t)row : INT_MAX;
#pragma unroll
                for (int o = 8; o; o >>= 1) {
                    float ov = __shfl_xor_sync(0xffffffffu, v, o);
                    int32_t oi = __shfl_xor_sync(0xffffffffu, i, o);
                    if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
                }
                if (rrow == 0 && (v > best_v || (v == best_v && i < best_i))) {
                    best_v = v;
                    best_i = i;
                }
            }
        }
    };

    auto flush_tile = [&]() {
        float* rp = red + (size_t)buf * kWarps * kTileRows * RED_COLS + warp * kTileRows * RED_COLS;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            rp[g * RED_COLS + t * 8 + 2 * c] = acc[t][0];
            rp[g * RED_COLS + t * 8 + 2 * c + 1] = acc[t][1];
            rp[(g + 8) * RED_COLS + t * 8 + 2 * c] = acc[t][2];
            rp[(g + 8) * RED_COLS + t * 8 + 2 * c + 1] = acc[t][3];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;
        }
        __syncthreads();
        reduce_tile(ct, buf);
        buf ^= 1;
    };

    auto consume = [&](int d) {
        const uint16_t* x0 = xs + (int64_t)g * p.kpad + cs * SLAB + c * V;
        const uint16_t* x1 = xs + (int64_t)(8 + g) * p.kpad + cs * SLAB + c * V;
        if (FMT == 0) {
            uint4 xa = xg0 ? lds128(x0) : make_uint4(0, 0, 0, 0);
            mma_bf16_16816(acc[0], ra[d].x, rb[d].x, ra[d].y, rb[d].y, xa.x, xa.y);
            mma_bf16_16816(acc[0], ra[d].z, rb[d].z, ra[d].w, rb[d].w, xa.z, xa.w);
            if (NT > 1) {
                uint4 xb = xg1 ? lds128(x1) : make_uint4(0, 0, 0, 0);
                mma_bf16_16816(acc[NT - 1], ra[d].x, rb[d].x, ra[d].y, rb[d].y, xb.x, xb.y);
                mma_bf16_16816(acc[NT - 1], ra[d].z, rb[d].z, ra[d].w, rb[d].w, xb.z, xb.w);
            }
        } else if (FMT == 1) {
            uint32_t wa[4] = {ra[d].x, ra[d].y, ra[d].z, ra[d].w};
            uint32_t wb[4] = {rb[d].x, rb[d].y, rb[d].z, rb[d].w};
            uint4 xa0 = xg0 ? lds128(x0) : make_uint4(0, 0, 0, 0);
            uint4 xa1 = xg0 ? lds128(x0 + 8) : make_uint4(0, 0, 0, 0);
            uint32_t xa[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
            uint32_t xb[8];
            if (NT > 1) {
                uint4 xb0 = xg1 ? lds128(x1) : make_uint4(0, 0, 0, 0);
                uint4 xb1 = xg1 ? lds128(x1 + 8) : make_uint4(0, 0, 0, 0);
                xb[0] = xb0.x; xb[1] = xb0.y; xb[2] = xb0.z; xb[3] = xb0.w;
                xb[4] = xb1.x; xb[5] = xb1.y; xb[6] = xb1.z; xb[7] = xb1.w;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t a0 = e4m3x2_to_f16x2((uint16_t)(wa[i] & 0xFFFFu));
                uint32_t a2 = e4m3x2_to_f16x2((uint16_t)(wa[i] >> 16));
                uint32_t a1 = e4m3x2_to_f16x2((uint16_t)(wb[i] & 0xFFFFu));
                uint32_t a3 = e4m3x2_to_f16x2((uint16_t)(wb[i] >> 16));
                mma_f16_16816(acc[0], a0, a1, a2, a3, xa[2 * i], xa[2 * i + 1]);
                if (NT > 1) mma_f16_16816(acc[NT - 1], a0, a1, a2, a3, xb[2 * i], xb[2 * i + 1]);
            }
        } else {
            uint32_t wa[4] = {ra[d].x, ra[d].y, ra[d].z, ra[d].w};
            uint32_t wb[4] = {rb[d].x, rb[d].y, rb[d].z, rb[d].w};
            // block scales: rows g / g+8, blocks 2c (words 0,1) and 2c+1 (words 2,3)
            uint32_t sa = e4m3x2_to_f16x2((uint16_t)(rsc[d] & 0xFFFFu));
            uint32_t sb = e4m3x2_to_f16x2((uint16_t)(rsc[d] >> 16));
            const uint32_t sa_lo = __byte_perm(sa, 0, 0x1010), sa_hi = __byte_perm(sa, 0, 0x3232);
            const uint32_t sb_lo = __byte_perm(sb, 0, 0x1010), sb_hi = __byte_perm(sb, 0, 0x3232);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t qa[4], qb[4];
                e2m1x8_to_f16x2x4(wa[i], qa);
                e2m1x8_to_f16x2x4(wb[i], qb);
                const uint32_t s_a = i < 2 ? sa_lo : sa_hi;
                const uint32_t s_b = i < 2 ? sb_lo : sb_hi;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    qa[j] = hmul2(qa[j], s_a);
                    qb[j] = hmul2(qb[j], s_b);
                }
                // x words for elements 8i .. 8i+7 of this lane's 32
                uint4 xv = xg0 ? lds128(x0 + 8 * i) : make_uint4(0, 0, 0, 0);
                mma_f16_16816(acc[0], qa[0], qb[0], qa[1], qb[1], xv.x, xv.y);
                mma_f16_16816(acc[0], qa[2], qb[2], qa[3], qb[3], xv.z, xv.w);
                if (NT > 1) {
                    uint4 xw = xg1 ? lds128(x1 + 8 * i) : make_uint4(0, 0, 0, 0);
                    mma_f16_16816(acc[NT - 1], qa[0], qb[0], qa[1], qb[1], xw.x, xw.y);
                    mma_f16_16816(acc[NT - 1], qa[2], qb[2], qa[3], qb[3], xw.z, xw.w);
                }
            }
        }
    };

    if (Sw > 0) {
#pragma unroll
        for (int d = 0; d < D; ++d)
            if (d < total) issue(d);
        for (int64_t j0 = 0; j0 < total; j0 += D) {
#pragma unroll
            for (int d = 0; d < D; ++d) {
                if (j0 + d < total) {
                    consume(d);
                    if (j0 + d + D < total) issue(d);
                    cs += kWarps;
                    if (cs >= S) {
                        flush_tile();
                        cs = warp;
                        ++ct;
                    }
                }
            }
        }
    } else {
        // this warp owns no slab of K: it still takes part in every tile's barrier
        for (; ct < t_end; ++ct) flush_tile();
    }

    if (MODE == 1) return;

    Partial* parts = reinterpret_cast<Partial*>(p.partials);
    if (tid < red_threads && rrow == 0 && rcol < M) {
        parts[(int64_t)blockIdx.x * 16 + rcol] = Partial{best_v, best_i};
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        unsigned int ticket = atomicAdd(p.ticket, 1u);
        *last_flag = (ticket == gridDim.x - 1) ? 1 : 0;
    }
    __syncthreads();
    if (*last_flag == 0) return;
    __threadfence();
    if (tid < M) {
        float bv = -INFINITY;
        int32_t bi = INT_MAX;
        for (int b = 0; b < (int)gridDim.x; ++b) {
            Partial q;
            const Partial* src = parts + (int64_t)b * 16 + tid;
            q.v = __ldcg(&src->v);
            q.i = __ldcg(&src->i);
            if (q.v > bv || (q.v == bv && q.i < bi)) { bv = q.v; bi = q.i; }
        }
        if (bi == INT_MAX) {
            bi = 0;
            bv = -INFINITY;
            raise_flag(p.dev_err, DEVFLAG_EMPTY_MASK);
        }
        p.out_idx[tid] = bi;
        if (p.out_val) p.out_val[tid] = bv;
    }
    if (tid == 0) *p.ticket = 0u;  // leave the workspace ready for the next call
}

template <int FMT, int NT, int MODE>
cudaError_t launch_one(const SweepParams& p, cudaStream_t s, SweepLaunch* info) {
    auto kern = sweep_kernel<FMT, NT, MODE>;
    int kpad = 0;
    size_t smem = sweep_smem_bytes(p.M, p.k, FMT, &kpad);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) !=
        cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    int64_t grid = (int64_t)sms * per_sm;
    if (grid > p.num_tiles) grid = p.num_tiles;
    if (grid > kMaxGrid) grid = kMaxGrid;
    if (grid < 1) grid = 1;
    SweepParams q = p;
    q.kpad = kpad;
    kern<<<(int)grid, kThreads, smem, s>>>(q);
    if (info) {
        info->grid = (int)grid;
        info->smem_bytes = (int)smem;
    }
    return cudaGetLastError();
}

}  // namespace

size_t sweep_smem_bytes(int M, int64_t k, int fmt, int* kpad_out) {
    const int V = fmt == 0 ? 8 : fmt == 1 ? 16 : 32;
    const int64_t slab = 4 * V;
    const int64_t Kp = ((k + slab - 1) / slab) * slab;
    const int64_t kpad = Kp + 8;  // 16-byte skew between staged rows
    if (kpad_out) *kpad_out = (int)kpad;
    const int NT = M > 8 ? 2 : 1;
    size_t xs = ((size_t)M * kpad * 2 + 15) & ~(size_t)15;
    size_t red = (size_t)2 * kWarps * kTileRows * 8 * NT * sizeof(float);
    return xs + red + 2 * kWarps * sizeof(float) + 17 * sizeof(int) + 16;
}

int sweep_max_grid() { return kMaxGrid; }

cudaError_t sweep_launch(const SweepParams& p, int fmt, int mode, cudaStream_t s,
                         SweepLaunch* info) {
    const bool two = p.M > 8;
#define MTP_SWEEP_CASE(F, NTV, MD) \
    if (fmt == F && (NTV == 2) == two && mode == MD) return launch_one<F, NTV, MD>(p, s, info);
    MTP_SWEEP_CASE(0, 1, 0) MTP_SWEEP_CASE(0, 2, 0)
    MTP_SWEEP_CASE(1, 1, 0) MTP_SWEEP_CASE(1, 2, 0)
    MTP_SWEEP_CASE(2, 1, 0) MTP_SWEEP_CASE(2, 2, 0)
    MTP_SWEEP_CASE(0, 1, 1) MTP_SWEEP_CASE(0, 2, 1)
    MTP_SWEEP_CASE(1, 1, 1) MTP_SWEEP_CASE(1, 2, 1)
    MTP_SWEEP_CASE(2, 1, 1) MTP_SWEEP_CASE(2, 2, 1)
#undef MTP_SWEEP_CASE
    return cudaErrorInvalidValue;
}

}  // namespace mtp
