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
// Design (B200, HBM-bound: every cached K and V byte is read once): CTA (g, piece) takes
// kv head g over a contiguous range of positions (as many CTAs as the SMs hold at once), in
// sub-pieces of 64 positions that a three-stage ring of 16-byte asynchronous copies
// brings into shared memory (rows of a missing block zero-filled). Both contractions run
// on the tensor cores (mma.sync m16n8k16, f16 operands, fp32 accumulators): the scores as
// K[64 positions, hd] . Q^T, with E4M3 K decoded exactly to f16 and each query head in
// f16 scaled by a power of two (exact), then an online softmax over the sub-pieces (fp32
// running maximum and sum) and the weighted V sum as V^T . W^T, the weights
// exp(s - max) in (0, 1] rounded to f16 (the same rounded weights in the sum of exps).
// Each CTA writes its heads' (max, sum, weighted V sum); a second kernel merges the pieces
// of each head in a fixed order (deterministic) and writes bf16. Rows whose block is
// missing or out of range are skipped and set MTP_DEVFLAG_BAD_SLOT.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace mtp {
namespace {

constexpr int kSP = 64;          // positions per sub-piece (four warps x 16)
constexpr int kAThreads = 128;
constexpr int kAStages = 3;
constexpr int kAMaxGroup = 16;  // query heads per kv head
constexpr int kAMaxHd = 256;
constexpr int kAMaxPieces = 1024;  // pieces per kv head (the merge keeps a factor per piece)
constexpr int kWPitch = kSP + 8;   // f16 weights per head row in shared memory

struct AttnParams {
    const uint16_t* q;  // [nq, hd] bf16
    int nq, nkv, hd, group;
    const uint8_t* k_cache;
    const uint8_t* v_cache;
    const int32_t* block_table;
    int64_t n_table;
    int block_size;
    int bs_shift;       // log2(block_size) when a power of two, else -1
    int64_t num_blocks;
    int64_t seq_len;
    int64_t per_piece;  // positions per piece (a multiple of kSP)
    float qk_scale;     // scale * k_scale
    float v_scale;
    float* part;        // [pieces][nq][hd + 2]: (max, sum of exp, weighted V sum)
    int pieces;
    uint16_t* out;
    int32_t* dev_err;
};

// 16-byte asynchronous copy global -> shared (L2 only), group commit and wait.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

template <int HD>
__host__ __device__ constexpr int attn_row_pitch() { return HD + 16; }  // bank-conflict-free
template <int HD>
__host__ __device__ constexpr int attn_q_pitch() { return HD + 8; }     // f16 elements

template <int HD>
__host__ __device__ constexpr size_t attn_smem_bytes() {
    return (size_t)kAStages * 2 * kSP * attn_row_pitch<HD>()  // K and V rings
           + (size_t)kAMaxGroup * attn_q_pitch<HD>() * 2         // q in f16
           + (size_t)kAMaxGroup * kWPitch * 2                    // weights in f16
           + (size_t)kAStages * kSP * 4                          // row valid flags
           + (size_t)2 * 4 * kAMaxGroup * 4                      // per-warp max and sum
           + (size_t)kAMaxGroup * 4;                             // per-head score factor
}

template <int HD, int NT>
__global__ void __launch_bounds__(kAThreads) attn_piece_kernel(const __grid_constant__ AttnParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int RP = attn_row_pitch<HD>();
    constexpr int QP = attn_q_pitch<HD>();
    constexpr int KC = HD / 16;          // 16-byte pieces of a row, and MMA K chunks
    constexpr int MT = HD / 64;          // 16-dim tiles of the V sum per warp
    uint8_t* kring = smem;                                          // [stages][kSP][RP]
    uint8_t* vring = kring + kAStages * kSP * RP;                   // [stages][kSP][RP]
    uint16_t* qh = reinterpret_cast<uint16_t*>(vring + kAStages * kSP * RP);  // [16][QP] f16
    uint16_t* wsm = qh + kAMaxGroup * QP;                           // [16][kWPitch] f16
    int* valid = reinterpret_cast<int*>(wsm + kAMaxGroup * kWPitch);  // [stages][kSP]
    float* redm = reinterpret_cast<float*>(valid + kAStages * kSP);   // [4][16]
    float* redl = redm + 4 * kAMaxGroup;                               // [4][16]
    float* hfac = redl + 4 * kAMaxGroup;                               // [16]

    const int g = blockIdx.x, piece = blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
    const int G = p.group;
    const int64_t pbeg = (int64_t)piece * p.per_piece;
    const int64_t pend = min(p.seq_len, pbeg + p.per_piece);
    const int nsub = (int)((pend - pbeg + kSP - 1) / kSP);
    pdl_launch_dependents();

    // copies of sub-piece i into ring stage i % 3 (positions past the piece: invalid)
    // 32-bit position arithmetic (seq_len <= 2^21); a power-of-two block size shifts
    const int pend32 = (int)pend;
    // copies of sub-piece i: thread t takes half of row t / 2 (its slot looked up once)
    static_assert(kAThreads == 2 * kSP, "two threads per row of a sub-piece");
    auto issue = [&](int i) {
        if (i < nsub) {
            const int st = i % kAStages;
            const int r = tid >> 1, hf = tid & 1;
            const int pos = (int)pbeg + i * kSP + r;
            int64_t slot = -1;
            if (pos < pend32) {
                const int b = p.bs_shift >= 0 ? pos >> p.bs_shift : pos / p.block_size;
                if (b < p.n_table) {
                    const int32_t blk = __ldg(p.block_table + b);
                    if (blk >= 0 && blk < p.num_blocks)
                        slot = (int64_t)blk * p.block_size + (pos - b * p.block_size);
                }
                if (slot < 0 && hf == 0) raise_flag(p.dev_err, DEVFLAG_BAD_SLOT);
            }
            if (hf == 0) valid[st * kSP + r] = slot >= 0;
            uint8_t* kdst = kring + (st * kSP + r) * RP;
            uint8_t* vdst = vring + (st * kSP + r) * RP;
            const int64_t off = (slot * p.nkv + g) * (int64_t)HD;
#pragma unroll
            for (int c = 0; c < KC / 2; ++c) {
                const int pc = hf * (KC / 2) + c;
                if (slot >= 0) {
                    cp_async16(kdst + 16 * pc, p.k_cache + off + 16 * pc);
                    cp_async16(vdst + 16 * pc, p.v_cache + off + 16 * pc);
                } else {  // zeros: the weight of the row is 0, and 0 * NaN would not be
                    *reinterpret_cast<uint4*>(kdst + 16 * pc) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(vdst + 16 * pc) = make_uint4(0, 0, 0, 0);
                }
            }
        }
        cp_async_commit();  // one group per sub-piece, empty past the end
    };
    issue(0);
    issue(1);

    // the group's query heads in f16, each scaled by 2^e so its largest |q| lies in
    // [2^14, 2^15) (exact: a bf16 value has 8 significant bits); heads past G are zero
    for (int h = warp; h < kAMaxGroup; h += kAThreads / 32) {
        float mx = 0.f;
        if (h < G)
            for (int d = lane; d < HD; d += 32)
                mx = fmaxf(mx, fabsf(bf16_to_f32(p.q[(int64_t)(g * G + h) * HD + d])));
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0;
        if (mx > 0.f) e = 14 - ilogbf(mx);
        for (int d = lane; d < HD; d += 32) {
            const float v = h < G ? ldexpf(bf16_to_f32(p.q[(int64_t)(g * G + h) * HD + d]), e) : 0.f;
            qh[h * QP + d] = (uint16_t)(f32x2_to_f16x2(v, 0.f) & 0xFFFFu);
        }
        if (lane == 0) hfac[h] = ldexpf(p.qk_scale, -e);
    }

    float m_run[NT][2], l_run[NT][2], acc[MT][NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        m_run[j][0] = m_run[j][1] = -INFINITY;
        l_run[j][0] = l_run[j][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[mt][j][k] = 0.f;
    }

    for (int i = 0; i < nsub; ++i) {
        cp_async_wait<1>();  // this thread's copies of sub-piece i have landed
        __syncthreads();     // everyone's; and sub-piece i - 1 is fully consumed
        issue(i + 2);
        const int st = i % kAStages;
        const uint8_t* ks = kring + st * kSP * RP;
        const uint8_t* vs = vring + st * kSP * RP;

        // scores of positions 16 warp + [0, 16) for every head: K (A) . Q^T (B). The K
        // dimension of each MMA is permuted -- k index 2t, 2t+1 is dims 4t, 4t+1 and
        // 2t+8, 2t+9 dims 4t+2, 4t+3 of the 16-dim chunk -- in A and B alike
        float sc[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int k = 0; k < 4; ++k) sc[j][k] = 0.f;
        const uint8_t* kr0 = ks + (16 * warp + gid) * RP + 4 * tig;
#pragma unroll
        for (int c = 0; c < KC; ++c) {
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(kr0 + 16 * c);
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(kr0 + 8 * RP + 16 * c);
            const uint32_t a0 = e4m3x2_to_f16x2((uint16_t)(w0 & 0xFFFFu));
            const uint32_t a2 = e4m3x2_to_f16x2((uint16_t)(w0 >> 16));
            const uint32_t a1 = e4m3x2_to_f16x2((uint16_t)(w1 & 0xFFFFu));
            const uint32_t a3 = e4m3x2_to_f16x2((uint16_t)(w1 >> 16));
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const uint2 b = *reinterpret_cast<const uint2*>(qh + (8 * j + gid) * QP + 16 * c + 4 * tig);
                mma_f16_16816(sc[j], a0, a1, a2, a3, b.x, b.y);
            }
        }
        // scale per head; rows that are not readable score -inf
        const bool v0 = valid[st * kSP + 16 * warp + gid] != 0;
        const bool v1 = valid[st * kSP + 16 * warp + gid + 8] != 0;
        float mloc[NT][2];
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float f = hfac[8 * j + 2 * tig + e];
                sc[j][e] = v0 ? sc[j][e] * f : -INFINITY;
                sc[j][2 + e] = v1 ? sc[j][2 + e] * f : -INFINITY;
                float m = fmaxf(sc[j][e], sc[j][2 + e]);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                mloc[j][e] = m;
            }
        if (gid == 0)
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) redm[warp * kAMaxGroup + 8 * j + 2 * tig + e] = mloc[j][e];
        __syncthreads();
        // the new running maximum; weights exp(s - max) as f16 into shared memory
        // ([head][position]); their sum per warp
        float alpha[NT][2];
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int h = 8 * j + 2 * tig + e;
                const float msub = fmaxf(fmaxf(redm[h], redm[kAMaxGroup + h]),
                                         fmaxf(redm[2 * kAMaxGroup + h], redm[3 * kAMaxGroup + h]));
                const float mnew = fmaxf(m_run[j][e], msub);
                alpha[j][e] = (m_run[j][e] == -INFINITY) ? 0.f : expf(m_run[j][e] - mnew);
                m_run[j][e] = mnew;
                float lsum = 0.f;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const float s = sc[j][2 * half + e];
                    const float w = (s == -INFINITY) ? 0.f : expf(s - mnew);
                    const uint16_t wh = (uint16_t)(f32x2_to_f16x2(w, 0.f) & 0xFFFFu);
                    wsm[h * kWPitch + 16 * warp + gid + 8 * half] = wh;
                    lsum += f16x2_to_f32x2((uint32_t)wh).x;
                }
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
                if (gid == 0) redl[warp * kAMaxGroup + h] = lsum;
            }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int h = 8 * j + 2 * tig + e;
                const float ls = (redl[h] + redl[kAMaxGroup + h]) + (redl[2 * kAMaxGroup + h] + redl[3 * kAMaxGroup + h]);
                l_run[j][e] = l_run[j][e] * alpha[j][e] + ls;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    acc[mt][j][e] *= alpha[j][e];
                    acc[mt][j][2 + e] *= alpha[j][e];
                }
            }
        // the weighted V sum of dims warp * HD/4 + [0, HD/4): V^T (A) . W^T (B). The M
        // dimension is permuted (vdim below gives the dim of each tile row), so that a
        // thread's dims are one 16-bit load (one 16-dim tile) or one 32-bit load (a pair
        // of tiles) per position
#pragma unroll
        for (int kk = 0; kk < kSP / 16; ++kk) {
            const int pr = 16 * kk + 2 * tig;  // positions pr, pr + 1, pr + 8, pr + 9
            uint32_t b[NT][2];
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                b[j][0] = *reinterpret_cast<const uint32_t*>(wsm + (8 * j + gid) * kWPitch + pr);
                b[j][1] = *reinterpret_cast<const uint32_t*>(wsm + (8 * j + gid) * kWPitch + pr + 8);
            }
            if constexpr (MT % 2 == 0) {
#pragma unroll
                for (int mp = 0; mp < MT / 2; ++mp) {  // tiles 2 mp, 2 mp + 1: dims d4 .. d4 + 3
                    const int d4 = warp * (HD / 4) + 32 * mp + 4 * gid;
                    const uint32_t y0 = *reinterpret_cast<const uint32_t*>(vs + pr * RP + d4);
                    const uint32_t y1 = *reinterpret_cast<const uint32_t*>(vs + (pr + 1) * RP + d4);
                    const uint32_t y8 = *reinterpret_cast<const uint32_t*>(vs + (pr + 8) * RP + d4);
                    const uint32_t y9 = *reinterpret_cast<const uint32_t*>(vs + (pr + 9) * RP + d4);
#pragma unroll
                    for (int u = 0; u < 2; ++u) {  // dims d4 + 2u (row g), d4 + 2u + 1 (row g + 8)
                        const uint32_t s0 = 0x0040u + 0x0022u * u, s1 = s0 + 0x0011u;
                        const uint32_t a0 = e4m3x2_to_f16x2((uint16_t)__byte_perm(y0, y1, s0));
                        const uint32_t a1 = e4m3x2_to_f16x2((uint16_t)__byte_perm(y0, y1, s1));
                        const uint32_t a2 = e4m3x2_to_f16x2((uint16_t)__byte_perm(y8, y9, s0));
                        const uint32_t a3 = e4m3x2_to_f16x2((uint16_t)__byte_perm(y8, y9, s1));
#pragma unroll
                        for (int j = 0; j < NT; ++j)
                            mma_f16_16816(acc[2 * mp + u][j], a0, a1, a2, a3, b[j][0], b[j][1]);
                    }
                }
            } else {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {  // dims d0 (row g), d0 + 1 (row g + 8)
                    const int d0 = warp * (HD / 4) + 16 * mt + 2 * gid;
                    const uint32_t x0 = *reinterpret_cast<const uint16_t*>(vs + pr * RP + d0);
                    const uint32_t x1 = *reinterpret_cast<const uint16_t*>(vs + (pr + 1) * RP + d0);
                    const uint32_t x8 = *reinterpret_cast<const uint16_t*>(vs + (pr + 8) * RP + d0);
                    const uint32_t x9 = *reinterpret_cast<const uint16_t*>(vs + (pr + 9) * RP + d0);
                    const uint32_t lo = x0 | (x1 << 16), hi = x8 | (x9 << 16);
                    const uint32_t a0 = e4m3x2_to_f16x2((uint16_t)__byte_perm(lo, 0, 0x0020));
                    const uint32_t a1 = e4m3x2_to_f16x2((uint16_t)__byte_perm(lo, 0, 0x0031));
                    const uint32_t a2 = e4m3x2_to_f16x2((uint16_t)__byte_perm(hi, 0, 0x0020));
                    const uint32_t a3 = e4m3x2_to_f16x2((uint16_t)__byte_perm(hi, 0, 0x0031));
#pragma unroll
                    for (int j = 0; j < NT; ++j) mma_f16_16816(acc[mt][j], a0, a1, a2, a3, b[j][0], b[j][1]);
                }
            }
        }
    }

    // this CTA's partials: (max, sum) per head, then its dims of the weighted V sums; tile
    // mt's row g holds dim vdim(mt), row g + 8 dim vdim(mt) + 1
    auto vdim = [&](int mt) {
        return MT % 2 == 0 ? warp * (HD / 4) + 32 * (mt / 2) + 4 * gid + 2 * (mt % 2)
                           : warp * (HD / 4) + 16 * mt + 2 * gid;
    };
    const int64_t rs = (int64_t)HD + 2;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 8 * j + 2 * tig + e;
            if (h >= G) continue;
            float* dst = p.part + ((int64_t)piece * p.nq + g * G + h) * rs;
            if (warp == 0 && gid == 0) {
                dst[0] = m_run[j][e];
                dst[1] = l_run[j][e];
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int d0 = vdim(mt);
                dst[2 + d0] = acc[mt][j][e];
                dst[2 + d0 + 1] = acc[mt][j][2 + e];
            }
        }
}

// One CTA per query head: out = sum_s e^(m_s - M) acc_s / sum_s e^(m_s - M) l_s (zero
// when no row was readable), as bf16. The pieces' (max, sum) pairs are loaded in parallel
// and folded from shared memory in a fixed order; the dimensions' sums over the pieces
// are split over 256 / hd thread groups (eight loads in flight each) and added in order.
__global__ void __launch_bounds__(kAMaxHd) attn_merge_kernel(const __grid_constant__ AttnParams p) {
    __shared__ float msm[kAMaxPieces];
    __shared__ float lsm[kAMaxPieces];
    __shared__ float fac[kAMaxPieces];
    __shared__ float accp[kAMaxHd];  // [parts][hd]
    __shared__ float red[kAMaxHd / 32];
    __shared__ float tot[2];
    const int i = blockIdx.x, t = threadIdx.x, hd = p.hd;
    const int lane = t & 31, warp = t >> 5;
    const int parts = kAMaxHd / hd, d = t % hd, part = t / hd;  // 1, 2 or 4 parts of the pieces
    pdl_wait();
    const int64_t rs = (int64_t)p.nq * (hd + 2);  // floats between a head's pieces
    const float* base = p.part + (int64_t)i * (hd + 2);
    float mloc = -INFINITY;
    for (int s = t; s < p.pieces; s += kAMaxHd) {
        msm[s] = base[s * rs];
        lsm[s] = base[s * rs + 1];
        mloc = fmaxf(mloc, msm[s]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
    if (lane == 0) red[warp] = mloc;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAMaxHd / 32; ++w) M = fmaxf(M, red[w]);
    for (int s = t; s < p.pieces; s += kAMaxHd)
        fac[s] = (M == -INFINITY || msm[s] == -INFINITY) ? 0.f : expf(msm[s] - M);
    __syncthreads();
    if (warp == 0) {  // the denominator: lane-strided partial sums, then a fixed shuffle tree
        float L = 0.f;
        for (int s = lane; s < p.pieces; s += 32) L = fmaf(fac[s], lsm[s], L);
#pragma unroll
        for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (lane == 0) tot[1] = L;
    }
    // the weighted V sums: thread (part, d) takes pieces part, part + parts, ..., eight
    // loads in flight at a time; the parts are added in order afterwards
    float a = 0.f;
    int s = part;
    for (; s + 7 * parts < p.pieces; s += 8 * parts) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = base[(s + j * parts) * rs + 2 + d];
#pragma unroll
        for (int j = 0; j < 8; ++j) a = fmaf(fac[s + j * parts], v[j], a);
    }
    for (; s < p.pieces; s += parts) a = fmaf(fac[s], base[s * rs + 2 + d], a);
    accp[part * hd + d] = a;
    __syncthreads();
    if (part == 0) {
        float sum = accp[d];
        for (int q = 1; q < parts; ++q) sum += accp[q * hd + d];
        const float L = tot[1];
        p.out[(int64_t)i * hd + d] = f32_to_bf16(L > 0.f ? sum / L * p.v_scale : 0.f);
    }
}

}  // namespace

int attn_max_group() { return kAMaxGroup; }

// Pieces per kv head: as many CTAs over all kv heads as the SMs hold at once, at least one
// sub-piece each, at most kAMaxPieces; the positions per piece a multiple of kSP.
static int64_t attn_pieces_cap(int64_t seq_len) {
    const int64_t subs = (seq_len + kSP - 1) / kSP;
    return subs < kAMaxPieces ? subs : kAMaxPieces;
}

size_t attn_ws_bytes(int nq, int hd, int64_t seq_len) {
    const int64_t pieces = attn_pieces_cap(seq_len);
    return (size_t)(pieces < 1 ? 1 : pieces) * (size_t)nq * (size_t)(hd + 2) * sizeof(float);
}

template <int HD, int NT>
cudaError_t launch_pieces(const AttnParams& p, cudaStream_t s) {
    constexpr size_t smem = attn_smem_bytes<HD>();
    auto kern = attn_piece_kernel<HD, NT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)p.nkv, (unsigned)p.pieces), kAThreads, smem, s>>>(p);
    return cudaGetLastError();
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
    p.bs_shift = (block_size & (block_size - 1)) == 0 ? __builtin_ctz((unsigned)block_size) : -1;
    p.num_blocks = num_blocks;
    p.seq_len = seq_len;
    p.qk_scale = scale * k_scale;
    p.v_scale = v_scale;
    p.part = static_cast<float*>(ws);
    p.out = out;
    p.dev_err = dev_err;
    int dev = 0, sms = 148;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // as many CTAs as fit on the SMs at once (shared memory bound, at most four per SM)
    const size_t smem = hd == 64 ? attn_smem_bytes<64>() : hd == 128 ? attn_smem_bytes<128>()
                                                                      : attn_smem_bytes<256>();
    int per_sm = (int)((size_t)227 * 1024 / smem);
    per_sm = per_sm < 1 ? 1 : per_sm > 4 ? 4 : per_sm;
    int64_t pieces = ((int64_t)per_sm * sms + nkv - 1) / nkv;
    const int64_t cap = attn_pieces_cap(seq_len);
    if (pieces > cap) pieces = cap;
    const int64_t subs = (seq_len + kSP - 1) / kSP;
    p.per_piece = (int64_t)kSP * ((subs + pieces - 1) / pieces);
    p.pieces = (int)((seq_len + p.per_piece - 1) / p.per_piece);
    const bool two = p.group > 8;
    if (hd == 64) e = two ? launch_pieces<64, 2>(p, s) : launch_pieces<64, 1>(p, s);
    else if (hd == 128) e = two ? launch_pieces<128, 2>(p, s) : launch_pieces<128, 1>(p, s);
    else e = two ? launch_pieces<256, 2>(p, s) : launch_pieces<256, 1>(p, s);
    if (e != cudaSuccess) return e;
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
