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
// sub-pieces of 64 positions that a three-stage ring brings into shared memory: tensor
// copies of 16 cache rows (128-dim heads, blocks of a multiple of 16 rows), else 16-byte
// asynchronous copies; rows of a missing block are zero-filled. Warp w owns positions
// 16 w + [0, 16) of every sub-piece and runs its own online softmax (fp32 running maximum
// and sum per query head) and its own weighted V sum over all head dims, so the warps
// meet once per sub-piece (the ring) and once at the end. Both contractions run on the
// tensor cores (mma.sync m16n8k16, f16 operands, fp32 accumulators): the scores as
// K[16 positions, hd] . Q^T, with E4M3 K decoded exactly to f16 and each query head in
// f16 scaled by a power of two (exact); the weights exp(s - max) in (0, 1] (the hardware
// exponential) rounded to f16 (the same rounded weights in the sum of exps) go from the
// score accumulators to the B operand of V^T . W^T in registers (an 8 x 8 transpose,
// movmatrix). At the end the four warps' states merge in a fixed order into the CTA's
// (max, sum, weighted V sum) per head; a second kernel merges the pieces of each head in a
// fixed order (deterministic) and writes bf16. Rows whose block is missing or out of range
// are skipped and set MTP_DEVFLAG_BAD_SLOT.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace mtp {
namespace {

constexpr int kSP = 64;          // positions per sub-piece (four warps x 16)
constexpr int kAThreads = 128;
constexpr int kAStages = 3;
constexpr int kAMaxGroup = 16;  // query heads per kv head
constexpr int kAMaxPieces = 1024;  // pieces per kv head (the merge keeps a factor per piece)

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

// Transpose of an 8 x 8 matrix of 16-bit values in the mma fragment layout (lane holds
// row lane / 4, columns 2 (lane % 4) + {0, 1}).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t v) {
    uint32_t r;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

// Row pitch of a staged cache row: HD + 16 bytes with the 16-byte copies (bank-conflict
// free); HD = 128 bytes, 128-byte swizzled, with the tensor copies.
template <int HD, bool TMA>
__host__ __device__ constexpr int attn_row_pitch() { return TMA ? HD : HD + 16; }
template <int HD>
__host__ __device__ constexpr int attn_q_pitch() { return HD + 8; }     // f16 elements

template <int HD, bool TMA>
__host__ __device__ constexpr size_t attn_smem_bytes() {
    return (size_t)kAStages * 2 * kSP * attn_row_pitch<HD, TMA>()  // K and V rings
           + (size_t)kAMaxGroup * attn_q_pitch<HD>() * 2         // q in f16
           + (size_t)kAStages * kSP * 4                          // row valid flags
           + (size_t)2 * 4 * kAMaxGroup * 4                      // per-warp max and sum
           + (size_t)kAMaxGroup * 4                              // per-head score factor
           + (TMA ? (size_t)kAStages * 8 + 1024 : 0);            // stage barriers, alignment
}

__device__ __forceinline__ void tma_load_3d_attn(void* dst, const CUtensorMap* map, int x, int y, int z,
                                                 uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// TMA (HD = 128, block size a multiple of 16): warp 0 brings each sub-piece in as four
// tensor copies of 16 cache rows (one per 16 positions, each inside one block) per K and
// V, completing on the stage's barrier; rows of a missing block and past the sequence are
// zero-filled by the warp (a group cut by the sequence's end is copied row by row).
template <int HD, int NT, bool TMA>
__global__ void __launch_bounds__(kAThreads) attn_piece_kernel(const __grid_constant__ AttnParams p,
                                                               const __grid_constant__ CUtensorMap kmap,
                                                               const __grid_constant__ CUtensorMap vmap) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    static_assert(!TMA || HD == 128, "tensor copies: 128-byte rows");
    // (the tensor copies' 128-byte swizzle wants 1024-byte aligned stages)
    uint8_t* smem = TMA ? smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u) : smem_raw;
    constexpr int RP = attn_row_pitch<HD, TMA>();
    constexpr int QP = attn_q_pitch<HD>();
    constexpr int KC = HD / 16;          // 16-byte pieces of a row, and MMA K chunks
    uint8_t* kring = smem;                                          // [stages][kSP][RP]
    uint8_t* vring = kring + kAStages * kSP * RP;                   // [stages][kSP][RP]
    uint16_t* qh = reinterpret_cast<uint16_t*>(vring + kAStages * kSP * RP);  // [16][QP] f16
    int* valid = reinterpret_cast<int*>(qh + kAMaxGroup * QP);       // [stages][kSP]
    float* redm = reinterpret_cast<float*>(valid + kAStages * kSP);   // [4][16]
    float* redl = redm + 4 * kAMaxGroup;                               // [4][16]
    float* hfac = redl + 4 * kAMaxGroup;                               // [16]
    uint64_t* fullb = reinterpret_cast<uint64_t*>(hfac + kAMaxGroup);  // [stages] (TMA)
    // byte offset of 16-byte chunk c of staged row r (the swizzle of the tensor copies)
    auto chunk_at = [](int r, int c) -> int { return TMA ? r * RP + ((c ^ (r & 7)) << 4) : r * RP + (c << 4); };

    static_assert((size_t)kAStages * 2 * kSP * RP >= (size_t)4 * kAMaxGroup * HD * 4,
                  "the ring holds the warps' sums at the end");
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
    // copies of sub-piece i: thread t takes half of row t / 2 (its slot looked up once).
    // The block-table entry of the thread's row in the next sub-piece is loaded one issue
    // ahead, so that its latency is not paid in front of the copies.
    static_assert(kAThreads == 2 * kSP, "two threads per row of a sub-piece");
    auto load_blk = [&](int i) -> int32_t {  // -1: no readable block (or past the piece)
        const int pos = (int)pbeg + i * kSP + (tid >> 1);
        if (i >= nsub || pos >= pend32) return -1;
        const int b = p.bs_shift >= 0 ? pos >> p.bs_shift : pos / p.block_size;
        return b < p.n_table ? __ldg(p.block_table + b) : -1;
    };
    int32_t blk_next = load_blk(0);
    auto issue_cp = [&](int i) {
        const int32_t blk = blk_next;
        blk_next = load_blk(i + 1);
        if (i < nsub) {
            const int st = i % kAStages;
            const int r = tid >> 1, hf = tid & 1;
            const int pos = (int)pbeg + i * kSP + r;
            int64_t slot = -1;
            if (pos < pend32) {
                const int b = p.bs_shift >= 0 ? pos >> p.bs_shift : pos / p.block_size;
                if (b < p.n_table && blk >= 0 && blk < p.num_blocks)
                    slot = (int64_t)blk * p.block_size + (pos - b * p.block_size);
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
    if (TMA && tid == 0) {
        for (int b = 0; b < kAStages; ++b) mbar_init(&fullb[b], 1);
        mbar_fence_init();
    }
    if (TMA) __syncthreads();
    // tensor copies of sub-piece i (warp 0): lane q < 4 takes positions 16 q + [0, 16)
    auto issue_tma = [&](int i) {
        if (i >= nsub) return;
        const int st = i % kAStages;
        const int pos0 = (int)pbeg + i * kSP + 16 * (lane & 3);
        const int nv = lane < 4 ? max(0, min(16, pend32 - pos0)) : 0;  // rows before the end
        int row0 = -1;                                                  // first cache row
        if (nv > 0) {
            const int b = p.bs_shift >= 0 ? pos0 >> p.bs_shift : pos0 / p.block_size;
            const int32_t blk = b < p.n_table ? __ldg(p.block_table + b) : -1;
            if (blk >= 0 && blk < p.num_blocks) row0 = blk * p.block_size + (pos0 - b * p.block_size);
            else raise_flag(p.dev_err, DEVFLAG_BAD_SLOT);
        }
        const uint32_t whole = __ballot_sync(0xffffffffu, nv == 16 && row0 >= 0);  // groups by tensor copy
        uint8_t* kst = kring + st * kSP * RP;
        uint8_t* vst = vring + st * kSP * RP;
        // the other groups: zeros, and the readable rows of a group cut by the end
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            if ((whole >> q) & 1u) continue;
            const int qnv = __shfl_sync(0xffffffffu, nv, q);
            const int qrow = __shfl_sync(0xffffffffu, row0, q);
            for (int u = lane; u < 16 * KC; u += 32) {  // 16 rows x KC chunks
                const int r = u / KC, c = u - r * KC;
                uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
                if (qrow >= 0 && r < qnv) {
                    const int64_t off = ((int64_t)(qrow + r) * p.nkv + g) * HD + 16 * c;
                    kv = *reinterpret_cast<const uint4*>(p.k_cache + off);
                    vv = *reinterpret_cast<const uint4*>(p.v_cache + off);
                }
                *reinterpret_cast<uint4*>(kst + chunk_at(16 * q + r, c)) = kv;
                *reinterpret_cast<uint4*>(vst + chunk_at(16 * q + r, c)) = vv;
            }
        }
        // row valid flags: row 16 q + j of the sub-piece
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = lane + 32 * h, q = r >> 4;
            const int qnv = __shfl_sync(0xffffffffu, nv, q);
            const int qrow = __shfl_sync(0xffffffffu, row0, q);
            valid[st * kSP + r] = qrow >= 0 && (r & 15) < qnv;
        }
        __syncwarp();  // the warp's stores above, before the barrier's arrival below
        // (and every earlier access to the stage through plain loads and stores ordered
        // before the tensor copies rewrite it)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (lane == 0) mbar_arrive_expect_tx(&fullb[st], (uint32_t)__popc(whole) * 2u * 16u * HD);
        __syncwarp();
        if ((whole >> lane) & 1u) {
            tma_load_3d_attn(kst + 16 * lane * RP, &kmap, 0, g, row0, &fullb[st]);
            tma_load_3d_attn(vst + 16 * lane * RP, &vmap, 0, g, row0, &fullb[st]);
        }
    };
    auto issue = [&](int i) {
        if constexpr (TMA) {
            if (warp == 0) issue_tma(i);
        } else {
            issue_cp(i);
        }
    };
    for (int i = 0; i < kAStages - 1; ++i) issue(i);

    // the group's query heads in f16, each scaled by 2^e so its largest |q| lies in
    // [2^14, 2^15) (exact: a bf16 value has 8 significant bits); heads past G are zero.
    // Warp w takes heads 4 w .. 4 w + 3: lane l holds 8 dims of head 4 w + k HPL + l / LH,
    // all loads issued at once, each head's maximum folded over its LH lanes (q 16-byte
    // aligned; else one head at a time)
    if ((reinterpret_cast<uintptr_t>(p.q) & 15u) == 0) {
        constexpr int LH = HD / 8, HPL = 32 / LH, NL = 4 / HPL;
        static_assert(kAMaxGroup == 4 * (kAThreads / 32) && 4 % HPL == 0, "four heads per warp");
        uint4 qr[NL];
#pragma unroll
        for (int k = 0; k < NL; ++k) {
            const int h = 4 * warp + k * HPL + lane / LH;
            qr[k] = h < G ? *reinterpret_cast<const uint4*>(p.q + (int64_t)(g * G + h) * HD + 8 * (lane % LH))
                          : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < NL; ++k) {
            const int h = 4 * warp + k * HPL + lane / LH;
            const uint32_t w[4] = {qr[k].x, qr[k].y, qr[k].z, qr[k].w};
            float mx = 0.f;
#pragma unroll
            for (int t = 0; t < 4; ++t) mx = fmaxf(mx, fmaxf(fabsf(bf16_lo(w[t])), fabsf(bf16_hi(w[t]))));
#pragma unroll
            for (int o = LH / 2; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            int e = 0;
            if (mx > 0.f) e = 14 - ilogbf(mx);
            uint4 o4;
            o4.x = f32x2_to_f16x2(ldexpf(bf16_lo(w[0]), e), ldexpf(bf16_hi(w[0]), e));
            o4.y = f32x2_to_f16x2(ldexpf(bf16_lo(w[1]), e), ldexpf(bf16_hi(w[1]), e));
            o4.z = f32x2_to_f16x2(ldexpf(bf16_lo(w[2]), e), ldexpf(bf16_hi(w[2]), e));
            o4.w = f32x2_to_f16x2(ldexpf(bf16_lo(w[3]), e), ldexpf(bf16_hi(w[3]), e));
            *reinterpret_cast<uint4*>(qh + h * QP + 8 * (lane % LH)) = o4;
            if (lane % LH == 0) hfac[h] = ldexpf(p.qk_scale, -e);
        }
    } else {
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
    }

    // Each warp runs its own online softmax over its 16 positions of every sub-piece
    // (positions 16 warp + [0, 16)) and its own weighted V sum over all hd dims; the four
    // warps' states merge once, at the end. Lane (gid, tig) holds heads 8 j + 2 tig + e.
    constexpr int DT = HD / 16;  // 16-dim tiles of the weighted V sum
    float m_run[NT][2], l_run[NT][2], acc[DT][NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        m_run[j][0] = m_run[j][1] = -INFINITY;
        l_run[j][0] = l_run[j][1] = 0.f;  // this lane's positions' weights (summed at the end)
#pragma unroll
        for (int dt = 0; dt < DT; ++dt)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[dt][j][k] = 0.f;
    }

    for (int i = 0; i < nsub; ++i) {
        if constexpr (TMA) {
            if (!mbar_wait_bounded(&fullb[i % kAStages], (uint32_t)((i / kAStages) & 1), nullptr) && tid == 0)
                raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
        } else {
            cp_async_wait<kAStages - 2>();  // this thread's copies of sub-piece i have landed
        }
        __syncthreads();  // everyone's; and sub-piece i - 1 is fully consumed
        issue(i + kAStages - 1);
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
        const int kr = 16 * warp + gid;
#pragma unroll
        for (int c = 0; c < KC; ++c) {
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(ks + chunk_at(kr, c) + 4 * tig);
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(ks + chunk_at(kr + 8, c) + 4 * tig);
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
        // scale per head; rows that are not readable score -inf. The warp's running
        // maximum per head; weights exp(s - max) rounded to f16 (the same rounded weights
        // in the sum of exps), packed per position as (head 2 tig, head 2 tig + 1) and
        // transposed (movmatrix) into the B fragments of the V sum: (positions, head gid)
        const bool v0 = valid[st * kSP + 16 * warp + gid] != 0;
        const bool v1 = valid[st * kSP + 16 * warp + gid + 8] != 0;
        uint32_t bp[NT][2];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            uint16_t wl[2], wh[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float f = hfac[8 * j + 2 * tig + e];
                const float s0 = v0 ? sc[j][e] * f : -INFINITY;
                const float s1 = v1 ? sc[j][2 + e] * f : -INFINITY;
                float m = fmaxf(s0, s1);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                const float mnew = fmaxf(m_run[j][e], m);
                // (the hardware exponential: its ~1e-6 relative error is far below the f16
                // rounding of the weights)
                const float alpha = (m_run[j][e] == -INFINITY) ? 0.f : __expf(m_run[j][e] - mnew);
                m_run[j][e] = mnew;
                const float w0 = (s0 == -INFINITY) ? 0.f : __expf(s0 - mnew);
                const float w1 = (s1 == -INFINITY) ? 0.f : __expf(s1 - mnew);
                const uint32_t hw = f32x2_to_f16x2(w0, w1);  // (position gid, position gid + 8)
                wl[e] = (uint16_t)(hw & 0xFFFFu);
                wh[e] = (uint16_t)(hw >> 16);
                const float2 wf = f16x2_to_f32x2(hw);
                l_run[j][e] = l_run[j][e] * alpha + (wf.x + wf.y);
#pragma unroll
                for (int dt = 0; dt < DT; ++dt) {
                    acc[dt][j][e] *= alpha;
                    acc[dt][j][2 + e] *= alpha;
                }
            }
            bp[j][0] = movmatrix_trans((uint32_t)wl[0] | ((uint32_t)wl[1] << 16));
            bp[j][1] = movmatrix_trans((uint32_t)wh[0] | ((uint32_t)wh[1] << 16));
        }
        // the weighted V sum over the warp's 16 positions, all dims: V^T (A) . W^T (B). The
        // M dimension is permuted: tile 2 mp + u has dim 32 mp + 4 gid + 2 u in row gid and
        // the next dim in row gid + 8, so a thread's dims are one 32-bit load per position
        const int pr = 16 * warp + 2 * tig;  // positions pr, pr + 1, pr + 8, pr + 9
#pragma unroll
        for (int mp = 0; mp < HD / 32; ++mp) {
            const int vc = 2 * mp + (gid >> 2), vo = 4 * (gid & 3);  // chunk, byte in it
            const uint32_t y0 = *reinterpret_cast<const uint32_t*>(vs + chunk_at(pr, vc) + vo);
            const uint32_t y1 = *reinterpret_cast<const uint32_t*>(vs + chunk_at(pr + 1, vc) + vo);
            const uint32_t y8 = *reinterpret_cast<const uint32_t*>(vs + chunk_at(pr + 8, vc) + vo);
            const uint32_t y9 = *reinterpret_cast<const uint32_t*>(vs + chunk_at(pr + 9, vc) + vo);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t s0 = 0x0040u + 0x0022u * u, s1 = s0 + 0x0011u;
                const uint32_t a0 = e4m3x2_to_f16x2((uint16_t)__byte_perm(y0, y1, s0));
                const uint32_t a1 = e4m3x2_to_f16x2((uint16_t)__byte_perm(y0, y1, s1));
                const uint32_t a2 = e4m3x2_to_f16x2((uint16_t)__byte_perm(y8, y9, s0));
                const uint32_t a3 = e4m3x2_to_f16x2((uint16_t)__byte_perm(y8, y9, s1));
#pragma unroll
                for (int j = 0; j < NT; ++j) mma_f16_16816(acc[2 * mp + u][j], a0, a1, a2, a3, bp[j][0], bp[j][1]);
            }
        }
    }

    // merge the four warps (fixed order) into this CTA's partials: per head the largest
    // warp maximum M, sum_w e^(m_w - M) l_w and sum_w e^(m_w - M) acc_w; tile dt's row gid
    // holds dim vdim(dt), row gid + 8 dim vdim(dt) + 1
    auto vdim = [&](int dt) { return 32 * (dt / 2) + 4 * gid + 2 * (dt % 2); };
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) l_run[j][e] += __shfl_xor_sync(0xffffffffu, l_run[j][e], o);
    __syncthreads();  // every warp is past the ring: it holds the warps' sums from here
    float* accs = reinterpret_cast<float*>(kring);  // [4 warps][kAMaxGroup heads][HD]
    if (gid == 0)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                redm[warp * kAMaxGroup + 8 * j + 2 * tig + e] = m_run[j][e];
                redl[warp * kAMaxGroup + 8 * j + 2 * tig + e] = l_run[j][e];
            }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int h = 8 * j + 2 * tig + e;
            const float M = fmaxf(fmaxf(redm[h], redm[kAMaxGroup + h]),
                                  fmaxf(redm[2 * kAMaxGroup + h], redm[3 * kAMaxGroup + h]));
            const float f = (m_run[j][e] == -INFINITY) ? 0.f : expf(m_run[j][e] - M);
            float* dst = accs + (warp * kAMaxGroup + h) * HD;
#pragma unroll
            for (int dt = 0; dt < DT; ++dt) {
                const int d0 = vdim(dt);
                dst[d0] = acc[dt][j][e] * f;
                dst[d0 + 1] = acc[dt][j][2 + e] * f;
            }
        }
    __syncthreads();
    const int64_t rs = (int64_t)HD + 2;
    for (int idx = tid; idx < G * HD; idx += kAThreads) {
        const int h = idx / HD, d = idx - h * HD;
        const float v = ((accs[h * HD + d] + accs[(kAMaxGroup + h) * HD + d]) +
                         accs[(2 * kAMaxGroup + h) * HD + d]) +
                        accs[(3 * kAMaxGroup + h) * HD + d];
        p.part[((int64_t)piece * p.nq + g * G + h) * rs + 2 + d] = v;
    }
    for (int h = tid; h < G; h += kAThreads) {
        float M = -INFINITY;
        for (int w = 0; w < 4; ++w) M = fmaxf(M, redm[w * kAMaxGroup + h]);
        float L = 0.f;
        for (int w = 0; w < 4; ++w) {
            const float mw = redm[w * kAMaxGroup + h];
            L += (mw == -INFINITY) ? 0.f : expf(mw - M) * redl[w * kAMaxGroup + h];
        }
        float* dst = p.part + ((int64_t)piece * p.nq + g * G + h) * rs;
        dst[0] = M;
        dst[1] = L;
    }
}

constexpr int kMThreads = 1024;  // merge: hd-thread groups, each a share of the pieces

// One CTA per query head: out = sum_s e^(m_s - M) acc_s / sum_s e^(m_s - M) l_s (zero
// when no row was readable), as bf16. The pieces' (max, sum) pairs are loaded in parallel
// and folded from shared memory in a fixed order; the dimensions' sums over the pieces
// are split over 1024 / hd thread groups (eight loads in flight each) and added in order.
__global__ void __launch_bounds__(kMThreads) attn_merge_kernel(const __grid_constant__ AttnParams p) {
    __shared__ float msm[kAMaxPieces];
    __shared__ float lsm[kAMaxPieces];
    __shared__ float fac[kAMaxPieces];
    __shared__ float accp[kMThreads];  // [parts][hd]
    __shared__ float red[kMThreads / 32];
    __shared__ float tot[2];
    const int i = blockIdx.x, t = threadIdx.x, hd = p.hd;
    const int lane = t & 31, warp = t >> 5;
    const int parts = kMThreads / hd, d = t % hd, part = t / hd;  // 4, 8 or 16 parts of the pieces
    pdl_wait();
    const int64_t rs = (int64_t)p.nq * (hd + 2);  // floats between a head's pieces
    const float* base = p.part + (int64_t)i * (hd + 2);
    float mloc = -INFINITY;
    for (int s = t; s < p.pieces; s += kMThreads) {
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
    for (int w = 0; w < kMThreads / 32; ++w) M = fmaxf(M, red[w]);
    for (int s = t; s < p.pieces; s += kMThreads)
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

template <int HD, int NT, bool TMA>
cudaError_t launch_pieces(const AttnParams& p, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          cudaStream_t s) {
    constexpr size_t smem = attn_smem_bytes<HD, TMA>();
    auto kern = attn_piece_kernel<HD, NT, TMA>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)p.nkv, (unsigned)p.pieces), kAThreads, smem, s>>>(p, kmap, vmap);
    return cudaGetLastError();
}

typedef CUresult (*AttnEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                 CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                 CUtensorMapFloatOOBfill);

AttnEncodeFn attn_encode_fn() {
    static AttnEncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AttnEncodeFn>(f);
    });
    return fn;
}

// A cache [num_blocks * block_size rows][nkv][128] E4M3 as a 3-D tensor (byte of the head
// row, kv head, cache row); boxes of 128 bytes x 1 head x 16 rows, 128-byte swizzle.
bool attn_cache_map(CUtensorMap* m, const uint8_t* base, int nkv, int64_t rows) {
    AttnEncodeFn fn = attn_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)nkv, (cuuint64_t)rows};
    cuuint64_t strides[2] = {128, (cuuint64_t)nkv * 128};
    cuuint32_t box[3] = {128, 1, 16};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
    // tensor copies for 128-dim heads in blocks of a multiple of 16 rows (16-byte aligned
    // caches, cache rows addressable as 32-bit coordinates); 16-byte copies otherwise
    CUtensorMap kmap{}, vmap{};
    const int64_t cache_rows = num_blocks * (int64_t)block_size;
    const bool tma = hd == 128 && block_size % 16 == 0 && cache_rows < ((int64_t)1 << 31) &&
                     (reinterpret_cast<uintptr_t>(k_cache) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(v_cache) & 15) == 0 &&
                     attn_cache_map(&kmap, k_cache, nkv, cache_rows) &&
                     attn_cache_map(&vmap, v_cache, nkv, cache_rows);
    // as many CTAs as fit on the SMs at once (shared memory bound, at most four per SM)
    const size_t smem = tma ? attn_smem_bytes<128, true>()
                            : hd == 64 ? attn_smem_bytes<64, false>()
                                       : hd == 128 ? attn_smem_bytes<128, false>() : attn_smem_bytes<256, false>();
    int per_sm = (int)((size_t)227 * 1024 / smem);
    per_sm = per_sm < 1 ? 1 : per_sm > 4 ? 4 : per_sm;
    int64_t pieces = ((int64_t)per_sm * sms + nkv - 1) / nkv;
    const int64_t cap = attn_pieces_cap(seq_len);
    if (pieces > cap) pieces = cap;
    const int64_t subs = (seq_len + kSP - 1) / kSP;
    p.per_piece = (int64_t)kSP * ((subs + pieces - 1) / pieces);
    p.pieces = (int)((seq_len + p.per_piece - 1) / p.per_piece);
    const bool two = p.group > 8;
    if (tma) e = two ? launch_pieces<128, 2, true>(p, kmap, vmap, s) : launch_pieces<128, 1, true>(p, kmap, vmap, s);
    else if (hd == 64) e = two ? launch_pieces<64, 2, false>(p, kmap, vmap, s) : launch_pieces<64, 1, false>(p, kmap, vmap, s);
    else if (hd == 128) e = two ? launch_pieces<128, 2, false>(p, kmap, vmap, s) : launch_pieces<128, 1, false>(p, kmap, vmap, s);
    else e = two ? launch_pieces<256, 2, false>(p, kmap, vmap, s) : launch_pieces<256, 1, false>(p, kmap, vmap, s);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)nq);
    cfg.blockDim = dim3(kMThreads);
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
