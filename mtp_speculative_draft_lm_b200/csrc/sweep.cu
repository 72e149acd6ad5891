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
// Design (B200, HBM-bound): one persistent CTA per SM. Tiles of 16 table rows are
// handed out at run time: CTA b starts with tile b, then takes the next tile from an
// atomic counter in the workspace, so SMs that stream faster take more tiles (per-SM
// HBM throughput varies by ~20%; a fixed split leaves a long tail). A producer warp
// claims tiles one ahead and streams each through a shared-memory ring with ONE TMA
// tensor copy per stage -- 16 rows x up to 32 128-byte segments (64 KB), written with
// the 128-byte swizzle, plus one copy of the NVFP4 block scales -- completing on an
// mbarrier; each stage carries its tile index, and a stage tagged -1 ends the CTA's
// work. Large copies matter: the TMA unit's per-copy cost caps a ring fed by 1 KB row
// copies at about half of HBM bandwidth. Out-of-range rows and K tails arrive as
// zeros (tensor-map bounds). Sixteen compute warps (eight for the combiner past eight
// inputs) split each stage's K range into slabs of 4 lanes x 16 B per row, decode the
// codes exactly into
// f16/bf16 fragments and run tensor-core MMAs with 16 table rows as the A operand and
// up to 16 inputs as the B operand (swap-AB). MMA row g reads table row s(g) of the
// tile, a fixed permutation that, with the swizzle, makes every shared-memory read
// conflict-free. E4M3 codes and E2M1 codes times their E4M3 block scale are exact in
// f16; NVFP4 with one or two inputs instead keeps the codes unscaled and applies the
// block scales to per-block fp32 sums (see slab_mma_blocks). x is staged once per CTA
// (bf16 for BF16 tables; f16 scaled by a per-row power of two for quantized tables,
// undone in fp32), so the only roundings are fp32 ones. At the end of a tile each
// compute warp hands its partial to a reducer warp through a double-buffered shared
// slot (mbarrier hand-off, no CTA-wide barrier on the streaming path). The reducer
// sums the partials in a fixed warp order (deterministic and independent of M),
// scales, masks and keeps per lane a running (max, lowest row); the 16 row slots are
// folded once per CTA. Tiles whose 16 rows are masked out for every input are neither
// loaded nor computed. Each CTA publishes its partial and takes a ticket; the last CTA
// (no waiting) folds all partials with 32 lanes and re-zeroes the ticket and the tile
// counter. The launch allows programmatic dependent launch: the next kernel in the
// stream may set up and start streaming its own table while this grid finishes, and
// this kernel waits for the previous grid before reading x, masks or the workspace.
// Every mbarrier wait is bounded: a wait that runs out sets an abort flag and
// MTP_DEVFLAG_TIMEOUT, and the kernel runs to its end.
// More inputs than this design serves well (BF16 from 9, FP8 from 7) go to the tcgen05
// sweep further down; NVFP4 from 3 inputs to the block-scaled FP4 sweep (3-16) and the
// tcgen05 sweep with A in tensor memory (17-32).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace mtp {
namespace {

constexpr int kTileRows = 16;
constexpr int kPartSlots = 32;  // partials per CTA (one per input, up to 32 inputs)
constexpr int kMaxGrid = 1024;
constexpr int kMaxStages = 12;
constexpr int kMaxSegs = 32;  // 128-byte segments of a row per stage (box of 16 rows x 4 KB)
constexpr int kSmemLimit = 227 * 1024;
// Gathered (masked) sweep: rows claimed per hand-out (8 mask words per input), the
// producer's queue of allowed rows, and the shared-memory ints it adds.
constexpr int kGatherRows = 256;
constexpr int kGatherQueue = 64;  // a power of two above 15 + 32
constexpr int kGatherInts = kGatherQueue + kMaxStages * 16 + 2 * 16;

// Warp roles: CW compute warps, then one reducer warp, then one producer warp.
// M <= 8 uses 16 compute warps; M > 8 uses 8, which leaves shared memory for the
// larger staged input.
template <int NT> struct Roles {
    static constexpr int CW = NT == 1 ? 16 : 8;
    static constexpr int THREADS = (CW + 2) * 32;
    static constexpr int RED_COLS = 8 * NT;
};

// A CTA's result for one input: the allowed maximum, its lowest row, and the sum of
// exp(l - v) over the allowed rows it saw (for the top-1 log-probability).
struct Partial {
    float v;
    int32_t i;
    float s;
    float pad;
};

// Merges (v2, s2) into (v, s): sums of exp(l - max) over two row sets.
__device__ __forceinline__ void lse_merge(float& v, float& s, float v2, float s2) {
    const float m = fmaxf(v, v2);
    if (m == -INFINITY) return;
    s = s * expf(v - m) + s2 * expf(v2 - m);
    v = m;
}

// V: K elements per 16-byte piece of codes. A slab is 64 bytes of one row (4 lanes x
// 16 B, 4V elements); a stage holds `segs` 128-byte segments (2 * segs slabs) of each
// of the tile's 16 rows, plus for NVFP4 the matching 16 * segs block-scale bytes.
template <int FMT> struct Fmt;
template <> struct Fmt<0> { static constexpr int V = 8; };
template <> struct Fmt<1> { static constexpr int V = 16; };
template <> struct Fmt<2> { static constexpr int V = 32; };

__host__ __device__ inline int code_stage_bytes(int segs) { return kTileRows * 128 * segs; }
__host__ __device__ inline int scale_stage_bytes(int segs) { return kTileRows * 16 * segs; }
__host__ __device__ inline int stage_bytes_for(int fmt, int segs, bool gather = false) {
    // a gathered stage skews its 16 rows by 16 bytes each
    int b = code_stage_bytes(segs) + (gather ? kTileRows * 16 : 0) +
            (fmt == 2 ? scale_stage_bytes(segs) : 0);
    return (b + 1023) & ~1023;
}

// MMA row g of a tile reads table row s(g) (a bijection on 0..15 with s(g+8) = s(g)+8).
__device__ __forceinline__ int tile_row(int g) { return (g & 8) | ((g & 1) << 2) | ((g >> 1) & 3); }

// Byte offset of a logical byte inside a stage written by a 128-byte-swizzled box of
// 128-byte segments: 16-byte chunk bits [4:6] are XORed with bits [7:9].
__device__ __forceinline__ uint32_t swz(uint32_t logical) {
    return logical ^ (((logical >> 7) & 7u) << 4);
}

// 3-D / 2-D TMA tensor loads into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Pulls this CTA's 1/gridDim share of [base, base + bytes) into L2 (bulk prefetches of
// whole 16-byte units inside the range; the ragged ends are left to demand loads).
__device__ __forceinline__ void l2_prefetch_share(const void* base, int64_t bytes) {
    uint64_t g;
    asm("cvta.to.global.u64 %0, %1;" : "=l"(g) : "l"(base));
    const uint64_t lo = (g + 15u) & ~(uint64_t)15u;
    const uint64_t hi = (g + (uint64_t)bytes) & ~(uint64_t)15u;
    if (bytes <= 0 || hi <= lo) return;
    const uint64_t per = ((hi - lo) / gridDim.x + 16u) & ~(uint64_t)15u;
    uint64_t a = lo + per * blockIdx.x;
    const uint64_t e = a + per < hi ? a + per : hi;
    while (a < e) {
        const uint64_t piece = e - a < 65536u ? e - a : 65536u;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"((uint32_t)piece)
                     : "memory");
        a += piece;
    }
}

// Mask bit of table row `row` (token row + row_offset: a vocab shard reads the global mask).
__device__ __forceinline__ bool mask_allows(const SweepParams& p, int m, int64_t row) {
    if (!p.mask) return true;
    const int64_t t = row + p.row_offset;
    int64_t word = t >> 5;
    if (word >= p.mask_words) return false;
    uint32_t bits = (uint32_t)__ldg(p.mask + (int64_t)m * p.mask_stride + word);
    return (bits >> (t & 31)) & 1u;
}

// Gathered sweep: the mask words of a claimed range of kGatherRows rows. Lane l loads
// word (l % 8) of the range for inputs l / 8 and l / 8 + 4 (two words each, since a vocab
// shard's rows start at any token), issued early; gather_union consumes them.
__device__ __forceinline__ void gather_mask_load(const SweepParams& p, int64_t claim, int lane,
                                                 uint32_t (&w)[4]) {
    const int64_t t0 = claim * kGatherRows + (lane & 7) * 32 + p.row_offset;
    const int64_t wi = t0 >> 5;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int m = (lane >> 3) + 4 * j;
        w[2 * j] = w[2 * j + 1] = 0u;
        if (m >= p.M) continue;
        const int32_t* row = p.mask + (int64_t)m * p.mask_stride;
        if (wi < p.mask_words) w[2 * j] = (uint32_t)__ldg(row + wi);
        if ((t0 & 31) != 0 && wi + 1 < p.mask_words) w[2 * j + 1] = (uint32_t)__ldg(row + wi + 1);
    }
}

// The OR over the inputs of the allowed bits of rows claim * kGatherRows + 32 j + [0, 32),
// rows at or past n cleared; lane j (j < 8) returns word j (whole warp).
__device__ __forceinline__ uint32_t gather_union(const SweepParams& p, int64_t claim, int lane,
                                                 const uint32_t (&w)[4]) {
    const int64_t row0 = claim * kGatherRows + (lane & 7) * 32;
    const int sh = (int)((row0 + p.row_offset) & 31);
    uint32_t v = 0u;
#pragma unroll
    for (int j = 0; j < 2; ++j)
        v |= (uint32_t)((((uint64_t)w[2 * j + 1] << 32) | w[2 * j]) >> sh);
    v |= __shfl_xor_sync(0xffffffffu, v, 8);
    v |= __shfl_xor_sync(0xffffffffu, v, 16);
    const int64_t rows = p.n - row0;
    if (rows < 32) v &= rows > 0 ? (1u << rows) - 1u : 0u;
    return v;
}

// Reductions over the CW compute warps (named barrier 1).
template <int CW>
__device__ __forceinline__ float compute_sum(float v, float* scratch) {
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    named_sync(1, CW * 32);
    if (lane == 0) scratch[warp] = v;
    named_sync(1, CW * 32);
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < CW; ++w) t += scratch[w];
    return t;
}

template <int CW>
__device__ __forceinline__ float compute_max(float v, float* scratch) {
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    named_sync(1, CW * 32);
    if (lane == 0) scratch[warp] = v;
    named_sync(1, CW * 32);
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < CW; ++w) t = fmaxf(t, scratch[w]);
    return t;
}

// Stage x (bf16) into xs[m][0..K): a copy (mode 0) or the combiner's concat
// [bf16(rms(e) w_e) || bf16(rms(hidden) w_h)] (mode 1). Compute warps only.
template <int MODE, int CW>
__device__ void stage_bf16(const SweepParams& p, uint16_t* xs, float* scratch) {
    constexpr int NTH = CW * 32;
    const int tid = threadIdx.x;
    const int64_t K = p.k;
    if (MODE == 0) {
        const int vecs = (int)(K / 8);
        for (int i = tid; i < p.M * vecs; i += NTH) {
            int m = i / vecs, v = i - m * vecs;
            uint4 val = *reinterpret_cast<const uint4*>(p.x + (int64_t)m * K + (int64_t)v * 8);
            *reinterpret_cast<uint4*>(xs + (int64_t)m * p.kpad + (int64_t)v * 8) = val;
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
            for (int j = tid; j < h; j += NTH) {
                float ev = e ? bf16_to_f32(e[j]) : 0.f;
                float xv = bf16_to_f32(hx[j]);
                se += ev * ev;
                sx += xv * xv;
            }
            se = compute_sum<CW>(se, scratch);
            sx = compute_sum<CW>(sx, scratch + CW);
            float inv_e = 1.0f / sqrtf(se / (float)h + p.eps);
            float inv_x = 1.0f / sqrtf(sx / (float)h + p.eps);
            const float add = p.norm_mode ? 1.f : 0.f;  // weights w or 1 + w
            uint16_t* row = xs + (int64_t)m * p.kpad;
            for (int j = tid; j < h; j += NTH) {
                float ev = e ? bf16_to_f32(e[j]) : 0.f;
                row[j] = f32_to_bf16(ev * inv_e * (bf16_to_f32(p.w_norm_embed[j]) + add));
                row[h + j] = f32_to_bf16(bf16_to_f32(hx[j]) * inv_x *
                                         (bf16_to_f32(p.w_norm_hidden[j]) + add));
            }
        }
    }
    named_sync(1, NTH);
}

// Quantized tables: rescale each staged row by 2^e_m (largest |x| lands in
// [2^14, 2^15)) and convert it in place to f16. Exact for every element within
// 2^29 of the row maximum; the power of two is undone on the fp32 logit.
template <int CW>
__device__ void stage_to_f16(const SweepParams& p, uint16_t* xs, int* xexp, float* scratch) {
    constexpr int NTH = CW * 32;
    const int tid = threadIdx.x;
    const int K = (int)p.k;
    for (int m = 0; m < p.M; ++m) {
        uint16_t* row = xs + (int64_t)m * p.kpad;
        float a = 0.f;
        for (int j = tid; j < K; j += NTH) a = fmaxf(a, fabsf(bf16_to_f32(row[j])));
        a = compute_max<CW>(a, scratch);
        int ex = 0;
        if (a > 0.f) frexpf(a, &ex);
        int e = (a > 0.f) ? 15 - ex : 0;
        if (tid == 0) xexp[m] = e;
        // 2^e as two factors, each a normal float: the product is exact whenever the
        // result is a normal float, and a result below that is zero in f16 anyway
        const float f1 = ldexpf(1.f, e / 2), f2 = ldexpf(1.f, e - e / 2);
        for (int j = tid; j < K; j += NTH) row[j] = f32_to_f16((bf16_to_f32(row[j]) * f1) * f2);
        named_sync(1, NTH);
    }
}

// Quantized tables with one or two inputs, mode 0: x read once from global memory into
// registers (up to 4 x 8 elements per thread per input), one block-wide max per input,
// then written to shared memory directly as f16 scaled by 2^e_m (the same scaling as
// stage_bf16 + stage_to_f16). Returns false (nothing done) when K is too long for it.
template <int CW>
__device__ bool stage_x_f16_direct(const SweepParams& p, uint16_t* xs, int* xexp, float* part) {
    constexpr int NTH = CW * 32, MAXV = 4;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = (int)p.k, vecs = K / 8, M = p.M;
    if (M > 2 || vecs > MAXV * NTH) return false;
    uint4 r[2][MAXV];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < MAXV; ++j) {
            const int i = tid + j * NTH;
            r[m][j] = make_uint4(0, 0, 0, 0);
            if (m < M && i < vecs) {
                r[m][j] = *reinterpret_cast<const uint4*>(p.x + (int64_t)m * K + (int64_t)i * 8);
                const uint32_t w[4] = {r[m][j].x, r[m][j].y, r[m][j].z, r[m][j].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    a = fmaxf(a, fabsf(bf16_to_f32((uint16_t)(w[q] & 0xFFFFu))));
                    a = fmaxf(a, fabsf(bf16_to_f32((uint16_t)(w[q] >> 16))));
                }
            }
        }
        for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (lane == 0) part[m * CW + warp] = a;
    }
    named_sync(1, NTH);
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        if (m >= M) break;
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < CW; ++w) a = fmaxf(a, part[m * CW + w]);
        int ex = 0;
        if (a > 0.f) frexpf(a, &ex);
        const int e = (a > 0.f) ? 15 - ex : 0;
        if (tid == 0) xexp[m] = e;
        const float f1 = ldexpf(1.f, e / 2), f2 = ldexpf(1.f, e - e / 2);
        uint16_t* row = xs + (int64_t)m * p.kpad;
#pragma unroll
        for (int j = 0; j < MAXV; ++j) {
            const int i = tid + j * NTH;
            if (i < vecs) {
                const uint32_t w[4] = {r[m][j].x, r[m][j].y, r[m][j].z, r[m][j].w};
                uint32_t o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t lo = f32_to_f16((bf16_to_f32((uint16_t)(w[q] & 0xFFFFu)) * f1) * f2);
                    const uint32_t hi = f32_to_f16((bf16_to_f32((uint16_t)(w[q] >> 16)) * f1) * f2);
                    o[q] = lo | (hi << 16);
                }
                *reinterpret_cast<uint4*>(row + (int64_t)i * 8) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
    named_sync(1, NTH);
    return true;
}

// One slab: per lane 16 B of codes of table rows r0 (at cw) and r0 + 8 (at cw + r8: 1 KB,
// the next 8-row swizzle atom, in a tensor-box stage; eight row pitches in a gathered
// stage), K elements [e0, e0 + V) for lane c, against the staged
// inputs at x0 (input row g) and x1 (input row g + 8). For NVFP4, sw points at the
// lane's two block scales of row r0 and sw + spitch8 at those of row r0 + 8. The
// accumulator set (mma index & 1) alternates to split the dependence chain.
template <int FMT, int NT>
__device__ __forceinline__ void slab_mma(float (&acc)[2][NT][4], const uint8_t* cw, uint32_t r8,
                                         const uint8_t* sw, uint32_t spitch8,
                                         const uint16_t* x0, const uint16_t* x1, bool l0,
                                         bool l1) {
    const uint4 ra = lds128(cw);
    const uint4 rb = lds128(cw + r8);
    const uint4 z = make_uint4(0, 0, 0, 0);
    if (FMT == 0) {
        const uint4 xa = l0 ? lds128(x0) : z;
        mma_bf16_16816(acc[0][0], ra.x, rb.x, ra.y, rb.y, xa.x, xa.y);
        mma_bf16_16816(acc[1][0], ra.z, rb.z, ra.w, rb.w, xa.z, xa.w);
        if (NT > 1) {
            const uint4 xb = l1 ? lds128(x1) : z;
            mma_bf16_16816(acc[0][NT - 1], ra.x, rb.x, ra.y, rb.y, xb.x, xb.y);
            mma_bf16_16816(acc[1][NT - 1], ra.z, rb.z, ra.w, rb.w, xb.z, xb.w);
        }
    } else if (FMT == 1) {
        const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
        const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
        const uint4 xa0 = l0 ? lds128(x0) : z;
        const uint4 xa1 = l0 ? lds128(x0 + 8) : z;
        const uint32_t xa[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
        uint32_t xb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (NT > 1) {
            const uint4 xb0 = l1 ? lds128(x1) : z;
            const uint4 xb1 = l1 ? lds128(x1 + 8) : z;
            xb[0] = xb0.x; xb[1] = xb0.y; xb[2] = xb0.z; xb[3] = xb0.w;
            xb[4] = xb1.x; xb[5] = xb1.y; xb[6] = xb1.z; xb[7] = xb1.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t a0 = e4m3x2_to_f16x2((uint16_t)(wa[i] & 0xFFFFu));
            const uint32_t a2 = e4m3x2_to_f16x2((uint16_t)(wa[i] >> 16));
            const uint32_t a1 = e4m3x2_to_f16x2((uint16_t)(wb[i] & 0xFFFFu));
            const uint32_t a3 = e4m3x2_to_f16x2((uint16_t)(wb[i] >> 16));
            mma_f16_16816(acc[i & 1][0], a0, a1, a2, a3, xa[2 * i], xa[2 * i + 1]);
            if (NT > 1) mma_f16_16816(acc[i & 1][NT - 1], a0, a1, a2, a3, xb[2 * i], xb[2 * i + 1]);
        }
    } else {
        const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
        const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
        // block scales of rows r0 / r0+8: blocks 2c (words 0,1) and 2c+1 (words 2,3)
        const uint16_t s0v = *reinterpret_cast<const uint16_t*>(sw);
        const uint16_t s1v = *reinterpret_cast<const uint16_t*>(sw + spitch8);
        const uint32_t sa = e4m3x2_to_f16x2(s0v);
        const uint32_t sb = e4m3x2_to_f16x2(s1v);
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
            for (int q = 0; q < 4; ++q) {
                qa[q] = hmul2(qa[q], s_a);
                qb[q] = hmul2(qb[q], s_b);
            }
            const uint4 xv = l0 ? lds128(x0 + 8 * i) : z;
            mma_f16_16816(acc[0][0], qa[0], qb[0], qa[1], qb[1], xv.x, xv.y);
            mma_f16_16816(acc[1][0], qa[2], qb[2], qa[3], qb[3], xv.z, xv.w);
            if (NT > 1) {
                const uint4 xw = l1 ? lds128(x1 + 8 * i) : z;
                mma_f16_16816(acc[0][NT - 1], qa[0], qb[0], qa[1], qb[1], xw.x, xw.y);
                mma_f16_16816(acc[1][NT - 1], qa[2], qb[2], qa[3], qb[3], xw.z, xw.w);
            }
        }
    }
}

// NVFP4 with one or two inputs: the block scale moves out of the fragments. An MMA's
// k = 16 covers four elements of each lane group c, and lane group c's elements in
// MMAs 0-3 of the slab all belong to block 2c of the slab, in MMAs 4-7 to block 2c + 1.
// B is block-diagonal over the lane groups: column 4m + j holds input m on the k of
// lane group j and zero elsewhere, so D0 (MMAs 0-3) and D1 (MMAs 4-7) hold, per row,
// the unscaled E2M1 x input dot products of each block separately (products exact,
// fp32 sums). The lane holding D columns 2c + e (e = 0, 1; lane group j = 2(c % 2) + e)
// then adds s(block 2j) D0 + s(block 2j + 1) D1 for rows r0 and r0 + 8 in fp32: eight
// FFMAs per slab instead of 32 f16 scale multiplies. sw4 points at the row-r0 scale
// bytes of blocks 4(c % 2) .. 4(c % 2) + 3 of the slab, sw4 + spitch8 at row r0 + 8's.
// xv: the lane's B registers; lanes that feed no input (lx false) keep them zero.
__device__ __forceinline__ void slab_mma_blocks(float (&acc)[4], uint4 (&xv)[4], const uint8_t* cw,
                                                uint32_t r8, const uint8_t* sw4, uint32_t spitch8,
                                                const uint16_t* xp, bool lx) {
    const uint4 ra = lds128(cw);
    const uint4 rb = lds128(cw + r8);
    const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
    const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
    if (lx) {
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[i] = lds128(xp + 8 * i);
    }
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t qa[4], qb[4];
        e2m1x8_to_f16x2x4(wa[i], qa);
        e2m1x8_to_f16x2x4(wb[i], qb);
        float(&d)[4] = i < 2 ? d0 : d1;
        mma_f16_16816(d, qa[0], qb[0], qa[1], qb[1], xv[i].x, xv[i].y);
        mma_f16_16816(d, qa[2], qb[2], qa[3], qb[3], xv[i].z, xv[i].w);
    }
    const uint32_t sa = *reinterpret_cast<const uint32_t*>(sw4);
    const uint32_t sb = *reinterpret_cast<const uint32_t*>(sw4 + spitch8);
    const float2 a01 = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)(sa & 0xFFFFu)));
    const float2 a23 = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)(sa >> 16)));
    const float2 b01 = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)(sb & 0xFFFFu)));
    const float2 b23 = f16x2_to_f32x2(e4m3x2_to_f16x2((uint16_t)(sb >> 16)));
    acc[0] = fmaf(a01.y, d1[0], fmaf(a01.x, d0[0], acc[0]));
    acc[1] = fmaf(a23.y, d1[1], fmaf(a23.x, d0[1], acc[1]));
    acc[2] = fmaf(b01.y, d1[2], fmaf(b01.x, d0[2], acc[2]));
    acc[3] = fmaf(b23.y, d1[3], fmaf(b23.x, d0[3], acc[3]));
}

// After a CTA has published its partials: take a ticket (release before, acquire after);
// the last CTA folds every CTA's partials in a fixed pattern and writes the outputs (or,
// for a vocab shard, the shard's partial), then re-zeroes the ticket and the tile counter.
__device__ void ticket_and_fold(const SweepParams& p, int lane, bool lp) {
    const int M = p.M;
    const Partial* parts = reinterpret_cast<const Partial*>(p.partials);
    int last = 0;
    if (lane == 0) last = atom_add_acq_rel_gpu(p.ticket, 1u) == gridDim.x - 1;
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    fence_acq_rel_gpu();
    // the last CTA folds every CTA's partial: lane l reads CTAs l, l + 32, ...
    // (independent loads in flight together), then a shuffle reduction; ties go
    // to the lowest row index, so the result does not depend on the order
    const int G = (int)gridDim.x;
    constexpr int FOLD = 8;  // partials per lane in flight at a time
    for (int m = 0; m < M; ++m) {
        float bv = -INFINITY, bs = 0.f;
        int32_t bi = INT_MAX;
        for (int base = 0; base < G; base += 32 * FOLD) {
            float qv[FOLD], qs[FOLD];
            int32_t qi[FOLD];
#pragma unroll
            for (int j = 0; j < FOLD; ++j) {
                const int b = base + lane + 32 * j;
                qv[j] = -INFINITY;
                qi[j] = INT_MAX;
                qs[j] = 0.f;
                if (b < G) {
                    const float4 e = __ldcg(reinterpret_cast<const float4*>(parts + (int64_t)b * kPartSlots + m));
                    qv[j] = e.x;
                    qi[j] = __float_as_int(e.y);
                    qs[j] = e.z;
                }
            }
#pragma unroll
            for (int j = 0; j < FOLD; ++j) {
                if (lp) {
                    float v = bv;
                    lse_merge(v, bs, qv[j], qs[j]);
                }
                if (qv[j] > bv || (qv[j] == bv && qi[j] < bi)) {
                    bv = qv[j];
                    bi = qi[j];
                }
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
            const float os = __shfl_xor_sync(0xffffffffu, bs, o);
            if (lp) {
                float v = bv;
                lse_merge(v, bs, ov, os);
            }
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if (lane == 0 && p.out_partial) {
            // a vocab shard: the global row of its maximum (INT_MAX: nothing allowed here)
            const int32_t gi = bi == INT_MAX ? INT_MAX : (int32_t)(bi + p.row_offset);
            reinterpret_cast<Partial*>(p.out_partial)[m] = Partial{bv, gi, bs, 0.f};
        } else if (lane == 0) {
            const bool empty = bi == INT_MAX;
            if (empty) {
                bi = 0;
                bv = -INFINITY;
                raise_flag(p.dev_err, DEVFLAG_EMPTY_MASK);
            }
            p.out_idx[m] = bi;
            if (p.out_val) p.out_val[m] = bv;
            // the maximum's own term is exp(0) = 1, so bs >= 1 and the result is <= 0
            if (lp) p.out_logprob[m] = empty ? -INFINITY : -logf(bs);
        }
    }
    __syncwarp();
    if (lane == 0) {  // leave the workspace ready for the next call
        p.ticket[0] = 0u;
        p.ticket[1] = 0u;
    }
}

template <int FMT, int NT, int MODE, int BD, int G>
__global__ void __launch_bounds__(Roles<NT>::THREADS, 1)
    sweep_kernel(const __grid_constant__ SweepParams p, const __grid_constant__ CUtensorMap map_codes,
                 const __grid_constant__ CUtensorMap map_scales) {
    constexpr int V = Fmt<FMT>::V;
    constexpr int SLAB = 4 * V;  // K elements of one slab
    constexpr int CW = Roles<NT>::CW;
    constexpr int RED_COLS = Roles<NT>::RED_COLS;
    constexpr int RED_WARP_FLOATS = kTileRows * RED_COLS;
    constexpr int REDUCER = CW, PRODUCER = CW + 1;
    static_assert(G == 0 || MODE == 0, "the gathered sweep is an argmax sweep");

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* red_full = empty + kMaxStages;  // [2]
    uint64_t* red_empty = red_full + 2;       // [2]
    // misc: [0] abort, [2..17] xexp, [18..29] tile of each ring slot, [30..31] tile of
    // each reducer buffer (-1: no more tiles)
    int* misc = reinterpret_cast<int*>(red_empty + 2);
    volatile int* abort_flag = misc;
    int* xexp = misc + 2;
    volatile int* slot_tile = misc + 18;
    volatile int* red_tile = misc + 30;
    float* red = reinterpret_cast<float*>(misc + 32);  // [2][CW][16][RED_COLS]
    float* scratch = red + 2 * CW * RED_WARP_FLOATS;   // [32]
    // gathered sweep: the producer's queue of allowed rows [256], the 16 table rows of
    // each ring slot's tile [kMaxStages][16] (-1: an unused row slot), and those of each
    // reducer buffer [2][16]
    int* gq = reinterpret_cast<int*>(scratch + 32);
    volatile int* slot_rows = gq + kGatherQueue;
    volatile int* red_rows = slot_rows + kMaxStages * kTileRows;
    uint16_t* xs = reinterpret_cast<uint16_t*>(scratch + 32 + (G ? kGatherInts : 0));
    // the ring starts on a 1 KB boundary of the shared window (the 128-byte swizzle atom)
    const uint32_t head_end = smem_u32(xs) + (uint32_t)p.M * (uint32_t)p.kpad * 2u;
    uint8_t* ring = smem + (((head_end + 1023u) & ~1023u) - smem_u32(smem));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t K = p.k;
    const int S = p.stages;
    const int stage_bytes = p.stage_bytes;
    const int segs = p.segs;                   // 128-byte segments per row per stage
    const int slabs_per_stage = 2 * segs;
    const int NC = p.stages_per_tile;          // ceil(row segments / segs)
    const int M = p.M;
    // a gathered stage holds row j's segments at j * gpitch (a 16-byte skew between rows
    // keeps the compute warps' reads conflict-free without a swizzle); its block scales
    // follow the 16 rows
    const uint32_t gpitch = (uint32_t)segs * 128u + 16u;
    const uint32_t code_area = G ? (uint32_t)kTileRows * gpitch : (uint32_t)code_stage_bytes(segs);

    // Tiles are handed out at run time (mode 0): CTA b starts with tile b, then takes
    // gridDim.x + (a counter in the workspace, post-incremented), so SMs that stream
    // faster take more tiles. Mode 1 (no workspace) splits the tiles evenly up front.
    // The gathered sweep hands out ranges of kGatherRows table rows the same way.
    const int64_t T = p.num_tiles;
    const bool dyn = MODE == 0;
    const int64_t t_begin = dyn ? blockIdx.x : (T * blockIdx.x) / gridDim.x;
    const int64_t t_end = dyn ? T : (T * (blockIdx.x + 1)) / gridDim.x;
    static_assert(kMaxStages <= 12, "slot_tile holds 12 entries");

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CW);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&red_full[b], CW);
            mbar_init(&red_empty[b], 1);
        }
        misc[0] = 0;
        mbar_fence_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    // ------------------------------------------------------------ producer warp
    if (warp == PRODUCER) {
        int slot = 0;
        uint32_t phase = 0;
        int64_t issued = 0;
        const uint32_t tx = code_stage_bytes(segs) + (FMT == 2 ? scale_stage_bytes(segs) : 0);
        bool stop = false;
        if (!G) {
            // the NC stages of one tile, each tagged with the tile
            auto issue_tile = [&](int64_t tile) {
                for (int ch = 0; ch < NC; ++ch) {
                    if (!mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag)) {
                        stop = true;
                        return;
                    }
                    if (lane == 0) {
                        uint8_t* dst = ring + (size_t)slot * stage_bytes;
                        slot_tile[slot] = (int)tile;
                        mbar_arrive_expect_tx(&full[slot], tx);
                        tma_load_3d(dst, &map_codes, 0, (int)(tile * kTileRows), ch * segs, &full[slot]);
                        if (FMT == 2)
                            tma_load_2d(dst + code_stage_bytes(segs), &map_scales, ch * 8 * segs,
                                        (int)(tile * kTileRows), &full[slot]);
                    }
                    __syncwarp();
                    ++issued;
                    if (++slot == S) {
                        slot = 0;
                        phase ^= 1u;
                    }
                }
            };
            // The first tile's stages read only the table, so they go out before waiting
            // for the previous grid. The next tile is claimed one tile ahead, so the
            // atomic's latency overlaps the waits for free ring slots.
            int64_t tile = t_begin;
            int64_t pending = 0;
            if (tile < t_end) issue_tile(tile);
            pdl_wait();
            if (dyn && lane == 0) pending = (int64_t)gridDim.x + atomicAdd(p.ticket + 1, 1u);
            while (!stop) {
                tile = dyn ? __shfl_sync(0xffffffffu, pending, 0) : tile + 1;
                if (tile >= t_end) break;
                if (dyn && lane == 0) pending = (int64_t)gridDim.x + atomicAdd(p.ticket + 1, 1u);
                issue_tile(tile);
            }
        } else {
            // Gathered sweep (a grammar mask): only rows that some input's mask allows are
            // read. Each claimed range of kGatherRows rows is scanned (the OR of the
            // inputs' mask words), its allowed rows join a queue in increasing order, and
            // every 16 queued rows become one tile whose rows are fetched by one bulk copy
            // each (their codes, plus for NVFP4 their block scales). The mask may be
            // written by the previous grid, so everything waits for it.
            const int row_segs = (int)(p.row_bytes / 128);
            int qhead = 0, qtail = 0;  // queue positions (warp-uniform; entries mod 256)
            int64_t vtile = 0;         // tiles issued (the tag a stage carries)
            auto issue_gtile = [&](int cnt) {
                const int myrow = lane < cnt ? gq[(qhead + lane) & (kGatherQueue - 1)] : -1;
                for (int ch = 0; ch < NC && !stop; ++ch) {
                    if (!mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    const int seg0 = ch * segs;
                    const int nseg = min(segs, row_segs - seg0);
                    const uint32_t cbytes = (uint32_t)nseg * 128u;
                    const uint32_t sbytes = FMT == 2 ? (uint32_t)nseg * 16u : 0u;
                    uint8_t* dst = ring + (size_t)slot * stage_bytes;
                    if (lane < kTileRows) slot_rows[slot * kTileRows + lane] = myrow;
                    __syncwarp();
                    if (lane == 0) {
                        slot_tile[slot] = (int)vtile;
                        mbar_arrive_expect_tx(&full[slot], (uint32_t)cnt * (cbytes + sbytes));
                    }
                    __syncwarp();
                    if (lane < cnt) {
                        bulk_copy_g2s(dst + lane * gpitch,
                                      p.w + (int64_t)myrow * p.row_bytes + (int64_t)seg0 * 128,
                                      cbytes, &full[slot]);
                        if (FMT == 2)
                            bulk_copy_g2s(dst + code_area + lane * 16u * (uint32_t)segs,
                                          p.block_scale + (int64_t)myrow * p.scale_pitch +
                                              (int64_t)seg0 * 16,
                                          sbytes, &full[slot]);
                    }
                    __syncwarp();
                    ++issued;
                    if (++slot == S) {
                        slot = 0;
                        phase ^= 1u;
                    }
                }
                qhead += cnt;
                ++vtile;
            };
            pdl_wait();
            int64_t claim = t_begin;
            int64_t pending = 0;
            if (lane == 0) pending = (int64_t)gridDim.x + atomicAdd(p.ticket + 1, 1u);
            uint32_t wc[4];
            gather_mask_load(p, claim, lane, wc);
            while (claim < t_end && !stop) {
                // claim the next range and start loading its mask words before this one
                // is scanned
                const int64_t cnext = __shfl_sync(0xffffffffu, pending, 0);
                if (lane == 0 && cnext < t_end) pending = (int64_t)gridDim.x + atomicAdd(p.ticket + 1, 1u);
                uint32_t wn[4] = {0u, 0u, 0u, 0u};
                if (cnext < t_end) gather_mask_load(p, cnext, lane, wn);
                const uint32_t u = gather_union(p, claim, lane, wc);  // lanes 0..7: words
#pragma unroll 1
                for (int w = 0; w < kGatherRows / 32; ++w) {
                    const uint32_t uw = __shfl_sync(0xffffffffu, u, w);
                    const int64_t row = claim * kGatherRows + w * 32 + lane;
                    const bool bit = (uw >> lane) & 1u;
                    const uint32_t bal = __ballot_sync(0xffffffffu, bit);
                    if (bit) gq[(qtail + __popc(bal & ((1u << lane) - 1u))) & (kGatherQueue - 1)] = (int)row;
                    qtail += __popc(bal);
                    if (!bit && p.out_logits && row < p.n)  // masked out for every input
                        for (int m = 0; m < M; ++m) p.out_logits[(int64_t)m * p.n + row] = 0xFF80u;
                    // drain whole tiles after every word: at most 15 + 32 rows stay queued
                    __syncwarp();
                    while (qtail - qhead >= kTileRows && !stop) issue_gtile(kTileRows);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) wc[j] = wn[j];
                claim = cnext;
            }
            if (!stop && qtail > qhead) issue_gtile(qtail - qhead);  // the CTA's last rows
        }
        // Leave no copy in flight: wait for the last stages issued (bounded). This comes
        // before the end marker, which advances the phase of a slot these waits name.
        for (int64_t j = issued > S ? issued - S : 0; j < issued; ++j)
            if (!mbar_wait_bounded(&full[j % S], (uint32_t)((j / S) & 1), nullptr)) break;
        // end of the CTA's tiles: a stage tagged -1 (an arrival with no copy)
        if (!stop && mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag) && lane == 0) {
            slot_tile[slot] = -1;
            mbar_arrive(&full[slot]);
        }
        __syncwarp();
        return;
    }

    // ------------------------------------------------------------ reducer warp
    if (warp == REDUCER) {
        // lane holds items (row = lane & 15, col = 2q + (lane >> 4)) for q < RED_COLS/2 and
        // keeps, per item, the running (max, lowest row) over the CTA's tiles; the 16 lanes
        // of a column are folded once, after the last tile
        constexpr int Q = RED_COLS / 2;
        float best_v[Q];
        int32_t best_i[Q];
        float fa[Q], fb[Q];  // 2^-xexp as two factors: (a fa) fb is exact for a normal result
        float se[Q];         // sum of exp(l - best_v) over the allowed rows seen
        const bool lp = MODE == 0 && (p.out_logprob != nullptr || p.out_partial != nullptr);
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            best_v[q] = -INFINITY;
            best_i[q] = INT_MAX;
            fa[q] = fb[q] = 1.f;
            se[q] = 0.f;
        }
        const int rrow = lane & 15;
        pdl_wait();
        const float gsc = FMT == 2 ? __ldg(p.global_scale) : 1.f;
        bool have_f = FMT == 0;
        // The row scales and the mask words are read per tile in an order known only at
        // run time: each CTA first pulls its share of them into L2.
        if (lane == 0) {
            if (FMT == 1) l2_prefetch_share(p.row_scale, p.n * 4);
            if (MODE == 0 && p.mask) l2_prefetch_share(p.mask, ((p.M - 1) * p.mask_stride + p.mask_words) * 4);
        }
        int buf = 0;
        uint32_t fph = 0u;  // bit b: phase parity of red_full[b]
        while (true) {
            if (!mbar_wait_bounded(&red_full[buf], (fph >> buf) & 1u, abort_flag)) break;
            fph ^= 1u << buf;
            const int tile_id = red_tile[buf];
            if (tile_id < 0) break;
            const int64_t tile = tile_id;
            // a gathered tile names its rows (-1: an unused row slot)
            const int64_t row = G ? (int64_t)red_rows[buf * kTileRows + rrow] : tile * kTileRows + rrow;
            const bool rvalid = row >= 0 && row < p.n;
            const float rs = (FMT == 1 && rvalid) ? __ldg(p.row_scale + row) : 0.f;
            if (!have_f) {  // xexp is visible once the first partials have arrived
#pragma unroll
                for (int q = 0; q < Q; ++q) {
                    const int col = 2 * q + (lane >> 4);
                    const int e = col < M ? -xexp[col] : 0;
                    fa[q] = ldexpf(1.f, e / 2);
                    fb[q] = ldexpf(1.f, e - e / 2);
                }
                have_f = true;
            }
            const float* rb = red + (size_t)buf * CW * RED_WARP_FLOATS;
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const int col = 2 * q + (lane >> 4);
                if (2 * q >= M) break;  // warp-uniform
                float a = 0.f;
                if (CW == 16) {
#pragma unroll
                    for (int w = 0; w < 8; ++w)
                        a += rb[w * RED_WARP_FLOATS + rrow * RED_COLS + col] +
                             rb[(w + 8) * RED_WARP_FLOATS + rrow * RED_COLS + col];
                } else {
#pragma unroll
                    for (int w = 0; w < CW; ++w) a += rb[w * RED_WARP_FLOATS + rrow * RED_COLS + col];
                }
                const bool valid = rvalid && col < M;
                float l = a;
                if (FMT != 0) l = (l * fa[q]) * fb[q];
                if (FMT == 1) l *= rs;
                if (FMT == 2) l *= gsc;
                if (MODE == 1) {
                    if (valid) p.out_y[(int64_t)col * p.n + row] = f32_to_bf16(l);
                } else {
                    const bool ok = valid && mask_allows(p, col, row);
                    if (valid && p.out_logits)
                        p.out_logits[(int64_t)col * p.n + row] = ok ? f32_to_bf16(l) : (uint16_t)0xFF80u;
                    if (lp && ok && l > -INFINITY) {
                        float v = best_v[q];
                        lse_merge(v, se[q], l, 1.f);
                    }
                    // rows arrive in increasing order, so the lowest row wins a tie
                    if (ok && (l > best_v[q] || (l == best_v[q] && best_i[q] == INT_MAX))) {
                        best_v[q] = l;
                        best_i[q] = (int32_t)row;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_empty[buf]);
            buf ^= 1;
        }
        if (*abort_flag) raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
        if (MODE == 1) return;

        // fold the 16 row slots of each column (lanes sharing lane >> 4)
#pragma unroll
        for (int q = 0; q < Q; ++q) {
#pragma unroll
            for (int o = 8; o; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, best_v[q], o);
                const int32_t oi = __shfl_xor_sync(0xffffffffu, best_i[q], o);
                const float os = __shfl_xor_sync(0xffffffffu, se[q], o);
                if (lp) {
                    float v = best_v[q];
                    lse_merge(v, se[q], ov, os);
                }
                if (ov > best_v[q] || (ov == best_v[q] && oi < best_i[q])) {
                    best_v[q] = ov;
                    best_i[q] = oi;
                }
            }
        }
        // lane 0 publishes the CTA's partials (columns 2q from itself, 2q + 1 from lane
        // 16), then takes a ticket: release before it, acquire after it
        Partial* parts = reinterpret_cast<Partial*>(p.partials);
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const float ov = __shfl_sync(0xffffffffu, best_v[q], 16);
            const int32_t oi = __shfl_sync(0xffffffffu, best_i[q], 16);
            const float os = __shfl_sync(0xffffffffu, se[q], 16);
            if (lane == 0 && 2 * q < M)
                parts[(int64_t)blockIdx.x * kPartSlots + 2 * q] = Partial{best_v[q], best_i[q], se[q], 0.f};
            if (lane == 0 && 2 * q + 1 < M)
                parts[(int64_t)blockIdx.x * kPartSlots + 2 * q + 1] = Partial{ov, oi, os, 0.f};
        }
        ticket_and_fold(p, lane, lp);
        return;
    }

    // ------------------------------------------------------------ compute warps
    const int g = lane >> 2, c = lane & 3;
    pdl_wait();
    if (!(MODE == 0 && FMT != 0 && stage_x_f16_direct<CW>(p, xs, xexp, red))) {
        stage_bf16<MODE, CW>(p, xs, scratch);
        if (FMT != 0) stage_to_f16<CW>(p, xs, xexp, scratch);
    }

    const bool xg0 = g < M;
    const bool xg1 = NT > 1 && (8 + g) < M;
    const int r0 = tile_row(g);  // table rows r0 and r0 + 8 of the tile feed MMA rows g, g+8

    // Per-lane offsets inside a stage. Slab l of a stage is 64 bytes of each row: segment
    // l / 2 (a 2 KB block of 16 rows x 128 B), half l % 2. With the 128-byte swizzle the
    // lane's 16-byte chunk of row r0 sits at r0 * 128 + ((64 (l % 2) + 16 c) ^ 16 (r0 % 8));
    // row r0 + 8 is 1 KB further on. A gathered stage keeps each row whole instead (row j
    // at j * gpitch, segment l / 2 at 128 (l / 2) within it); the 16-byte skew of gpitch
    // spreads the 8 rows x 4 chunks of a read over all banks. Block scales: [16 rows]
    // [16 segs bytes], unswizzled, after the codes.
    const uint32_t xr = (uint32_t)(r0 & 7) << 4;
    const uint32_t coff0 = G ? (uint32_t)r0 * gpitch + (uint32_t)c * 16u
                             : (uint32_t)r0 * 128u + (((uint32_t)c * 16u) ^ xr);
    const uint32_t coff1 = G ? (uint32_t)r0 * gpitch + 64u + (uint32_t)c * 16u
                             : (uint32_t)r0 * 128u + ((64u + (uint32_t)c * 16u) ^ xr);
    const uint32_t seg_stride = G ? 128u : 2048u;  // bytes between a row's segments
    const uint32_t r8 = G ? 8u * gpitch : 1024u;   // row r0 + 8 relative to row r0
    const uint32_t spitch = 16u * (uint32_t)segs;
    const uint32_t soff = code_area + (uint32_t)r0 * spitch + 2u * (uint32_t)c;
    const uint16_t* xrow0 = xs + g * p.kpad + c * V;
    const uint16_t* xrow1 = xs + (8 + g) * p.kpad + c * V;
    const int total_slabs = (int)(K / SLAB);  // K is a whole number of slabs
    // per-block scaling (NVFP4, M <= 2): lane (g, c) feeds B column g, which is input
    // g / 4 on lane group g % 4, so only lanes with g % 4 == c load an input
    const bool xbd = (g & 3) == c && (g >> 2) < M;
    const uint16_t* xrowb = xs + (g >> 2) * p.kpad + c * V;
    const uint32_t soffb = code_area + (uint32_t)r0 * spitch + 4u * (uint32_t)(c & 1);
    float accb[4] = {0.f, 0.f, 0.f, 0.f};
    uint4 xvb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xvb[i] = make_uint4(0, 0, 0, 0);

    // Accumulation chains follow the absolute slab index a (64-byte column block of
    // the row): chain a % 16 takes slabs in increasing a. With 16 compute warps warp w
    // owns chain w; with 8, warp w owns chains w and w + 8. The same chains, summed
    // in the same order, whatever M, the warp count or the stage geometry.
    constexpr int CH = CW == 16 ? 1 : 2;
    float acc[CH][2][NT][4];
#pragma unroll
    for (int j = 0; j < CH; ++j)
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[j][a][t][i] = 0.f;

    int buf = 0;
    uint32_t eph = 0u;  // bit b: phase parity of red_empty[b]
    int slot = 0;
    uint32_t phase = 0;

    while (true) {
        // the stages of one tile arrive in order; a stage tagged -1 ends the CTA's work
        if (!mbar_wait_bounded(&full[slot], phase, abort_flag)) break;
        const int tile = slot_tile[slot];
        if (tile < 0) break;
        // gathered sweep: the table row behind row slot `lane` of this tile (warp 0 hands
        // the tile's rows to the reducer)
        const int vrow = (G && warp == 0 && lane < kTileRows) ? slot_rows[slot * kTileRows + lane] : -1;
        for (int ch = 0; ch < NC; ++ch) {
            if (ch > 0 && !mbar_wait_bounded(&full[slot], phase, abort_flag)) break;
            const uint8_t* st = ring + (size_t)slot * stage_bytes;
            const int a0 = ch * slabs_per_stage;  // absolute slab index of the stage's first slab
            const int nv = min(slabs_per_stage, total_slabs - a0);  // slabs inside the row
            // this warp's slabs in the stage: l = a - a0 with a % CW == warp
            int l = (warp - a0) & (CW - 1);
            const uint8_t* cw = st + (l >> 1) * seg_stride + ((l & 1) ? coff1 : coff0);
            const uint32_t cstep = (CW / 2) * seg_stride;  // l += CW moves CW / 2 segments
            const uint8_t* sw = st + soff + l * 8;
            int xo = (a0 + l) * SLAB;
            if (BD) {
                const uint8_t* swb = st + soffb + l * 8;
                for (; l < nv; l += CW, cw += cstep, swb += CW * 8, xo += CW * SLAB)
                    slab_mma_blocks(accb, xvb, cw, r8, swb, 8u * spitch, xrowb + xo, xbd);
            } else {
                for (; l < nv; l += CW, cw += cstep, sw += CW * 8, xo += CW * SLAB) {
                    if (CH == 2 && (((a0 + l) >> 3) & 1))
                        slab_mma<FMT, NT>(acc[CH - 1], cw, r8, sw, 8u * spitch, xrow0 + xo, xrow1 + xo, xg0, xg1);
                    else
                        slab_mma<FMT, NT>(acc[0], cw, r8, sw, 8u * spitch, xrow0 + xo, xrow1 + xo, xg0, xg1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
            if (++slot == S) {
                slot = 0;
                phase ^= 1u;
            }
        }
        // hand this warp's partial of the tile to the reducer (double-buffered). The
        // summation order is fixed: a chain's partial is acc[0] + acc[1]; chains w and
        // w + 8 are added first (here when one warp owns both, by the reducer
        // otherwise), then the eight pair sums in order of w.
        mbar_wait_bounded(&red_empty[buf], ((eph >> buf) & 1u) ^ 1u, abort_flag);
        eph ^= 1u << buf;
        float* rp = red + (size_t)buf * CW * RED_WARP_FLOATS + warp * RED_WARP_FLOATS;
        if (BD) {
            // input m's logit part: lane groups 0, 1 (lane c = 2m) plus 2, 3 (lane 2m + 1)
            const float v0 = accb[0] + accb[1], v1 = accb[2] + accb[3];
            const float u0 = __shfl_xor_sync(0xffffffffu, v0, 1);
            const float u1 = __shfl_xor_sync(0xffffffffu, v1, 1);
            if ((c & 1) == 0) {
                rp[r0 * RED_COLS + (c >> 1)] = v0 + u0;
                rp[(r0 + 8) * RED_COLS + (c >> 1)] = v1 + u1;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) accb[i] = 0.f;
        }
#pragma unroll
        for (int t = 0; t < (BD ? 0 : NT); ++t) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v = acc[0][0][t][i] + acc[0][1][t][i];
                if (CH == 2) v = v + (acc[CH - 1][0][t][i] + acc[CH - 1][1][t][i]);
                const int row = (i < 2 ? r0 : r0 + 8);
                rp[row * RED_COLS + t * 8 + 2 * c + (i & 1)] = v;
#pragma unroll
                for (int j = 0; j < CH; ++j) acc[j][0][t][i] = acc[j][1][t][i] = 0.f;
            }
        }
        if (warp == 0 && lane == 0) red_tile[buf] = tile;
        if (G && warp == 0 && lane < kTileRows) red_rows[buf * kTileRows + lane] = vrow;
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_full[buf]);
        buf ^= 1;
    }
    // tell the reducer there are no more tiles
    if (mbar_wait_bounded(&red_empty[buf], ((eph >> buf) & 1u) ^ 1u, abort_flag)) {
        if (warp == 0 && lane == 0) red_tile[buf] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&red_full[buf]);
    }
}

// ---------------------------------------------------------------- tcgen05 sweep
// BF16 and FP8 tables with 9-32 inputs run the contraction on the tcgen05 tensor cores:
// one 128 x N x k MMA per 16 (BF16) or 32 (FP8) elements of K, with 128 table rows as A
// and the N = 16 or 32 (padded) inputs as B, both read by the tensor core straight from
// the TMA-written stage (K-major, 128-byte swizzle), the fp32 accumulator in tensor
// memory. Nothing is decoded: FP8 codes are E4M3 operands as stored. x enters FP8 MMAs as
// two E4M3 terms, hi = e4m3(x 2^e) and lo = e4m3(x 2^e - hi) (one B operand of 2N rows;
// the two dot products are added in fp32 in the epilogue), with e_m chosen per input
// so that its largest |x| lands in [128, 256); hi + lo equals x 2^e exactly wherever
// x 2^e >= 1/4 (a bf16 value has 8 significant bits, hi keeps 4 and the rest fits lo's 4),
// and within 2^-10 below that, i.e. within 2^-17 of the input's largest |x|.
// Roles: warp 0 streams stages (128 table rows x segs 128-byte segments, plus the inputs'
// same K range) through an mbarrier ring; warp 1 allocates tensor memory, issues the
// MMAs from one thread and releases each stage with tcgen05.commit; warps 2-5 (tensor
// memory lane quarters warp % 4) read the accumulator, one table row per thread, scale,
// mask, keep per input a running (max, lowest row, sum of exp) and write the optional
// logits. Two accumulators alternate so the MMAs of a tile overlap the previous tile's
// epilogue. Tiles of 128 rows are handed out at run time as in the narrow sweep; the CTA
// partials are folded by the last CTA (ticket_and_fold).
constexpr int kTRows = 128;     // table rows per tile: the MMA's M
constexpr int kTThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kTEpiWarps = 4;

__host__ __device__ inline int tc_x_rows(int fmt, int N) { return fmt == 1 ? 2 * N : N; }
__host__ __device__ inline int tc_stage_bytes(int fmt, int N, int segs) {
    return (kTRows + tc_x_rows(fmt, N)) * 128 * segs;
}

// x [M, k] bf16 -> the two E4M3 planes the FP8 MMAs read, [hi: N rows | lo: N rows] x k,
// of x scaled by 2^e_m (the largest |x| of row m lands in [128, 256)); rows m >= M are
// zero. One CTA per plane row.
__global__ void __launch_bounds__(256) tc_xq_kernel(const uint16_t* __restrict__ x, int M, int k,
                                                    int N, uint8_t* __restrict__ xq,
                                                    int32_t* __restrict__ xexp) {
    __shared__ float red[8];
    const int m = blockIdx.x, tid = threadIdx.x;
    uint8_t* hi = xq + (int64_t)m * k;
    uint8_t* lo = xq + (int64_t)(N + m) * k;
    if (m >= M) {
        for (int j = tid; j < k; j += 256) hi[j] = lo[j] = 0;
        return;
    }
    const uint16_t* row = x + (int64_t)m * k;
    float a = 0.f;
    for (int j = tid; j < k; j += 256) a = fmaxf(a, fabsf(bf16_to_f32(row[j])));
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((tid & 31) == 0) red[tid >> 5] = a;
    __syncthreads();
    a = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) a = fmaxf(a, red[w]);
    int ex = 0;
    if (a > 0.f) frexpf(a, &ex);  // a in [2^(ex-1), 2^ex)
    const int e = (a > 0.f) ? 8 - ex : 0;
    if (tid == 0) xexp[m] = e;
    const float f1 = ldexpf(1.f, e / 2), f2 = ldexpf(1.f, e - e / 2);
    for (int j = 2 * tid; j < k; j += 512) {  // k is even
        const float v0 = (bf16_to_f32(row[j]) * f1) * f2;
        const float v1 = (bf16_to_f32(row[j + 1]) * f1) * f2;
        const uint16_t h = f32x2_to_e4m3x2(v0, v1);
        const float r0 = v0 - e4m3_to_f32(h & 0xFFu), r1 = v1 - e4m3_to_f32(h >> 8);
        const uint16_t l = f32x2_to_e4m3x2(r0, r1);
        *reinterpret_cast<uint16_t*>(hi + j) = h;
        *reinterpret_cast<uint16_t*>(lo + j) = l;
    }
}

template <int FMT, int N>
__global__ void __launch_bounds__(kTThreads, 1)
    sweep_tc_kernel(const __grid_constant__ SweepParams p, const __grid_constant__ CUtensorMap map_codes,
                    const __grid_constant__ CUtensorMap map_x) {
    static_assert(FMT == 0 || FMT == 1, "BF16 and FP8 tables");
    static_assert(N == 16 || N == 32, "16 or 32 input columns");
    // x rows per stage segment, and accumulator columns per tile: for FP8 the hi and lo
    // rows of x are one B operand of 2N rows, so D holds x_hi and x_lo dot products side
    // by side (columns m and N + m), added in the epilogue
    constexpr int XR = FMT == 1 ? 2 * N : N;
    constexpr int DC = XR;
    constexpr uint32_t kTmemCols = 2 * DC < 32 ? 32 : 2 * DC;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* tfull = empty + kMaxStages;  // [2]: the tile's MMAs done + its tile index posted
    uint64_t* tempty = tfull + 2;          // [2]: the epilogue has read the accumulator
    uint64_t* done = tempty + 2;           // every MMA done (before tensor memory is freed)
    // bytes [0, 232): barriers; [232, 360): misc; [512, 768): sfac; [768, 2816): fold
    int* misc = reinterpret_cast<int*>(done + 1);
    volatile int* abort_flag = misc;            // [0]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    volatile int* slot_tile = misc + 2;         // [2 .. 2 + kMaxStages)
    volatile int* acc_tile = misc + 2 + kMaxStages;  // [2]
    float* sfac = reinterpret_cast<float*>(smem + 512);    // [2][32]: 2^-e_m as two factors
    float4* fold = reinterpret_cast<float4*>(smem + 768);  // [4 warps][32 inputs]
    const uint32_t head_end = smem_u32(fold + kTEpiWarps * 32);
    uint8_t* ring = smem + (((head_end + 1023u) & ~1023u) - smem_u32(smem));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.stages;
    const int stage_bytes = p.stage_bytes;
    const int segs = p.segs;
    const int NC = p.stages_per_tile;
    const int M = p.M;
    const int64_t T = p.num_tiles;
    const int a_bytes = kTRows * 128 * segs;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 2);
            mbar_init(&tempty[b], kTEpiWarps);
        }
        mbar_init(done, 1);
        misc[0] = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- producer: the tiles' stages, each tagged with its tile
        int slot = 0;
        uint32_t phase = 0;
        int64_t issued = 0;
        const uint32_t tx = (uint32_t)stage_bytes;
        bool stop = false;
        pdl_wait();  // x (and for FP8 its E4M3 planes) come from the previous grid
        int64_t tile = blockIdx.x;
        int64_t pending = 0;
        if (lane == 0) pending = (int64_t)gridDim.x + atomicAdd(p.ticket + 1, 1u);
        while (tile < T && !stop) {
            for (int ch = 0; ch < NC; ++ch) {
                if (!mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    uint8_t* dst = ring + (size_t)slot * stage_bytes;
                    slot_tile[slot] = (int)tile;
                    mbar_arrive_expect_tx(&full[slot], tx);
                    tma_load_3d(dst, &map_codes, 0, (int)(tile * kTRows), ch * segs, &full[slot]);
                    tma_load_3d(dst + a_bytes, &map_x, 0, 0, ch * segs, &full[slot]);
                }
                __syncwarp();
                ++issued;
                if (++slot == S) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
            tile = __shfl_sync(0xffffffffu, pending, 0);
            if (lane == 0 && tile < T) pending = (int64_t)gridDim.x + atomicAdd(p.ticket + 1, 1u);
        }
        // no copy left in flight; then the end marker (a stage tagged -1, no copy)
        for (int64_t j = issued > S ? issued - S : 0; j < issued; ++j)
            if (!mbar_wait_bounded(&full[j % S], (uint32_t)((j / S) & 1), nullptr)) break;
        if (!stop && mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag) && lane == 0) {
            slot_tile[slot] = -1;
            mbar_arrive(&full[slot]);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (lane 0)
        constexpr uint32_t idesc = FMT == 0 ? idesc_bf16(kTRows, DC) : idesc_e4m3(kTRows, DC);
        int slot = 0;
        uint32_t phase = 0;
        int local = 0;
        while (true) {
            if (!mbar_wait_bounded(&full[slot], phase, abort_flag)) break;
            const int tile = slot_tile[slot];
            const int buf = local & 1;
            const uint32_t tph = (uint32_t)((local >> 1) & 1);
            if (!mbar_wait_bounded(&tempty[buf], tph ^ 1u, abort_flag)) break;
            if (lane == 0) {  // the tile index for the epilogue (its own arrival, release)
                acc_tile[buf] = tile;
                mbar_arrive(&tfull[buf]);
                if (tile < 0) mbar_arrive(&tfull[buf]);  // no MMAs behind the end marker
            }
            __syncwarp();
            if (tile < 0) break;
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * DC);
            bool ok = true;
            for (int ch = 0; ch < NC; ++ch) {
                if (ch > 0 && !mbar_wait_bounded(&full[slot], phase, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(ring + (size_t)slot * stage_bytes);
                    const uint32_t x0 = a0 + (uint32_t)a_bytes;
                    for (int sg = 0; sg < segs; ++sg) {
                        const uint32_t as = a0 + (uint32_t)sg * (kTRows * 128);
                        const uint32_t xs = x0 + (uint32_t)sg * (XR * 128);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t acc = (ch > 0 || sg > 0 || k > 0) ? 1u : 0u;
                            if (FMT == 0)
                                umma_bf16(d_tmem, sdesc_k128(as + k * 32), sdesc_k128(xs + k * 32), idesc, acc);
                            else
                                umma_e4m3(d_tmem, sdesc_k128(as + k * 32), sdesc_k128(xs + k * 32), idesc, acc);
                        }
                    }
                    umma_commit(&empty[slot]);  // frees the stage once these MMAs have read it
                }
                __syncwarp();
                if (++slot == S) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
            if (lane == 0) umma_commit(&tfull[buf]);  // the accumulator, once complete
            __syncwarp();
            ++local;
            if (!ok) break;
        }
        if (lane == 0) umma_commit(done);
        __syncwarp();
        mbar_wait_bounded(done, 0u, nullptr);
    } else {
        // ---------------- epilogue: warp w reads tensor memory lanes 32 (w % 4) + [0, 32)
        const int q = warp & 3;
        const int ew = warp - 2;  // 0..3
        const bool lp = p.out_logprob != nullptr || p.out_partial != nullptr;
        pdl_wait();
        if (ew == 0) {
            const int e = (FMT == 1 && lane < M) ? -__ldg(p.xexp + lane) : 0;
            sfac[lane] = ldexpf(1.f, e / 2);
            sfac[32 + lane] = ldexpf(1.f, e - e / 2);
        }
        named_sync(1, kTEpiWarps * 32);
        float best_v[N], se[N];
        int32_t best_i[N];
#pragma unroll
        for (int m = 0; m < N; ++m) {
            best_v[m] = -INFINITY;
            best_i[m] = INT_MAX;
            se[m] = 0.f;
        }
        int local = 0;
        while (true) {
            const int buf = local & 1;
            const uint32_t tph = (uint32_t)((local >> 1) & 1);
            if (!mbar_wait_bounded(&tfull[buf], tph, abort_flag)) break;
            const int tile = acc_tile[buf];
            if (tile < 0) break;
            tc_fence_after();
            uint32_t v[N];
            const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * DC);
            if constexpr (N == 32)
                tmem_ld32(ta, v);
            else
                tmem_ld16(ta, v);
            if constexpr (FMT == 1) {  // + the x_lo dot products
                uint32_t w[N];
                if constexpr (N == 32)
                    tmem_ld32(ta + N, w);
                else
                    tmem_ld16(ta + N, w);
                tmem_ld_wait();
#pragma unroll
                for (int m = 0; m < N; ++m) v[m] = __float_as_uint(__uint_as_float(v[m]) + __uint_as_float(w[m]));
            }
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);  // the accumulator is free again
            const int64_t row = (int64_t)tile * kTRows + q * 32 + lane;
            const bool rvalid = row < p.n;
            const float rs = (FMT == 1 && rvalid) ? __ldg(p.row_scale + row) : 1.f;
#pragma unroll
            for (int m = 0; m < N; ++m) {
                if (m >= M) break;
                float l = __uint_as_float(v[m]);
                if (FMT == 1) l = ((l * sfac[m]) * sfac[32 + m]) * rs;
                const bool ok = rvalid && mask_allows(p, m, row);
                if (rvalid && p.out_logits)
                    p.out_logits[(int64_t)m * p.n + row] = ok ? f32_to_bf16(l) : (uint16_t)0xFF80u;
                if (lp && ok && l > -INFINITY) {
                    float bv = best_v[m];
                    lse_merge(bv, se[m], l, 1.f);
                }
                // each thread's rows arrive in increasing order: the lowest wins a tie
                if (ok && (l > best_v[m] || (l == best_v[m] && best_i[m] == INT_MAX))) {
                    best_v[m] = l;
                    best_i[m] = (int32_t)row;
                }
            }
            ++local;
        }
        // per input: fold the 32 lanes, then the four warps in order; publish; ticket
#pragma unroll
        for (int m = 0; m < N; ++m) {
            if (m >= M) break;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, best_v[m], o);
                const int32_t oi = __shfl_xor_sync(0xffffffffu, best_i[m], o);
                const float os = __shfl_xor_sync(0xffffffffu, se[m], o);
                if (lp) {
                    float bv = best_v[m];
                    lse_merge(bv, se[m], ov, os);
                }
                if (ov > best_v[m] || (ov == best_v[m] && oi < best_i[m])) {
                    best_v[m] = ov;
                    best_i[m] = oi;
                }
            }
            if (lane == 0) fold[ew * 32 + m] = make_float4(best_v[m], __int_as_float(best_i[m]), se[m], 0.f);
        }
        named_sync(1, kTEpiWarps * 32);
        if (ew == 0) {
            if (lane < M) {
                float bv = -INFINITY, bs = 0.f;
                int32_t bi = INT_MAX;
                for (int w = 0; w < kTEpiWarps; ++w) {
                    const float4 f = fold[w * 32 + lane];
                    const int32_t fi = __float_as_int(f.y);
                    if (lp) {
                        float t = bv;
                        lse_merge(t, bs, f.x, f.z);
                    }
                    if (f.x > bv || (f.x == bv && fi < bi)) {
                        bv = f.x;
                        bi = fi;
                    }
                }
                reinterpret_cast<Partial*>(p.partials)[(int64_t)blockIdx.x * kPartSlots + lane] =
                    Partial{bv, bi, bs, 0.f};
            }
            __syncwarp();
            fence_acq_rel_gpu();  // every publishing lane's store before lane 0's ticket
            __syncwarp();
            if (*abort_flag && lane == 0) raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
            ticket_and_fold(p, lane, lp);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------- NVFP4 block-scaled sweep
// NVFP4 tables run the contraction on tcgen05 block-scaled FP4 MMAs (kind::mxf4nvf4, one
// E4M3 scale per 16 elements on each operand, K = 64 per instruction): the table's E2M1
// codes and E4M3 block scales are the A operand and its scale factors as stored, so
// nothing is decoded. The B operand must be FP4 too, so each input is written as six
// E2M1 terms (q4_xterms_kernel): per 16-element block a power-of-two scale s and balanced
// base-8 digits d_t in [-4, 4], x 2^e = sum_t d_t s 8^-t + r; term t is B row t MP + m with
// codes d_t / 2 and block scale 2 s, and the epilogue weighs accumulator column t MP + m
// by 8^-t in fp32. Every element whose binary exponent is within 9 of its block's
// largest |x| is represented exactly (a bf16 value has 8 significant bits and the last
// digit's unit is s 8^-5 < 2^-16 of the block's largest), the rest within s 8^-5 / 2, i.e.
// 2^-17 of the block's largest |x|; s is at least 2^-10 (x 2^e units, the input's largest
// |x 2^e| in [128, 256)), so blocks below 2^-8 there are represented within 2^-26.
// Products and sums are fp32 in the tensor core.
// Roles: warp 0 streams stages (128 table rows x segs 128-byte code segments and their
// block scales, the x terms' codes and block scales for the same K range); warps 6-9
// write the stage's scale factors into the ring slot's tensor-memory columns with
// tcgen05.st, in the layout the MMA reads (in every lane quarter, lane l and columns
// 4 j + c hold K block j's scales of row l + 32 c, four per 32-bit column); warp 1 issues
// the MMAs from one thread; warps 2-5 sum the six term columns per input, scale, mask
// and keep per input a running (max, lowest row, sum of exp). Tiles of 128 rows are
// handed out at run time; the last CTA folds the CTA partials.
constexpr int kQ4Terms = 6;
constexpr int kQ4Threads = 320;  // warp 0 TMA, 1 MMA, 2-5 epilogue, 6-9 scale factors
constexpr int kQ4Epi = 4;
constexpr int kQ4Head = 3072;    // barriers, misc, factors, fold; then the ring
constexpr int kQ4MaxM = 16;      // N = 6 MP <= 128: one group of scale rows

__host__ __device__ constexpr int q4_mp(int M) { return M <= 4 ? 4 : M <= 8 ? 8 : 16; }
__host__ __device__ constexpr int q4_n(int MP) { return (kQ4Terms * MP + 15) / 16 * 16; }
inline size_t q4_code_bytes(int N, int64_t k) { return ((size_t)N * (size_t)(k / 2) + 1023) & ~(size_t)1023; }
inline size_t q4_scale_bytes(int N, int64_t k) { return ((size_t)N * (size_t)(k / 16) + 1023) & ~(size_t)1023; }
__host__ __device__ inline int q4_stage_bytes(int N, int segs) {
    const int b = segs * (16384 + N * 128 + N * 16 + 2048);
    return (b + 1023) & ~1023;
}
// tensor-memory columns: the two accumulators, then per ring slot 16 segs for the table's
// scale factors and 16 segs for x's
__host__ __device__ inline int q4_max_slots(int N, int segs) { return (512 - 2 * N) / (32 * segs); }

// The E4M3 code of 2^e, e in [-9, 8] (normal from 2^-6, subnormal below).
__device__ __forceinline__ uint32_t e4m3_pow2(int e) {
    return e >= -6 ? (uint32_t)(e + 7) << 3 : 1u << (e + 9);
}

// x [M, k] bf16 -> the block-scaled sweep's B operand. CTA m < M: input m scaled by 2^e_m
// (its largest |x| lands in [128, 256)), then per 16-element block b: s = 2^ceil(log2(a /
// 4)) for the block's largest |x 2^e| = a (s >= 2^-10), digits d_t = rint(r_t / (s 8^-t))
// with r_0 = x 2^e, r_{t+1} = r_t - d_t s 8^-t (all exact in fp32; |d_t| <= 4 since
// |r_t| <= 4 s 8^-t); row t MP + m gets the E2M1 codes of d_t / 2 (magnitude |d_t|, sign
// bit 3) and the block scale E4M3(2 s). CTAs M .. MP - 1 zero their rows and CTA MP the
// rows past 6 MP. codes [N][k / 2], scales [N][k / 16].
__global__ void __launch_bounds__(256) q4_xterms_kernel(const uint16_t* __restrict__ x, int M, int k,
                                                        int MP, int N, uint8_t* __restrict__ codes,
                                                        uint8_t* __restrict__ scales,
                                                        int32_t* __restrict__ xexp) {
    __shared__ float red[8];
    const int m = blockIdx.x, tid = threadIdx.x;
    const int64_t rb = k / 2, sp = k / 16;
    if (m >= M) {  // zero rows: inputs past M (their six rows), or the rows past 6 MP
        const int n0 = m < MP ? m : kQ4Terms * MP;
        const int step = m < MP ? MP : 1;
        const int n1 = m < MP ? kQ4Terms * MP : N;
        for (int n = n0; n < n1; n += step) {
            for (int64_t j = tid; j < rb; j += 256) codes[(int64_t)n * rb + j] = 0;
            for (int64_t j = tid; j < sp; j += 256) scales[(int64_t)n * sp + j] = 0;
        }
        return;
    }
    const uint16_t* row = x + (int64_t)m * k;
    float a = 0.f;
    for (int j = tid; j < k; j += 256) a = fmaxf(a, fabsf(bf16_to_f32(row[j])));
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((tid & 31) == 0) red[tid >> 5] = a;
    __syncthreads();
    a = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) a = fmaxf(a, red[w]);
    int ex = 0;
    if (a > 0.f) frexpf(a, &ex);  // a in [2^(ex-1), 2^ex)
    const int e = (a > 0.f) ? 8 - ex : 0;
    if (tid == 0) xexp[m] = e;
    const float f1 = ldexpf(1.f, e / 2), f2 = ldexpf(1.f, e - e / 2);
    for (int b = tid; b < k / 16; b += 256) {
        float v[16];
        float bm = 0.f;
        const uint4* src = reinterpret_cast<const uint4*>(row + 16 * b);
        const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = (bf16_lo(w[i]) * f1) * f2;
            v[2 * i + 1] = (bf16_hi(w[i]) * f1) * f2;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) bm = fmaxf(bm, fabsf(v[i]));
        int se = -10;  // s = 2^se
        if (bm > 0.f) {
            int be = 0;
            const float fr = frexpf(bm, &be);  // bm = fr 2^be, fr in [1/2, 1)
            se = max(fr == 0.5f ? be - 3 : be - 2, -10);
        }
        const uint8_t sc = (uint8_t)e4m3_pow2(se + 1);
#pragma unroll
        for (int t = 0; t < kQ4Terms; ++t) {
            const float u = ldexpf(1.f, se - 3 * t), iu = ldexpf(1.f, 3 * t - se);
            uint32_t lo = 0, hi = 0;  // 16 codes, element i in nibble i
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float d = rintf(v[i] * iu);
                d = fminf(fmaxf(d, -4.f), 4.f);
                v[i] = fmaf(-d, u, v[i]);
                const uint32_t c = (d < 0.f ? 8u : 0u) | (uint32_t)fabsf(d);
                if (i < 8) lo |= c << (4 * i);
                else hi |= c << (4 * (i - 8));
            }
            const int n = t * MP + m;
            *reinterpret_cast<uint2*>(codes + (int64_t)n * rb + 8 * b) = make_uint2(lo, hi);
            scales[(int64_t)n * sp + b] = sc;
        }
    }
}

// D[tmem] (+)= (A sfa) . (B sfb)^T, E2M1 operands from shared memory, E4M3 scales per 16
// elements from tensor memory, K = 64. One thread.
__device__ __forceinline__ void umma_q4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Warp-wide: this warp's 32 TMEM lanes, 4 consecutive 32-bit columns from `taddr` (a
// multiple of 4) written.
__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b),
                 "r"(c), "r"(d)
                 : "memory");
}

template <int MP>
__global__ void __launch_bounds__(kQ4Threads, 1)
    sweep_q4_kernel(const __grid_constant__ SweepParams p, const __grid_constant__ CUtensorMap map_codes,
                    const __grid_constant__ CUtensorMap map_scales, const __grid_constant__ CUtensorMap map_x,
                    const __grid_constant__ CUtensorMap map_xs) {
    constexpr int N = q4_n(MP);
    static_assert(N <= 128, "one group of scale rows");
    constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (8u << 24);
    constexpr uint32_t kSfCol = 2 * N;  // accumulators: columns [0, 2N)
    constexpr uint32_t kTmemCols = 512;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* sfull = empty + kMaxStages;  // the slot's scale factors are in tensor memory
    uint64_t* tfull = sfull + kMaxStages;  // [2]
    uint64_t* tempty = tfull + 2;          // [2]
    uint64_t* done = tempty + 2;
    int* misc = reinterpret_cast<int*>(done + 1);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    volatile int* slot_tile = misc + 2;              // [kMaxStages]
    volatile int* acc_tile = misc + 2 + kMaxStages;  // [2]
    float* sfac = reinterpret_cast<float*>(smem + 512);    // [2][32]: 2^-e_m as two factors
    float4* fold = reinterpret_cast<float4*>(smem + 768);  // [4 warps][32 inputs]
    uint8_t* ring = smem + kQ4Head;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.stages;
    const int stage_bytes = p.stage_bytes;
    const int segs = p.segs;
    const int NC = p.stages_per_tile;
    const int M = p.M;
    const int64_t T = p.num_tiles;
    // stage layout: table codes | x term codes | x term scales [N][16 segs] | table scales
    // [128][16 segs]
    const int a_bytes = 16384 * segs;
    const int x_off = a_bytes, x_bytes = N * 128 * segs;
    const int xs_off = x_off + x_bytes, xs_bytes = N * 16 * segs;
    const int as_off = xs_off + xs_bytes, as_bytes = 2048 * segs;
    const uint32_t tx = (uint32_t)(a_bytes + x_bytes + xs_bytes + as_bytes);
    const uint32_t slot_cols = 32u * (uint32_t)segs;  // per ring slot: table's, then x's

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfull[s], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 2);
            mbar_init(&tempty[b], kQ4Epi);
        }
        mbar_init(done, 1);
        misc[0] = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- producer: the tiles' stages, each tagged with its tile
        int slot = 0;
        uint32_t phase = 0;
        int64_t issued = 0;
        bool stop = false;
        pdl_wait();  // the x terms come from the previous grid
        int64_t tile = blockIdx.x;
        int64_t pending = 0;
        if (lane == 0) pending = (int64_t)gridDim.x + atomicAdd(p.ticket + 1, 1u);
        while (tile < T && !stop) {
            for (int ch = 0; ch < NC; ++ch) {
                if (!mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    uint8_t* dst = ring + (size_t)slot * stage_bytes;
                    slot_tile[slot] = (int)tile;
                    mbar_arrive_expect_tx(&full[slot], tx);
                    tma_load_3d(dst, &map_codes, 0, (int)(tile * 128), ch * segs, &full[slot]);
                    tma_load_3d(dst + x_off, &map_x, 0, 0, ch * segs, &full[slot]);
                    tma_load_2d(dst + xs_off, &map_xs, ch * 8 * segs, 0, &full[slot]);
                    tma_load_2d(dst + as_off, &map_scales, ch * 8 * segs, (int)(tile * 128), &full[slot]);
                }
                __syncwarp();
                ++issued;
                if (++slot == S) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
            tile = __shfl_sync(0xffffffffu, pending, 0);
            if (lane == 0 && tile < T) pending = (int64_t)gridDim.x + atomicAdd(p.ticket + 1, 1u);
        }
        for (int64_t j = issued > S ? issued - S : 0; j < issued; ++j)
            if (!mbar_wait_bounded(&full[j % S], (uint32_t)((j / S) & 1), nullptr)) break;
        if (!stop && mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag) && lane == 0) {
            slot_tile[slot] = -1;
            mbar_arrive(&full[slot]);
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ---------------- scale factors: warp 6 + q writes lane quarter q; its lane l holds,
        // for K block j, the scale words (four 16-element blocks each) of table rows and x
        // term rows l, l + 32, l + 64, l + 96 at columns 4 j .. 4 j + 3 of the slot's regions
        const int q = warp - 6;
        int slot = 0;
        uint32_t phase = 0;
        const uint32_t lq = tmem_base + ((uint32_t)(q * 32) << 16);
        while (true) {
            if (!mbar_wait_bounded(&full[slot], phase, abort_flag)) break;
            if (slot_tile[slot] < 0) break;
            const uint8_t* st = ring + (size_t)slot * stage_bytes;
            const uint32_t ca = lq + kSfCol + (uint32_t)slot * slot_cols;  // table's
            const uint32_t cx = ca + 16u * (uint32_t)segs;                  // x's
            for (int sg = 0; sg < segs; ++sg) {
                uint4 ra[4], rx[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int r = lane + 32 * c;
                    ra[c] = lds128(st + as_off + r * 16 * segs + 16 * sg);
                    rx[c] = r < N ? lds128(st + xs_off + r * 16 * segs + 16 * sg) : make_uint4(0, 0, 0, 0);
                }
                const uint32_t c0 = 16u * (uint32_t)sg;
                tmem_st4(ca + c0 + 0, ra[0].x, ra[1].x, ra[2].x, ra[3].x);
                tmem_st4(ca + c0 + 4, ra[0].y, ra[1].y, ra[2].y, ra[3].y);
                tmem_st4(ca + c0 + 8, ra[0].z, ra[1].z, ra[2].z, ra[3].z);
                tmem_st4(ca + c0 + 12, ra[0].w, ra[1].w, ra[2].w, ra[3].w);
                tmem_st4(cx + c0 + 0, rx[0].x, rx[1].x, rx[2].x, rx[3].x);
                tmem_st4(cx + c0 + 4, rx[0].y, rx[1].y, rx[2].y, rx[3].y);
                tmem_st4(cx + c0 + 8, rx[0].z, rx[1].z, rx[2].z, rx[3].z);
                tmem_st4(cx + c0 + 12, rx[0].w, rx[1].w, rx[2].w, rx[3].w);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfull[slot]);
            if (++slot == S) {
                slot = 0;
                phase ^= 1u;
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (lane 0)
        int slot = 0;
        uint32_t phase = 0;
        int local = 0;
        while (true) {
            if (!mbar_wait_bounded(&full[slot], phase, abort_flag)) break;
            const int tile = slot_tile[slot];
            const int buf = local & 1;
            const uint32_t tph = (uint32_t)((local >> 1) & 1);
            if (!mbar_wait_bounded(&tempty[buf], tph ^ 1u, abort_flag)) break;
            if (lane == 0) {  // the tile index for the epilogue (its own arrival, release)
                acc_tile[buf] = tile;
                mbar_arrive(&tfull[buf]);
                if (tile < 0) mbar_arrive(&tfull[buf]);  // no MMAs behind the end marker
            }
            __syncwarp();
            if (tile < 0) break;
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * N);
            bool ok = true;
            for (int ch = 0; ch < NC; ++ch) {
                if ((ch > 0 && !mbar_wait_bounded(&full[slot], phase, abort_flag)) ||
                    !mbar_wait_bounded(&sfull[slot], phase, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t st = smem_u32(ring + (size_t)slot * stage_bytes);
                    const uint32_t ca = tmem_base + kSfCol + (uint32_t)slot * slot_cols;
                    const uint32_t cx = ca + 16u * (uint32_t)segs;
                    const int kbs = 4 * segs;
                    for (int kb = 0; kb < kbs; ++kb) {
                        const uint32_t as = st + (uint32_t)((kb >> 2) * 16384 + (kb & 3) * 32);
                        const uint32_t xs = st + (uint32_t)(x_off + (kb >> 2) * (N * 128) + (kb & 3) * 32);
                        umma_q4(d_tmem, sdesc_k128(as), sdesc_k128(xs), kIdesc, ca + 4u * (uint32_t)kb,
                                cx + 4u * (uint32_t)kb, (ch > 0 || kb > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[slot]);  // frees the stage (and its scale columns) once read
                }
                __syncwarp();
                if (++slot == S) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
            if (lane == 0) umma_commit(&tfull[buf]);  // the accumulator, once complete
            __syncwarp();
            ++local;
            if (!ok) break;
        }
        if (lane == 0) umma_commit(done);
        __syncwarp();
        mbar_wait_bounded(done, 0u, nullptr);
    } else {
        // ---------------- epilogue: warp w reads tensor memory lanes 32 (w % 4) + [0, 32)
        const int q = warp & 3;
        const int ew = warp - 2;  // 0..3
        const bool lp = p.out_logprob != nullptr || p.out_partial != nullptr;
        pdl_wait();
        if (ew == 0) {
            const int e = lane < M ? -__ldg(p.xexp + lane) : 0;
            sfac[lane] = ldexpf(1.f, e / 2);
            sfac[32 + lane] = ldexpf(1.f, e - e / 2);
        }
        const float gsc = __ldg(p.global_scale);
        named_sync(1, kQ4Epi * 32);
        float best_v[MP], se[MP];
        int32_t best_i[MP];
#pragma unroll
        for (int m = 0; m < MP; ++m) {
            best_v[m] = -INFINITY;
            best_i[m] = INT_MAX;
            se[m] = 0.f;
        }
        int local = 0;
        while (true) {
            const int buf = local & 1;
            const uint32_t tph = (uint32_t)((local >> 1) & 1);
            if (!mbar_wait_bounded(&tfull[buf], tph, abort_flag)) break;
            const int tile = acc_tile[buf];
            if (tile < 0) break;
            tc_fence_after();
            // per input, the six term columns t MP + m weighed by 8^-t, in order of t
            float l[MP];
#pragma unroll
            for (int m = 0; m < MP; ++m) l[m] = 0.f;
            const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * N);
#pragma unroll
            for (int c0 = 0; c0 < N; c0 += 32) {
                uint32_t v[32];
                if (c0 + 32 <= N) {
                    tmem_ld32(ta + c0, v);
                } else {
                    uint32_t h[16];
                    tmem_ld16(ta + c0, h);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = h[i];
                }
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int n = c0 + i;
                    if (n < N && n < kQ4Terms * MP)
                        l[n % MP] = fmaf(__uint_as_float(v[i]), 1.0f / (float)(1 << (3 * (n / MP))), l[n % MP]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);  // the accumulator is free again
            const int64_t row = (int64_t)tile * 128 + q * 32 + lane;
            const bool rvalid = row < p.n;
#pragma unroll
            for (int m = 0; m < MP; ++m) {
                if (m >= M) break;
                const float lv = ((l[m] * sfac[m]) * sfac[32 + m]) * gsc;
                const bool ok = rvalid && mask_allows(p, m, row);
                if (rvalid && p.out_logits)
                    p.out_logits[(int64_t)m * p.n + row] = ok ? f32_to_bf16(lv) : (uint16_t)0xFF80u;
                if (lp && ok && lv > -INFINITY) {
                    float bv = best_v[m];
                    lse_merge(bv, se[m], lv, 1.f);
                }
                // each thread's rows arrive in increasing order: the lowest wins a tie
                if (ok && (lv > best_v[m] || (lv == best_v[m] && best_i[m] == INT_MAX))) {
                    best_v[m] = lv;
                    best_i[m] = (int32_t)row;
                }
            }
            ++local;
        }
        // per input: fold the 32 lanes, then the four warps in order; publish; ticket
#pragma unroll
        for (int m = 0; m < MP; ++m) {
            if (m >= M) break;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, best_v[m], o);
                const int32_t oi = __shfl_xor_sync(0xffffffffu, best_i[m], o);
                const float os = __shfl_xor_sync(0xffffffffu, se[m], o);
                if (lp) {
                    float bv = best_v[m];
                    lse_merge(bv, se[m], ov, os);
                }
                if (ov > best_v[m] || (ov == best_v[m] && oi < best_i[m])) {
                    best_v[m] = ov;
                    best_i[m] = oi;
                }
            }
            if (lane == 0) fold[ew * 32 + m] = make_float4(best_v[m], __int_as_float(best_i[m]), se[m], 0.f);
        }
        named_sync(1, kQ4Epi * 32);
        if (ew == 0) {
            if (lane < M) {
                float bv = -INFINITY, bs = 0.f;
                int32_t bi = INT_MAX;
                for (int w = 0; w < kQ4Epi; ++w) {
                    const float4 f = fold[w * 32 + lane];
                    const int32_t fi = __float_as_int(f.y);
                    if (lp) {
                        float t = bv;
                        lse_merge(t, bs, f.x, f.z);
                    }
                    if (f.x > bv || (f.x == bv && fi < bi)) {
                        bv = f.x;
                        bi = fi;
                    }
                }
                reinterpret_cast<Partial*>(p.partials)[(int64_t)blockIdx.x * kPartSlots + lane] =
                    Partial{bv, bi, bs, 0.f};
            }
            __syncwarp();
            fence_acq_rel_gpu();  // every publishing lane's store before lane 0's ticket
            __syncwarp();
            if (*abort_flag && lane == 0) raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
            ticket_and_fold(p, lane, lp);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// The same contraction for 17-32 inputs (N = 192 term rows) on CTA pairs (2-CTA clusters,
// cta_group::2): a tile is 256 table rows and one MMA of M = 256 covers both CTAs' 128 rows.
// The B operand (x's terms) is split between the pair, so each CTA stages half of x's term
// rows next to its table rows -- 66 KB stages, three deep, where one CTA alone would have
// room for two. (A paired MMA keeps each SM's tensor pipe as long as a single-CTA one of
// its 128 rows, so pairs only pay where the x stages are this large.) Roles per CTA: warp 0
// streams stages (its 128 rows x 2 code segments and its half of x's term codes, both
// completing on rank 0's barrier; on its own barrier its rows' block scales and all of x's
// term scales); warps 6-9 write the stage's scale factors into its tensor memory (table
// rows at columns 4 j + c, x term rows 128 .. at 4 j + 4 + c, K blocks 8 columns apart)
// and tell rank 0; rank 0's warp 1 issues the MMAs once both CTAs' scale warps are done;
// warps 2-5 of each CTA drain its 128 rows. Rank 0 claims the tiles at run time and
// announces each to both CTAs through a small FIFO in each one's shared memory.
constexpr int kQ4Fifo = 8;  // tiles announced ahead
__host__ __device__ inline int q4p_stage_bytes(int segs) {  // per CTA, N = 192
    return ((segs * (16384 + 96 * 128 + 192 * 16 + 2048)) + 1023) & ~1023;
}
__host__ __device__ inline int q4p_max_slots(int segs) { return (512 - 192) / (16 * segs * 3); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kQ4Threads, 1)
    sweep_q4p_kernel(const __grid_constant__ SweepParams p, const __grid_constant__ CUtensorMap map_codes,
                    const __grid_constant__ CUtensorMap map_scales, const __grid_constant__ CUtensorMap map_x,
                    const __grid_constant__ CUtensorMap map_xs) {
    constexpr int MP = 32;
    constexpr int N = q4_n(MP);          // 192
    constexpr int NH = N / 2;            // x term rows this CTA stages
    constexpr int G = 2;                 // groups of 128 B rows (scale-factor column blocks)
    constexpr int NBUF = 1;              // one accumulator (2 N columns would leave no room)
    constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (16u << 24);  // M 256
    constexpr uint32_t kSfCol = NBUF * N;  // accumulators: columns [0, NBUF N)
    constexpr uint32_t kTmemCols = 512;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);  // rank 0's: both CTAs' codes
    uint64_t* empty = full + kMaxStages;                 // the MMA commit, to both CTAs
    uint64_t* sraw = empty + kMaxStages;                 // this CTA's scale bytes landed
    uint64_t* sfull = sraw + kMaxStages;                 // rank 0's: both CTAs' scale factors written
    uint64_t* tfull = sfull + kMaxStages;                // [2] the MMA commit, to both CTAs
    uint64_t* tempty = tfull + 2;                        // [2] rank 0's: both CTAs' epilogues
    uint64_t* qfull = tempty + 2;                        // [kQ4Fifo]
    uint64_t* qempty = qfull + kQ4Fifo;                  // [kQ4Fifo] rank 0's
    uint64_t* done = qempty + kQ4Fifo;
    int* misc = reinterpret_cast<int*>(done + 1);
    volatile int* abort_flag = misc;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 1);
    volatile int* slot_tile = misc + 2;              // [kMaxStages]
    int* fifo = misc + 2 + kMaxStages;               // [kQ4Fifo]
    float* sfac = reinterpret_cast<float*>(smem + 768);     // [2][32]: 2^-e_m as two factors
    float4* fold = reinterpret_cast<float4*>(smem + 1024);  // [4 warps][32 inputs]
    uint8_t* ring = smem + kQ4Head;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
    const int S = p.stages;
    const int stage_bytes = p.stage_bytes;
    const int segs = p.segs;
    const int NC = p.stages_per_tile;
    const int M = p.M;
    const int64_t T = p.num_tiles;  // 256-row tiles
    // stage layout: table codes (this CTA's 128 rows) | x term codes (its N / 2 rows) |
    // x term scales [N][16 segs] | table scales [128][16 segs]
    const int a_bytes = 16384 * segs;
    const int x_off = a_bytes, x_bytes = NH * 128 * segs;
    const int xs_off = x_off + x_bytes, xs_bytes = N * 16 * segs;
    const int as_off = xs_off + xs_bytes, as_bytes = 2048 * segs;
    const uint32_t code_tx = (uint32_t)(2 * (a_bytes + x_bytes));  // both CTAs', on rank 0's barrier
    const uint32_t scale_tx = (uint32_t)(xs_bytes + as_bytes);
    const uint32_t sfa_cols = 16u * (uint32_t)segs;                  // per ring slot
    const uint32_t slot_cols = sfa_cols * (1u + (uint32_t)G);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sraw[s], 1);
            mbar_init(&sfull[s], 8);  // four scale warps of each CTA
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * kQ4Epi);
        }
        for (int q = 0; q < kQ4Fifo; ++q) {
            mbar_init(&qfull[q], 1);
            mbar_init(&qempty[q], 3);  // rank 0's epilogue, rank 1's producer and epilogue
        }
        mbar_init(done, 1);
        misc[0] = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised, the pair's tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_launch_dependents();

    if (warp == 0) {
        // ---------------- producer: rank 0 claims tiles and announces them; both CTAs stream
        int slot = 0;
        uint32_t phase = 0;
        int q = 0;
        uint32_t qph = 0;
        int64_t issued = 0;
        bool stop = false;
        pdl_wait();  // the x terms come from the previous grid
        int64_t tile = pair;
        int64_t pending = 0;
        if (leader && lane == 0) pending = (int64_t)npairs + atomicAdd(p.ticket + 1, 1u);
        while (!stop) {
            bool end;
            if (leader) {
                end = tile >= T;
                if (!mbar_wait_cluster_bounded(&qempty[q], qph ^ 1u, abort_flag)) break;
                if (lane == 0) {
                    const int v = end ? -1 : (int)tile;
                    fifo[q] = v;
                    st_cluster_u32(map_rank(&fifo[q], 1), (uint32_t)v);
                    mbar_arrive(&qfull[q]);
                    mbar_arrive_cluster(map_rank(&qfull[q], 1));
                }
                __syncwarp();
            } else {
                if (!mbar_wait_cluster_bounded(&qfull[q], qph, abort_flag)) break;
                const int v = fifo[q];
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(map_rank(&qempty[q], 0));
                end = v < 0;
                tile = v;
            }
            if (++q == kQ4Fifo) {
                q = 0;
                qph ^= 1u;
            }
            if (end) break;
            const int arow = (int)(tile * 256 + rank * 128);
            for (int ch = 0; ch < NC; ++ch) {
                if (!mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    uint8_t* dst = ring + (size_t)slot * stage_bytes;
                    slot_tile[slot] = (int)tile;
                    const uint32_t fb = map_rank(&full[slot], 0);
                    if (leader) mbar_arrive_expect_tx(&full[slot], code_tx);
                    tma_load_3d_pair(dst, &map_codes, 0, arow, ch * segs, fb);
                    tma_load_3d_pair(dst + x_off, &map_x, 0, (int)rank * NH, ch * segs, fb);
                    mbar_arrive_expect_tx(&sraw[slot], scale_tx);
                    tma_load_2d(dst + xs_off, &map_xs, ch * 8 * segs, 0, &sraw[slot]);
                    tma_load_2d(dst + as_off, &map_scales, ch * 8 * segs, arow, &sraw[slot]);
                }
                __syncwarp();
                ++issued;
                if (++slot == S) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
            if (leader) {
                tile = __shfl_sync(0xffffffffu, pending, 0);
                if (lane == 0 && tile < T) pending = (int64_t)npairs + atomicAdd(p.ticket + 1, 1u);
            }
        }
        // no copy left in flight: rank 0's full barriers count both CTAs' codes; rank 1's
        // stages are free once the MMAs that read them completed; each CTA's scale bytes
        for (int64_t j = issued > S ? issued - S : 0; j < issued; ++j) {
            const uint32_t par = (uint32_t)((j / S) & 1);
            if (!mbar_wait_bounded(leader ? &full[j % S] : &empty[j % S], par, nullptr)) break;
            if (!mbar_wait_bounded(&sraw[j % S], par, nullptr)) break;
        }
        // the end marker for this CTA's scale warps (and rank 0's MMA thread): a stage tagged
        // -1, no copy; if rank 0 stopped early, still tell every FIFO reader
        if (!stop && mbar_wait_bounded(&empty[slot], phase ^ 1u, abort_flag) && lane == 0) {
            slot_tile[slot] = -1;
            mbar_arrive(&sraw[slot]);
            if (leader) mbar_arrive(&full[slot]);
        }
        if (leader && stop && mbar_wait_cluster_bounded(&qempty[q], qph ^ 1u, nullptr) && lane == 0) {
            fifo[q] = -1;
            st_cluster_u32(map_rank(&fifo[q], 1), 0xFFFFFFFFu);
            mbar_arrive(&qfull[q]);
            mbar_arrive_cluster(map_rank(&qfull[q], 1));
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ---------------- scale factors: warp 6 + q writes lane quarter q of this CTA's tensor
        // memory -- its table rows' scale words and all x term rows' -- for each stage, then
        // tells rank 0's MMA thread
        const int qd = warp - 6;
        int slot = 0;
        uint32_t phase = 0;
        const uint32_t lq = tmem_base + ((uint32_t)(qd * 32) << 16);
                while (true) {
            if (!mbar_wait_bounded(&sraw[slot], phase, abort_flag)) break;
            if (slot_tile[slot] < 0) break;
            const uint8_t* st = ring + (size_t)slot * stage_bytes;
            const uint32_t ca = lq + kSfCol + (uint32_t)slot * slot_cols;  // table rows'
            const uint32_t cx = ca + sfa_cols;                              // x term rows'
            for (int sg = 0; sg < segs; ++sg) {
                uint4 ra[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) ra[c] = lds128(st + as_off + (lane + 32 * c) * 16 * segs + 16 * sg);
                const uint32_t c0 = 16u * (uint32_t)sg;
                tmem_st4(ca + c0 + 0, ra[0].x, ra[1].x, ra[2].x, ra[3].x);
                tmem_st4(ca + c0 + 4, ra[0].y, ra[1].y, ra[2].y, ra[3].y);
                tmem_st4(ca + c0 + 8, ra[0].z, ra[1].z, ra[2].z, ra[3].z);
                tmem_st4(ca + c0 + 12, ra[0].w, ra[1].w, ra[2].w, ra[3].w);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    uint4 rx[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int r = 128 * g + lane + 32 * c;
                        rx[c] = r < N ? lds128(st + xs_off + r * 16 * segs + 16 * sg) : make_uint4(0, 0, 0, 0);
                    }
                    // K block 4 sg + j at columns 4 G (4 sg + j) + 4 g
                    const uint32_t b0 = cx + 4u * (uint32_t)G * (4u * (uint32_t)sg) + 4u * (uint32_t)g;
                    tmem_st4(b0 + 0u * 4u * G, rx[0].x, rx[1].x, rx[2].x, rx[3].x);
                    tmem_st4(b0 + 1u * 4u * G, rx[0].y, rx[1].y, rx[2].y, rx[3].y);
                    tmem_st4(b0 + 2u * 4u * G, rx[0].z, rx[1].z, rx[2].z, rx[3].z);
                    tmem_st4(b0 + 3u * 4u * G, rx[0].w, rx[1].w, rx[2].w, rx[3].w);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(&sfull[slot]);
                else mbar_arrive_cluster(map_rank(&sfull[slot], 0));
            }
            if (++slot == S) {
                slot = 0;
                phase ^= 1u;
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: one thread of rank 0, for the pair
        int slot = 0;
        uint32_t phase = 0;
        int local = 0;
        bool stop = !leader;
        while (!stop) {
            if (!mbar_wait_bounded(&full[slot], phase, abort_flag)) break;
            const int tile = slot_tile[slot];
            if (tile < 0) break;
            const int buf = NBUF == 2 ? (local & 1) : 0;
            const uint32_t tph = (uint32_t)((NBUF == 2 ? (local >> 1) : local) & 1);
            // both CTAs' epilogues have read this accumulator's previous tile
            if (!mbar_wait_cluster_bounded(&tempty[buf], tph ^ 1u, abort_flag)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * N);
            for (int ch = 0; ch < NC; ++ch) {
                if ((ch > 0 && !mbar_wait_bounded(&full[slot], phase, abort_flag)) ||
                    !mbar_wait_cluster_bounded(&sfull[slot], phase, abort_flag)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t st = smem_u32(ring + (size_t)slot * stage_bytes);
                    const uint32_t ca = tmem_base + kSfCol + (uint32_t)slot * slot_cols;
                    const uint32_t cx = ca + sfa_cols;
                    const int kbs = 4 * segs;
                    for (int kb = 0; kb < kbs; ++kb) {
                        const uint32_t as = st + (uint32_t)((kb >> 2) * 16384 + (kb & 3) * 32);
                        const uint32_t xs = st + (uint32_t)(x_off + (kb >> 2) * (NH * 128) + (kb & 3) * 32);
                        umma_q4_pair(d_tmem, sdesc_k128(as), sdesc_k128(xs), kIdesc, ca + 4u * (uint32_t)kb,
                                     cx + 4u * (uint32_t)G * (uint32_t)kb, (ch > 0 || kb > 0) ? 1u : 0u);
                    }
                    umma_commit_pair(&empty[slot], 3);  // frees both CTAs' stage and scale columns
                }
                __syncwarp();
                if (++slot == S) {
                    slot = 0;
                    phase ^= 1u;
                }
            }
            if (lane == 0 && !stop) umma_commit_pair(&tfull[buf], 3);  // both CTAs' accumulators
            __syncwarp();
            ++local;
        }
        if (leader) {
            if (lane == 0) umma_commit_pair(done, 1);
            __syncwarp();
            mbar_wait_bounded(done, 0u, nullptr);
        }
    } else {
        // ---------------- epilogue: warp w reads tensor memory lanes 32 (w % 4) + [0, 32) of
        // this CTA (its 128 rows of the tile); the tiles come from the FIFO
        const int q = warp & 3;
        const int ew = warp - 2;  // 0..3
        const int et = threadIdx.x - 64;
        const bool lp = p.out_logprob != nullptr || p.out_partial != nullptr;
        pdl_wait();
        if (ew == 0) {
            const int e = lane < M ? -__ldg(p.xexp + lane) : 0;
            sfac[lane] = ldexpf(1.f, e / 2);
            sfac[32 + lane] = ldexpf(1.f, e - e / 2);
        }
        const float gsc = __ldg(p.global_scale);
        named_sync(1, kQ4Epi * 32);
        float best_v[MP], se[MP];
        int32_t best_i[MP];
#pragma unroll
        for (int m = 0; m < MP; ++m) {
            best_v[m] = -INFINITY;
            best_i[m] = INT_MAX;
            se[m] = 0.f;
        }
        int fq = 0;
        uint32_t fph = 0;
        int local = 0;
        while (true) {
            if (!mbar_wait_cluster_bounded(&qfull[fq], fph, abort_flag)) break;
            const int tile = fifo[fq];
            named_sync(1, kQ4Epi * 32);  // every epilogue thread has read the slot
            if (et == 0) {
                if (leader) mbar_arrive(&qempty[fq]);
                else mbar_arrive_cluster(map_rank(&qempty[fq], 0));
            }
            if (++fq == kQ4Fifo) {
                fq = 0;
                fph ^= 1u;
            }
            if (tile < 0) break;
            const int buf = NBUF == 2 ? (local & 1) : 0;
            const uint32_t tph = (uint32_t)((NBUF == 2 ? (local >> 1) : local) & 1);
            ++local;
            if (!mbar_wait_bounded(&tfull[buf], tph, abort_flag)) break;
            tc_fence_after();
            const int64_t row = (int64_t)tile * 256 + rank * 128 + q * 32 + lane;
            const bool rvalid = row < p.n;
            const uint32_t ta = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * N);
            // per input, the six term columns 32 t + m weighed by 8^-t, in order of t; 16
            // inputs at a time (registers)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float l[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) l[i] = 0.f;
#pragma unroll
                for (int t = 0; t < kQ4Terms; ++t) {
                    uint32_t v[16];
                    tmem_ld16(ta + (uint32_t)(32 * t + 16 * hh), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) l[i] = fmaf(__uint_as_float(v[i]), 1.0f / (float)(1 << (3 * t)), l[i]);
                }
                if (hh == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {  // the accumulator is free again (for this CTA)
                        if (leader) mbar_arrive(&tempty[buf]);
                        else mbar_arrive_cluster(map_rank(&tempty[buf], 0));
                    }
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = 16 * hh + i;
                    if (m >= M) break;
                    const float lv = ((l[i] * sfac[m]) * sfac[32 + m]) * gsc;
                    const bool ok = rvalid && mask_allows(p, m, row);
                    if (rvalid && p.out_logits)
                        p.out_logits[(int64_t)m * p.n + row] = ok ? f32_to_bf16(lv) : (uint16_t)0xFF80u;
                    if (lp && ok && lv > -INFINITY) {
                        float bv = best_v[m];
                        lse_merge(bv, se[m], lv, 1.f);
                    }
                    // each thread's rows arrive in increasing order: the lowest wins a tie
                    if (ok && (lv > best_v[m] || (lv == best_v[m] && best_i[m] == INT_MAX))) {
                        best_v[m] = lv;
                        best_i[m] = (int32_t)row;
                    }
                }
            }
        }
        // per input: fold the 32 lanes, then the four warps in order; publish; ticket
#pragma unroll
        for (int m = 0; m < MP; ++m) {
            if (m >= M) break;
            int32_t bi = best_i[m];
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, best_v[m], o);
                const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
                const float os = __shfl_xor_sync(0xffffffffu, se[m], o);
                if (lp) {
                    float bv = best_v[m];
                    lse_merge(bv, se[m], ov, os);
                }
                if (ov > best_v[m] || (ov == best_v[m] && oi < bi)) {
                    best_v[m] = ov;
                    bi = oi;
                }
            }
            if (lane == 0) fold[ew * 32 + m] = make_float4(best_v[m], __int_as_float(bi), se[m], 0.f);
        }
        named_sync(1, kQ4Epi * 32);
        if (ew == 0) {
            if (lane < M) {
                float bv = -INFINITY, bs = 0.f;
                int32_t bi = INT_MAX;
                for (int w = 0; w < kQ4Epi; ++w) {
                    const float4 f = fold[w * 32 + lane];
                    const int32_t fi = __float_as_int(f.y);
                    if (lp) {
                        float t = bv;
                        lse_merge(t, bs, f.x, f.z);
                    }
                    if (f.x > bv || (f.x == bv && fi < bi)) {
                        bv = f.x;
                        bi = fi;
                    }
                }
                reinterpret_cast<Partial*>(p.partials)[(int64_t)blockIdx.x * kPartSlots + lane] =
                    Partial{bv, bi, bs, 0.f};
            }
            __syncwarp();
            fence_acq_rel_gpu();  // every publishing lane's store before lane 0's ticket
            __syncwarp();
            if (*abort_flag && lane == 0) raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
            ticket_and_fold(p, lane, lp);
        }
    }
    tc_fence_before();
    cluster_sync();  // neither CTA leaves while an MMA, a copy or an arrival may reach it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}



struct Geometry {
    int kpad;
    int segs;             // 128-byte segments per row per stage
    int stages_per_tile;  // ceil(row segments / segs)
    int stage_bytes;
    int stages;
    size_t smem;
};

Geometry geometry(int M, int64_t k, int fmt, bool gather = false) {
    Geometry g{};
    g.kpad = (int)(k + 8);  // 16-byte skew between staged rows
    const int NT = M > 8 ? 2 : 1;
    const int CW = NT == 1 ? Roles<1>::CW : Roles<2>::CW;
    size_t head = (size_t)(2 * kMaxStages + 4) * 8 + 32 * sizeof(int) +
                  (size_t)2 * CW * kTileRows * 8 * NT * sizeof(float) + 32 * sizeof(float) +
                  (gather ? (size_t)kGatherInts * sizeof(int) : 0) + (size_t)M * g.kpad * 2;
    head = ((head + 1023) & ~(size_t)1023) + 1024;  // 1 KB-aligned ring, plus slack
    const int64_t row_bytes = fmt == 0 ? k * 2 : fmt == 1 ? k : k / 2;
    const int row_segs = (int)(row_bytes / 128);
    const long avail = (long)kSmemLimit - (long)head;
    // the widest stage (up to 32 segments) that still leaves a ring of >= 3 stages,
    // else >= 2; segments are spread evenly over the stages of a row
    for (int want = 3; want >= 2 && g.stages < 2; --want) {
        for (int max_segs = kMaxSegs; max_segs >= 1; max_segs /= 2) {
            const int nc = (row_segs + max_segs - 1) / max_segs;
            const int segs = (row_segs + nc - 1) / nc;
            const int sb = stage_bytes_for(fmt, segs, gather);
            int stages = avail > 0 ? (int)(avail / sb) : 0;
            if (stages > kMaxStages) stages = kMaxStages;
            if (stages >= want) {
                g.segs = segs;
                g.stages_per_tile = nc;
                g.stage_bytes = sb;
                g.stages = stages;
                break;
            }
        }
    }
    g.smem = head + (size_t)g.stages * g.stage_bytes;
    return g;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// Codes: a 3-D view (byte within a 128-byte segment, row, segment) so that one box of
// 128 B x 16 rows x 8 segments is a stage, with rows inside the 128-byte swizzle atom.
// Rows >= rows and segments past the row read as zeros.
cudaError_t make_code_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes,
                          int segs, int box_rows = kTileRows) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)(row_bytes / 128)};
    cuuint64_t strides[2] = {(cuuint64_t)row_bytes, 128};
    cuuint32_t box[3] = {128, (cuuint32_t)box_rows, (cuuint32_t)segs};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// NVFP4 block scales: [rows, pitch] bytes viewed as 16-bit elements, boxes of
// 16 * segs bytes x 16 rows (up to 512 bytes per row: two scale bytes per element).
cudaError_t make_scale_map(CUtensorMap* m, const void* base, int64_t rows, int64_t pitch,
                           int segs, int box_rows = kTileRows) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)(pitch / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)pitch};
    cuuint32_t box[2] = {(cuuint32_t)(8 * segs), (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// x [M, k] of 16-bit elements as 64-element segments: boxes of `cols` rows (inputs past
// M read as zeros) x xsegs segments, 128-byte swizzle.
cudaError_t make_x_map(CUtensorMap* m, const void* base, int M, int64_t k, int xsegs, int cols) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[3] = {64, (cuuint64_t)M, (cuuint64_t)(k / 64)};
    cuuint64_t strides[2] = {(cuuint64_t)k * 2, 128};
    cuuint32_t box[3] = {64, (cuuint32_t)cols, (cuuint32_t)xsegs};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

struct WideGeometry {
    int segs;             // 128-byte table segments per row per stage
    int stages_per_tile;
    int stage_bytes;
    int stages;
    size_t smem;
};

template <int FMT, int NT, int MODE, int BD, int G>
cudaError_t launch_one(const SweepParams& p, cudaStream_t s, SweepLaunch* info) {
    auto kern = sweep_kernel<FMT, NT, MODE, BD, G>;
    const Geometry geo = geometry(p.M, p.k, FMT, G != 0);
    if (geo.stages < 2) return cudaErrorInvalidValue;
    CUtensorMap map_codes{}, map_scales{};  // the gathered sweep copies rows without them
    cudaError_t e = cudaSuccess;
    if (!G) {
        if ((e = make_code_map(&map_codes, p.w, p.n, p.row_bytes, geo.segs)) != cudaSuccess) return e;
        if (FMT == 2) {
            if ((e = make_scale_map(&map_scales, p.block_scale, p.n, p.scale_pitch, geo.segs)) !=
                cudaSuccess)
                return e;
        } else {
            map_scales = map_codes;  // unused
        }
    }
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)geo.smem)) != cudaSuccess)
        return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    SweepParams q = p;
    if (G) q.num_tiles = (p.n + kGatherRows - 1) / kGatherRows;  // claims of kGatherRows rows
    int64_t grid = sms;
    if (grid > q.num_tiles) grid = q.num_tiles;
    if (grid > kMaxGrid) grid = kMaxGrid;
    if (grid < 1) grid = 1;
    q.kpad = geo.kpad;
    q.stages = geo.stages;
    q.stage_bytes = geo.stage_bytes;
    q.segs = geo.segs;
    q.stages_per_tile = geo.stages_per_tile;
    // programmatic stream serialization: this launch may begin while the previous
    // kernel in the stream finishes; the kernel waits for it before touching its data
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(Roles<NT>::THREADS);
    cfg.dynamicSmemBytes = geo.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, kern, q, map_codes, map_scales)) != cudaSuccess) return e;
    if (info) {
        info->grid = (int)grid;
        info->smem_bytes = (int)geo.smem;
    }
    return cudaGetLastError();
}

// Stage geometry of the tcgen05 sweep: the largest number of 128-byte segments per
// stage (at most 4) that still leaves at least four stages (else three, else two).
WideGeometry tc_geometry(int64_t k, int fmt, int N) {
    WideGeometry g{};
    size_t head = 768 + (size_t)kTEpiWarps * 32 * 16;  // barriers, misc, sfac, fold
    head = ((head + 1023) & ~(size_t)1023) + 1024;
    const int64_t row_bytes = fmt == 0 ? k * 2 : k;
    const int row_segs = (int)(row_bytes / 128);
    const long avail = (long)kSmemLimit - (long)head;
    for (int want = 4; want >= 2 && g.stages < 2; --want) {
        for (int max_segs = 4; max_segs >= 1; --max_segs) {
            const int nc = (row_segs + max_segs - 1) / max_segs;
            const int segs = (row_segs + nc - 1) / nc;
            const int sb = tc_stage_bytes(fmt, N, segs);
            int stages = avail > 0 ? (int)(avail / sb) : 0;
            if (stages > kMaxStages) stages = kMaxStages;
            if (stages >= want) {
                g.segs = segs;
                g.stages_per_tile = nc;
                g.stage_bytes = sb;
                g.stages = stages;
                break;
            }
        }
    }
    g.smem = head + (size_t)g.stages * g.stage_bytes;
    return g;
}

template <int FMT, int N>
cudaError_t launch_tc(const SweepParams& p, cudaStream_t s, SweepLaunch* info) {
    auto kern = sweep_tc_kernel<FMT, N>;
    const WideGeometry geo = tc_geometry(p.k, FMT, N);
    if (geo.stages < 2) return cudaErrorInvalidValue;
    CUtensorMap map_codes, map_x;
    cudaError_t e = make_code_map(&map_codes, p.w, p.n, p.row_bytes, geo.segs, kTRows);
    if (e != cudaSuccess) return e;
    uint8_t* xq = reinterpret_cast<uint8_t*>(p.x16);
    if (FMT == 0)
        e = make_x_map(&map_x, p.x, p.M, p.k, geo.segs, N);
    else
        e = make_code_map(&map_x, xq, 2 * N, p.k, geo.segs, 2 * N);
    if (e != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)geo.smem)) != cudaSuccess)
        return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    SweepParams q = p;
    q.num_tiles = (p.n + kTRows - 1) / kTRows;
    q.stages = geo.stages;
    q.stage_bytes = geo.stage_bytes;
    q.segs = geo.segs;
    q.stages_per_tile = geo.stages_per_tile;
    int64_t grid = sms;
    if (grid > q.num_tiles) grid = q.num_tiles;
    if (grid > kMaxGrid) grid = kMaxGrid;
    if (grid < 1) grid = 1;
    if (FMT == 1) {  // the two E4M3 planes of x the FP8 MMAs read
        tc_xq_kernel<<<N, 256, 0, s>>>(p.x, p.M, (int)p.k, N, xq, p.xexp);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kTThreads);
    cfg.dynamicSmemBytes = geo.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, kern, q, map_codes, map_x)) != cudaSuccess) return e;
    if (info) {
        info->grid = (int)grid;
        info->smem_bytes = (int)geo.smem;
    }
    return cudaGetLastError();
}

// Stage geometry of the NVFP4 tcgen05 sweep: two 128-byte segments per row per stage when
// that leaves at least three stages, else one segment (at least two stages).

WideGeometry q4_geometry(int64_t k, int N) {
    WideGeometry g{};
    const int row_segs = (int)(k / 256);  // 128-byte code segments per row
    const long avail = (long)kSmemLimit - (long)kQ4Head;
    for (int segs = 2; segs >= 1 && g.stages == 0; --segs) {
        if (segs > row_segs) continue;
        const int sb = q4_stage_bytes(N, segs);
        int stages = avail > 0 ? (int)(avail / sb) : 0;
        stages = min(stages, min(kMaxStages, q4_max_slots(N, segs)));
        if (stages >= (segs == 2 ? 3 : 2)) {
            g.segs = segs;
            g.stages_per_tile = (row_segs + segs - 1) / segs;
            g.stage_bytes = sb;
            g.stages = stages;
        }
    }
    g.smem = (size_t)kQ4Head + (size_t)g.stages * g.stage_bytes;
    return g;
}

template <int MP>
cudaError_t launch_q4(const SweepParams& p, cudaStream_t s, SweepLaunch* info) {
    constexpr int N = q4_n(MP);
    auto kern = sweep_q4_kernel<MP>;
    const WideGeometry geo = q4_geometry(p.k, N);
    if (geo.stages < 2) return cudaErrorInvalidValue;
    uint8_t* xcodes = reinterpret_cast<uint8_t*>(p.x16);
    uint8_t* xscales = xcodes + q4_code_bytes(N, p.k);
    CUtensorMap map_codes, map_scales, map_x, map_xs;
    cudaError_t e = make_code_map(&map_codes, p.w, p.n, p.row_bytes, geo.segs, 128);
    if (e != cudaSuccess) return e;
    if ((e = make_scale_map(&map_scales, p.block_scale, p.n, p.scale_pitch, geo.segs, 128)) != cudaSuccess)
        return e;
    if ((e = make_code_map(&map_x, xcodes, N, p.k / 2, geo.segs, N)) != cudaSuccess) return e;
    if ((e = make_scale_map(&map_xs, xscales, N, p.k / 16, geo.segs, N)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)geo.smem)) !=
        cudaSuccess)
        return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    SweepParams q = p;
    q.num_tiles = (p.n + 127) / 128;
    q.stages = geo.stages;
    q.stage_bytes = geo.stage_bytes;
    q.segs = geo.segs;
    q.stages_per_tile = geo.stages_per_tile;
    int64_t grid = sms;
    if (grid > q.num_tiles) grid = q.num_tiles;
    if (grid > kMaxGrid) grid = kMaxGrid;
    if (grid < 1) grid = 1;
    q4_xterms_kernel<<<MP + 1, 256, 0, s>>>(p.x, p.M, (int)p.k, MP, N, xcodes, xscales, p.xexp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kQ4Threads);
    cfg.dynamicSmemBytes = geo.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, kern, q, map_codes, map_scales, map_x, map_xs)) != cudaSuccess)
        return e;
    if (info) {
        info->grid = (int)grid;
        info->smem_bytes = (int)geo.smem;
    }
    return cudaGetLastError();
}

cudaError_t launch_q4_any(const SweepParams& p, cudaStream_t s, SweepLaunch* info) {
    switch (q4_mp(p.M)) {
        case 4: return launch_q4<4>(p, s, info);
        case 8: return launch_q4<8>(p, s, info);
        default: return launch_q4<16>(p, s, info);
    }
}

WideGeometry q4p_geometry(int64_t k) {
    WideGeometry g{};
    const int row_segs = (int)(k / 256);  // 128-byte code segments per row
    const long avail = (long)kSmemLimit - (long)kQ4Head;
    for (int segs = 2; segs >= 1 && g.stages == 0; --segs) {
        if (segs > row_segs) continue;
        const int sb = q4p_stage_bytes(segs);
        int stages = avail > 0 ? (int)(avail / sb) : 0;
        stages = min(stages, min(kMaxStages, q4p_max_slots(segs)));
        if (stages >= (segs == 2 ? 3 : 2)) {
            g.segs = segs;
            g.stages_per_tile = (row_segs + segs - 1) / segs;
            g.stage_bytes = sb;
            g.stages = stages;
        }
    }
    g.smem = (size_t)kQ4Head + (size_t)g.stages * g.stage_bytes;
    return g;
}

cudaError_t launch_q4p(const SweepParams& p, cudaStream_t s, SweepLaunch* info) {
    constexpr int MP = 32, N = q4_n(MP);
    auto kern = sweep_q4p_kernel;
    const WideGeometry geo = q4p_geometry(p.k);
    if (geo.stages < 2) return cudaErrorInvalidValue;
    uint8_t* xcodes = reinterpret_cast<uint8_t*>(p.x16);
    uint8_t* xscales = xcodes + q4_code_bytes(N, p.k);
    CUtensorMap map_codes, map_scales, map_x, map_xs;
    cudaError_t e = make_code_map(&map_codes, p.w, p.n, p.row_bytes, geo.segs, 128);
    if (e != cudaSuccess) return e;
    if ((e = make_scale_map(&map_scales, p.block_scale, p.n, p.scale_pitch, geo.segs, 128)) != cudaSuccess)
        return e;
    if ((e = make_code_map(&map_x, xcodes, N, p.k / 2, geo.segs, N / 2)) != cudaSuccess) return e;
    if ((e = make_scale_map(&map_xs, xscales, N, p.k / 16, geo.segs, N)) != cudaSuccess) return e;
    const size_t smem = geo.smem;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
        cudaSuccess)
        return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    SweepParams q = p;
    q.num_tiles = (p.n + 255) / 256;  // pair tiles
    q.stages = geo.stages;
    q.stage_bytes = geo.stage_bytes;
    q.segs = geo.segs;
    q.stages_per_tile = geo.stages_per_tile;
    int64_t pairs = sms / 2;
    if (pairs > q.num_tiles) pairs = q.num_tiles;
    if (pairs > kMaxGrid / 2) pairs = kMaxGrid / 2;
    if (pairs < 1) pairs = 1;
    q4_xterms_kernel<<<MP + 1, 256, 0, s>>>(p.x, p.M, (int)p.k, MP, N, xcodes, xscales, p.xexp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(kQ4Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, kern, q, map_codes, map_scales, map_x, map_xs)) != cudaSuccess)
        return e;
    if (info) {
        info->grid = (int)(2 * pairs);
        info->smem_bytes = (int)smem;
    }
    return cudaGetLastError();
}


// Argmax sweeps that stream x per K chunk -- the tcgen05 sweeps -- take FP8 tables from 7
// inputs on (measured faster than 16-row tiles from there), BF16 from 9; NVFP4 tables from
// 17 (3-16 run on the block-scaled sweep, which streams its x terms the same way). The
// NVFP4 sweep with A in tensor memory (17-32) is bound by its MMA issue: sixteen 128 x 32
// x 16 MMAs per 256-element slot at ~50 cycles each, with the decode warps waiting on
// them (221 us at M = 32 on the 131,072 x 5,120 table).
inline bool streams_x(int M, int fmt) { return fmt == 1 ? M >= 7 : M > 8; }

}  // namespace

// A grammar mask with up to eight inputs: the gathered sweep, which reads only the rows
// some input's mask allows.
inline bool gathers(int M, bool masked) { return masked && M <= 8; }

size_t sweep_smem_bytes(int M, int64_t k, int fmt, int* kpad_out, int mode, bool masked) {
    if (mode == 0 && gathers(M, masked)) {
        const Geometry g = geometry(M, k, fmt, true);
        if (kpad_out) *kpad_out = g.kpad;
        return g.stages >= 2 ? g.smem : (size_t)kSmemLimit + 1;
    }
    if (mode == 0 && fmt == 2 && M >= 3) {  // the block-scaled sweeps
        const WideGeometry w = M <= kQ4MaxM ? q4_geometry(k, q4_n(q4_mp(M))) : q4p_geometry(k);
        if (kpad_out) *kpad_out = (int)k;
        return w.stages >= 2 ? w.smem : (size_t)kSmemLimit + 1;
    }
    if (mode == 0 && streams_x(M, fmt)) {  // the tcgen05 sweeps stage x per K chunk
        const WideGeometry w = tc_geometry(k, fmt, M > 16 ? 32 : 16);
        if (kpad_out) *kpad_out = (int)k;
        return w.stages >= 2 ? w.smem : (size_t)kSmemLimit + 1;
    }
    const Geometry g = geometry(M, k, fmt);
    if (kpad_out) *kpad_out = g.kpad;
    return g.stages >= 2 ? g.smem : (size_t)kSmemLimit + 1;
}

int sweep_max_grid() { return kMaxGrid; }

size_t sweep_x16_bytes(int M, int64_t k, int fmt) {
    if (fmt == 2 && M <= 2) return 0;
    if (fmt == 2) {  // the block-scaled sweeps' x terms: codes, scales, exponents
        const int N = M <= kQ4MaxM ? q4_n(q4_mp(M)) : q4_n(32);
        return q4_code_bytes(N, k) + q4_scale_bytes(N, k) + 1024;
    }
    if (fmt == 0 || !streams_x(M, fmt)) return 0;
    // FP8: x's two E4M3 planes of 16 or 32 rows. Then 1 KB for the per-input exponents.
    const size_t body = (size_t)2 * (M > 16 ? 32 : 16) * (size_t)k;
    return ((body + 1023) & ~(size_t)1023) + 1024;
}

namespace {

// One warp per input: lane l folds parts l, l + 32, ... in order, then a fixed shuffle
// tree; ties go to the lowest row, so the argmax does not depend on the order.
__global__ void __launch_bounds__(32) merge_partials_kernel(const Partial* parts, int n_parts, int M,
                                                            int32_t* out_idx, float* out_val,
                                                            float* out_logprob, int32_t* dev_err) {
    const int m = blockIdx.x, lane = threadIdx.x;
    float bv = -INFINITY, bs = 0.f;
    int32_t bi = INT_MAX;
    for (int r = lane; r < n_parts; r += 32) {
        const float4 e = __ldg(reinterpret_cast<const float4*>(parts + (int64_t)r * M + m));
        const int32_t ei = __float_as_int(e.y);
        if (ei == INT_MAX) continue;  // nothing allowed in that shard
        float v = bv;
        lse_merge(v, bs, e.x, e.z);
        if (e.x > bv || (e.x == bv && ei < bi)) {
            bv = e.x;
            bi = ei;
        }
    }
    for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
        const float os = __shfl_xor_sync(0xffffffffu, bs, o);
        float v = bv;
        lse_merge(v, bs, ov, os);
        if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
        }
    }
    if (lane == 0) {
        const bool empty = bi == INT_MAX;
        if (empty) raise_flag(dev_err, DEVFLAG_EMPTY_MASK);
        out_idx[m] = empty ? 0 : bi;
        if (out_val) out_val[m] = empty ? -INFINITY : bv;
        if (out_logprob) out_logprob[m] = empty ? -INFINITY : -logf(bs);
    }
}

}  // namespace

cudaError_t merge_partials_launch(const void* parts, int n_parts, int M, int32_t* out_idx,
                                  float* out_val, float* out_logprob, int32_t* dev_err,
                                  cudaStream_t s) {
    merge_partials_kernel<<<M, 32, 0, s>>>(static_cast<const Partial*>(parts), n_parts, M, out_idx,
                                            out_val, out_logprob, dev_err);
    return cudaGetLastError();
}

cudaError_t sweep_launch(const SweepParams& p, int fmt, int mode, cudaStream_t s,
                         SweepLaunch* info) {
    const bool two = p.M > 8;
    if (mode == 0 && gathers(p.M, p.mask != nullptr)) {
        if (fmt == 0) return launch_one<0, 1, 0, 0, 1>(p, s, info);
        if (fmt == 1) return launch_one<1, 1, 0, 0, 1>(p, s, info);
        if (fmt == 2)
            return p.M <= 2 ? launch_one<2, 1, 0, 1, 1>(p, s, info) : launch_one<2, 1, 0, 0, 1>(p, s, info);
    }
    // NVFP4 with one or two inputs: per-block fp32 sums of unscaled codes (measured faster
    // than the block-scaled sweep there, 67.8 against 71.5 us on the 131,072 x 5,120 table)
    if (fmt == 2 && mode == 0 && p.M <= 2) return launch_one<2, 1, 0, 1, 0>(p, s, info);
    if (fmt == 2 && mode == 0 && p.M <= kQ4MaxM) return launch_q4_any(p, s, info);
    if (fmt == 2 && mode == 0) return launch_q4p(p, s, info);  // 17-32 inputs, CTA pairs
    if (mode == 0 && streams_x(p.M, fmt)) {
        const bool four = p.M > 16;
        if (fmt == 0) return four ? launch_tc<0, 32>(p, s, info) : launch_tc<0, 16>(p, s, info);
        if (fmt == 1) return four ? launch_tc<1, 32>(p, s, info) : launch_tc<1, 16>(p, s, info);
    }
#define MTP_SWEEP_CASE(F, NTV, MD) \
    if (fmt == F && (NTV == 2) == two && mode == MD) return launch_one<F, NTV, MD, 0, 0>(p, s, info);
    // (mode 0 inputs past streams_x went to the tcgen05 sweeps above, NVFP4 ones to the
    // block-scaled and block-diagonal sweeps)
    MTP_SWEEP_CASE(0, 1, 0) MTP_SWEEP_CASE(1, 1, 0)
    MTP_SWEEP_CASE(0, 1, 1) MTP_SWEEP_CASE(0, 2, 1)
    MTP_SWEEP_CASE(1, 1, 1) MTP_SWEEP_CASE(1, 2, 1)
    MTP_SWEEP_CASE(2, 1, 1) MTP_SWEEP_CASE(2, 2, 1)
#undef MTP_SWEEP_CASE
    return cudaErrorInvalidValue;
}

}  // namespace mtp
