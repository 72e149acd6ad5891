// Drafter-context prefill: the K/V cache rows of the MTP drafter for a whole prompt.
//
// What it computes (spark_model/layers/mtp_head.rs, the drafter-prefill docs and
// MtpPrefillScratch: the drafter's K/V for prompt row i depend only on
// (embed(token_{i+1}), target_hidden_i), so no attention runs; block size 16 and the
// FP8 cache in metrale_model_layers/layers/mtp_head/new.rs; the slot rule of
// metrale_model_arch/deepseek_v4_mtp.rs forward_one step 4). Per prompt row r:
//   c  = [bf16(rms(embed[tok_r]) w_e) || bf16(rms(hidden_r) w_h)]           (prologue)
//   y  = bf16(fc . c)                                                   (fc GEMM)
//   (optional input norm: y <- bf16(rms(y) w_in), by the row block's last fc tile)
//   k  = bf16(Wk . y), v = bf16(Wv . y)                                 (k/v GEMM)
//   (optional per-head k norm before RoPE, in the k/v epilogue)
//   k' = bf16(RoPE_neox(k, pos_r)) per head, codes = e4m3(k' / k_scale), e4m3(v / v_scale)
//   cache row p = cache_start + r, slot = block_table[p / bs] * bs + p % bs,
//   element (slot, head, d) of a [num_blocks, bs, nkv, hd] cache.       (k/v epilogue)
//
// Design (B200): rows are processed in chunks (the reference's PREFILL_CHUNK), whose
// buffers (concat rows, fc output, RoPE table) live in the caller's workspace. The whole
// call is ONE persistent kernel on the caller's stream, launched as CTA pairs (2-CTA
// clusters, one CTA per SM): the pairs take GEMM work items ("tiles") from one counter and
// every CTA's prologue warps take prologue tiles from another, each in a fixed global
// order, so that the tiles of the next chunk fill the SMs the current chunk leaves idle (a
// 2,048-row chunk's fc GEMM is 160 pair tiles, 2.16 waves on 74 pairs). Three kinds of
// tile:
//   P (chunk c, row block m, part n): the prologue of 8 rows, taken from its own counter
//     by each CTA's two prologue warps whenever they are free: they read each row's
//     embedding row and hidden row into registers, take the two RMSNorms, write the
//     bf16 concat rows and the rows' RoPE table (the angle reduced in double, cos and
//     sin in fp32), alongside the GEMM tiles, whose shared-memory ring they never use.
//   F (c, m, n): a 256 x 256 tile of the fc GEMM, y = c . fc^T, bf16 out (rows 256 m ..;
//     the pair's CTA r holds row block 2 m + r).
//   V (c, m, n): a 256 x 256 tile of the k/v GEMM whose epilogue rotates k (RoPE),
//     encodes E4M3 and writes each row's 32-byte pieces at its paged slot.
// GEMM order: for b = 0..chunks: F(b), then V(b - 1) (with a single lane V(b - 1) first).
// Completion counters per chunk slot and 128-row block (in the workspace header,
// release/acquire at GPU scope; each CTA of a pair waits for and counts its own block)
// order the tiles: F(c, m, .) waits for P(c, m, .);
// V(c, m, .) for all of F(c, m, .); and a tile that overwrites a buffer another chunk
// used (two lanes of concat and fc-output rows, three of RoPE rows) for that chunk's
// readers. A GEMM tile only waits for GEMM tiles earlier in its order and for P tiles; a
// P tile only for GEMM tiles of chunks two and three back, whose own P tiles were taken
// earlier from the P counter. Tiles are claimed only by running CTAs, so every wait
// ends (every pair of the grid is resident at once). GEMM tiles run on the 5th-generation
// tensor cores as cta_group::2 MMAs of 256 x 256 x 16: each CTA's 6-stage TMA ring (128-byte
// swizzle, K-major) holds its 128 rows of A and 128 of the tile's 256 B rows, so each SM
// stages and reads half the B it would alone; both CTAs' copies complete on rank 0's
// barrier, rank 0's thread issues the MMAs into both SMs' double-buffered 512-column
// TMEM accumulators and its commits free both CTAs' stages; each CTA's four epilogue
// warps read back its own 128 rows with tcgen05.ld while the next tile accumulates. Rank
// 0 announces each tile to both CTAs through a small FIFO in each one's shared memory
// (remote stores and mbarrier arrivals). Every wait is bounded (abort flag +
// MTP_DEVFLAG_TIMEOUT): nothing hangs.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace mtp {
namespace {

// A GEMM tile is 256 rows x BN columns, computed by a CTA pair (a 2-CTA cluster on one
// TPC) with cta_group::2 MMAs of M = 256: each CTA stages its own 128 rows of A and half
// of the tile's B rows, and holds its 128 rows x BN of the accumulator.
constexpr int BM = 128, BN = 256, BK = 64;
constexpr int BNH = BN / 2;                 // B rows each CTA of the pair stages
constexpr int kGStages = 6;
constexpr int kAStageBytes = BM * BK * 2;   // 16 KB
constexpr int kBStageBytes = BNH * BK * 2;  // 16 KB
constexpr int kGStageBytes = kAStageBytes + kBStageBytes;
// warp 0 TMA, warp 1 MMA, warps 2-5 epilogue, warps 6-7 prologue
constexpr int kGemmThreads = 256;
constexpr int kEpiThreads = 128;
constexpr int kProThreads = 64;
constexpr int kTmemCols = 2 * BN;  // two fp32 accumulators of 128 lanes x 256 columns
constexpr int kFifo = 8;           // tiles announced ahead to the MMA and epilogue warps
constexpr int kCtrSlots = 4;       // completion counters: chunk c uses slot c % 4
constexpr int kMaxLanes = 2;       // concat / fc-output lanes (RoPE rows: lanes + 1)
// shared memory after the ring: barriers, the tile FIFO, per-stage row tokens and the
// inverse frequencies
constexpr int kHeadBytes = 4096;
constexpr int kGemmSmem = kGStages * kGStageBytes + kHeadBytes + 1024 /* align */;
// After those, when they fit: the norm weights (w_ne, w_nh, then the input norm's), read
// by the epilogue warps for every row from shared memory instead of through L1.
constexpr int kSmemMax = 227 * 1024;

enum : int { TILE_P = 0, TILE_F = 1, TILE_V = 2 };
// A 128-row block's prologue is split into kPParts P tiles of kPRows rows, so that every
// SM's prologue warps share a chunk's prologue.
constexpr int kPParts = 16, kPRows = BM / kPParts;
constexpr int kArrivals = 3;  // counter kind: F tiles that finished (input norm only)

struct PrefillParams {
    // inputs
    const uint16_t* embed;
    int64_t vocab;
    const int32_t* tokens;
    const uint16_t* hidden;
    int64_t R;
    int h;
    const uint16_t* w_ne;
    const uint16_t* w_nh;
    float eps;
    int norm_mode;           // 0: weights w, 1: weights 1 + w
    const uint16_t* k_norm;  // [hd] or null: per-head RMSNorm of k before RoPE
    const uint16_t* in_norm;  // [h] or null: RMSNorm of y (in place) before the k/v GEMM
    int nkv, hd;
    double rope_base;
    const int32_t* rope_pos;
    int64_t cache_start;
    const int32_t* block_table;
    int64_t n_table;
    int block_size;
    int64_t num_blocks;
    uint8_t* k_cache;
    uint8_t* v_cache;
    float k_scale, v_scale;
    int32_t* dev_err;
    // schedule
    int plain;           // 1: a plain GEMM C = A . B^T (stage check), F tiles only
    int64_t chunk;       // rows per chunk
    int n_chunks;
    int mt_full;         // 128-row blocks of a full chunk
    int mt_last;         // of the last chunk
    int mp_full;         // 256-row pair blocks (GEMM tile rows) of a full chunk
    int mp_last;         // of the last chunk
    int nf;              // fc GEMM column tiles (h / 256)
    int nv;              // k/v GEMM column tiles (2 nkv hd / 256)
    int64_t total;       // GEMM tiles (the tile counter's range)
    int64_t p_total;     // prologue tiles (the prologue counter's range)
    int lanes;           // 1 or 2
    int w_in_smem;       // 1: the norm weights are staged in shared memory
    uint32_t* ctr;       // [0] GEMM tile counter, [1] prologue tile counter; then done
                         // counters [4][kCtrSlots][mt_full] from word 64
    uint16_t* concat[kMaxLanes];
    uint16_t* y[kMaxLanes];
    float2* rope[kMaxLanes + 1];
    // plain GEMM
    uint16_t* C;
    int M, N, K;
};

// kind, chunk, rows, column tile. m is a pair block (rows 256 m ..) for GEMM tiles, whose
// two 128-row blocks 2 m + r are those of the pair's CTA r; a 128-row block for P tiles.
struct Tile {
    int kind, c, m, n;
};

__device__ __forceinline__ int mt_of(const PrefillParams& p, int c) {
    return c == p.n_chunks - 1 ? p.mt_last : p.mt_full;
}
__device__ __forceinline__ int mp_of(const PrefillParams& p, int c) {
    return c == p.n_chunks - 1 ? p.mp_last : p.mp_full;
}

// Row blocks (pair blocks) of chunks 0 .. k - 1.
__device__ __forceinline__ int64_t cum_mt(const PrefillParams& p, int k) {
    k = max(0, min(k, p.n_chunks));
    return k <= p.n_chunks - 1 ? (int64_t)k * p.mt_full
                               : (int64_t)(p.n_chunks - 1) * p.mt_full + p.mt_last;
}
__device__ __forceinline__ int64_t cum_mp(const PrefillParams& p, int k) {
    k = max(0, min(k, p.n_chunks));
    return k <= p.n_chunks - 1 ? (int64_t)k * p.mp_full
                               : (int64_t)(p.n_chunks - 1) * p.mp_full + p.mp_last;
}

// First GEMM tile of block b (b = 0 .. n_chunks + 1). With two lanes block b holds F(b),
// then V(b - 1); with one lane V(b - 1), then F(b), since F(b) then reuses the fc-output
// rows V(b - 1) reads.
__device__ __forceinline__ int64_t block_start(const PrefillParams& p, int b) {
    return p.nf * cum_mp(p, b) + p.nv * cum_mp(p, b - 1);
}

// GEMM tile t of the global order.
__device__ Tile decode(const PrefillParams& p, int64_t t) {
    Tile r{};
    if (p.plain) {  // F tiles of one GEMM, M-fastest
        const int mp = (p.M + 2 * BM - 1) / (2 * BM);
        r.kind = TILE_F;
        r.c = 0;
        r.m = (int)(t % mp);
        r.n = (int)(t / mp);
        return r;
    }
    int lo = 0, hi = p.n_chunks;  // the last block starting at or before t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (block_start(p, mid) <= t) lo = mid;
        else hi = mid - 1;
    }
    const int b = lo, n = p.n_chunks;
    int64_t off = t - block_start(p, b);
    // the block's segments in order; the tile is in the first one that still covers off
    bool found = false;
    auto seg = [&](int kind, int c) {
        if (found) return;
        const int mp = mp_of(p, c);
        const int64_t cnt = (int64_t)mp * (kind == TILE_F ? p.nf : p.nv);
        if (off < cnt) {  // M-fastest
            r.kind = kind;
            r.c = c;
            r.m = (int)(off % mp);
            r.n = (int)(off / mp);
            found = true;
        } else {
            off -= cnt;
        }
    };
    if (p.lanes == 2) {
        if (b < n) seg(TILE_F, b);
        if (b >= 1) seg(TILE_V, b - 1);
    } else {
        if (b >= 1) seg(TILE_V, b - 1);
        if (b < n) seg(TILE_F, b);
    }
    return r;
}

// Prologue tile i: chunk by chunk, row block by row block, part by part.
__device__ Tile decode_p(const PrefillParams& p, int64_t i) {
    int lo = 0, hi = p.n_chunks - 1;  // the last chunk whose first P tile is at or before i
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (kPParts * cum_mt(p, mid) <= i) lo = mid;
        else hi = mid - 1;
    }
    const int64_t off = i - kPParts * cum_mt(p, lo);
    Tile r{};
    r.kind = TILE_P;
    r.c = lo;
    r.m = (int)(off / kPParts);
    r.n = (int)(off % kPParts);
    return r;
}

// Prompt rows of P tile (c, m, part n): up to kPRows, none past the chunk's last row.
__device__ __forceinline__ int p_tile_rows(const PrefillParams& p, const Tile& tl) {
    const int64_t rows_c = min(p.chunk, p.R - (int64_t)tl.c * p.chunk);
    const int64_t r = rows_c - (int64_t)tl.m * BM - (int64_t)tl.n * kPRows;
    return (int)max((int64_t)0, min((int64_t)kPRows, r));
}

// Completion counters: kind k (P, F, V, F arrivals) of the chunks in slot c % 4, row
// block m. They only grow within a call: after chunk c's tiles of row block m are all
// done, the P counter reads (c / 4 + 1) kPParts, F (c / 4 + 1) nf, V (c / 4 + 1) nv. With the input
// norm the F tiles count themselves on the arrivals counter instead, and the last of a row
// block normalizes the block's fc output rows in place, then adds nf to the F counter.
__device__ __forceinline__ uint32_t* counter(const PrefillParams& p, int kind, int c, int m) {
    return p.ctr + 64 + ((size_t)kind * kCtrSlots + (size_t)(c % kCtrSlots)) * p.mt_full + m;
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ bool wait_counter(const uint32_t* a, uint32_t target, volatile int* abort) {
    return counter_wait_bounded(a, target, abort);
}

// One thread of the writers adds 1 once every writer's stores are visible (the caller
// has synchronised the writers): a GPU-scope release.
__device__ __forceinline__ void counter_release_add(uint32_t* a, uint32_t v) {
    fence_acq_rel_gpu();
    atomicAdd(a, v);
}

// Cache slot of prompt row `prompt_row`, or -1 when its block is missing / out of range.
__device__ __forceinline__ int64_t cache_slot(const PrefillParams& p, int64_t prompt_row) {
    const int64_t pos = p.cache_start + prompt_row;
    if (pos < 0) return -1;
    const int64_t b = pos / p.block_size;
    if (b >= p.n_table) return -1;
    const int64_t blk = p.block_table[b];
    if (blk < 0 || blk >= p.num_blocks) return -1;
    return blk * p.block_size + pos % p.block_size;
}

// 32 bf16-rounded values (as fp32) -> E4M3 codes of value / scale -> 32 bytes at dst.
__device__ __forceinline__ void store_codes32(uint8_t* dst, const float (&v)[32], float scale) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t lo = f32x2_to_e4m3x2(__fdiv_rn(v[4 * i], scale), __fdiv_rn(v[4 * i + 1], scale));
        const uint32_t hi =
            f32x2_to_e4m3x2(__fdiv_rn(v[4 * i + 2], scale), __fdiv_rn(v[4 * i + 3], scale));
        w[i] = lo | (hi << 16);
    }
    uint4* d = reinterpret_cast<uint4*>(dst);
    d[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// Both values rounded to bf16 (round to nearest even) by one packed convert.
__device__ __forceinline__ void round_bf16x2(float& a, float& b) {
    const uint32_t r = f32x2_to_bf16x2(a, b);
    a = bf16_lo(r);
    b = bf16_hi(r);
}

// NeoX rotation of one head's pair block: lo = k[j], hi = k[j + hd/2] for 32 j's.
__device__ __forceinline__ void rope32(float (&lo)[32], float (&hi)[32], const float2* cs) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float2 t = cs[j];
        const float a = lo[j], b = hi[j];
        lo[j] = fmaf(a, t.x, -b * t.y);
        hi[j] = fmaf(b, t.x, a * t.y);
        round_bf16x2(lo[j], hi[j]);
    }
}

// Packed fp32 pairs (element 0 in the low word) and their round-to-nearest arithmetic:
// one instruction for two IEEE operations.
__device__ __forceinline__ uint64_t f32x2_of_bf16x2(uint32_t w) {
    return ((uint64_t)(w & 0xFFFF0000u) << 32) | (uint64_t)(w << 16);
}
__device__ __forceinline__ uint64_t f32x2_splat(float f) {
    const uint64_t b = __float_as_uint(f);
    return (b << 32) | b;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint32_t bf16x2_of_f32x2(uint64_t v) {
    return f32x2_to_bf16x2(__uint_as_float((uint32_t)v), __uint_as_float((uint32_t)(v >> 32)));
}

// 8 bf16 (one 16-byte piece) times a row factor and 8 norm weights (plus `add`: 0 for
// weights w, 1 for 1 + w), rounded to bf16: bf16((x inv) (w + add)) per element.
__device__ __forceinline__ uint4 norm8(uint4 v, uint64_t inv2, uint4 w, uint64_t add2) {
    const uint32_t a[4] = {v.x, v.y, v.z, v.w}, b[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        o[i] = bf16x2_of_f32x2(mul_f32x2(mul_f32x2(f32x2_of_bf16x2(a[i]), inv2),
                                         add_f32x2(f32x2_of_bf16x2(b[i]), add2)));
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Sum of squares of 8 bf16, accumulated as even and odd elements in a packed pair.
__device__ __forceinline__ uint64_t sumsq8(uint4 v, uint64_t acc) {
    const uint32_t a[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint64_t x = f32x2_of_bf16x2(a[i]);
        acc = fma_f32x2(x, x, acc);
    }
    return acc;
}
__device__ __forceinline__ float hsum_f32x2(uint64_t v) {
    return __uint_as_float((uint32_t)v) + __uint_as_float((uint32_t)(v >> 32));
}

// 32 bytes of a row that is read once: not kept in L1 and first out of L2, so that it does
// not push out the GEMM operands. `p` 32-byte aligned.
__device__ __forceinline__ void ld256_once(const void* p, uint4& a, uint4& b) {
    asm volatile(
        "ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
        : "l"(p));
}

// One warp: dst[j] = bf16((src[j] inv) (w[j] + add)) over a bf16 row of `pieces` 16-byte
// pieces (an even number; src 32-byte aligned), inv = 1 / sqrt(mean(src^2) + eps); src
// null reads as a zero row. Up to 32 x kNormRegs pieces are held in registers (one read,
// 32 bytes per lane and load), longer rows are read twice.
constexpr int kNormRegs = 20;
__device__ __forceinline__ void norm_row(const uint4* src, const uint4* w, uint4* dst, int pieces,
                                         int lane, float eps, uint64_t wadd) {
    const uint4 z = make_uint4(0, 0, 0, 0);
    uint64_t s2 = 0;
    if (pieces <= 32 * kNormRegs) {
        uint4 v[kNormRegs];
#pragma unroll
        for (int i = 0; i < kNormRegs / 2; ++i) {
            const int j = 2 * (lane + 32 * i);  // this lane's pair of pieces
            v[2 * i] = v[2 * i + 1] = z;
            if (src && j < pieces) ld256_once(src + j, v[2 * i], v[2 * i + 1]);
        }
#pragma unroll
        for (int i = 0; i < kNormRegs; ++i) s2 = sumsq8(v[i], s2);
        float ss = hsum_f32x2(s2);
#pragma unroll
        for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const uint64_t inv = f32x2_splat(1.0f / sqrtf(ss / (float)(8 * pieces) + eps));
#pragma unroll
        for (int i = 0; i < kNormRegs / 2; ++i) {
            const int j = 2 * (lane + 32 * i);
            if (j < pieces) {
                dst[j] = norm8(v[2 * i], inv, w[j], wadd);
                dst[j + 1] = norm8(v[2 * i + 1], inv, w[j + 1], wadd);
            }
        }
        return;
    }
#pragma unroll 4
    for (int j = lane; j < pieces; j += 32) s2 = sumsq8(src ? __ldg(src + j) : z, s2);
    float ss = hsum_f32x2(s2);
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const uint64_t inv = f32x2_splat(1.0f / sqrtf(ss / (float)(8 * pieces) + eps));
#pragma unroll 4
    for (int j = lane; j < pieces; j += 32) dst[j] = norm8(src ? __ldg(src + j) : z, inv, w[j], wadd);
}

struct Maps {
    CUtensorMap a_concat[kMaxLanes];  // plain GEMM: a_concat[0] is A
    CUtensorMap a_y[kMaxLanes];
    CUtensorMap b_fc;                 // plain GEMM: B
    CUtensorMap b_wk, b_wv;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ Maps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* stages = smem;
    uint8_t* head = smem + kGStages * kGStageBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(head);
    uint64_t* empty = full + kGStages;
    uint64_t* tfull = empty + kGStages;    // [2]
    uint64_t* tempty = tfull + 2;          // [2]
    uint64_t* done = tempty + 2;           // MMA drain at exit
    uint64_t* qfull = done + 1;            // [kFifo] a tile index is in the FIFO slot
    uint64_t* qempty = qfull + kFifo;      // [kFifo] every reader took it
    int* fifo = reinterpret_cast<int*>(qempty + kFifo);          // [kFifo]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fifo + kFifo);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;  // this F tile was its row block's last
    double* inv_freq = reinterpret_cast<double*>(head + 2048);   // [hd / 2 <= 128], in turns
    uint16_t* kn_s = reinterpret_cast<uint16_t*>(head + 3072);   // [hd <= 256] k norm weights
    uint4* w_s = reinterpret_cast<uint4*>(head + kHeadBytes);    // [2 or 3][h / 8] norm weights

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvd = p.nkv * p.hd;
    // The pair: rank 0 claims the GEMM tiles, announces each to both CTAs, and issues the
    // MMAs; both CTAs stage their operands and run their own epilogue and prologue warps.
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);   // rank 0's: its expect_tx; both CTAs' copies count on it
            mbar_init(&empty[s], 1);  // the MMA commit, to both CTAs
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);   // the MMA commit, to both CTAs
            mbar_init(&tempty[b], 2);  // rank 0's: one epilogue thread of each CTA
        }
        for (int q = 0; q < kFifo; ++q) {
            mbar_init(&qfull[q], 1);
            mbar_init(&qempty[q], 4);  // rank 0's: its MMA and epilogue warps, rank 1's
                                       // producer and epilogue warps
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    const int half = p.hd / 2;
    if (!p.plain) {  // the rotation per position of each pair, in turns; norm weights
        for (int j = threadIdx.x; j < half; j += kGemmThreads)
            inv_freq[j] = pow(p.rope_base, -2.0 * (double)j / (double)p.hd) /
                          (2.0 * 3.14159265358979323846);
        if (p.k_norm)
            for (int j = threadIdx.x; j < p.hd; j += kGemmThreads) kn_s[j] = p.k_norm[j];
        if (p.w_in_smem) {
            const int pc = p.h / 8;
            for (int j = threadIdx.x; j < pc; j += kGemmThreads) {
                w_s[j] = __ldg(reinterpret_cast<const uint4*>(p.w_ne) + j);
                w_s[pc + j] = __ldg(reinterpret_cast<const uint4*>(p.w_nh) + j);
                if (p.in_norm) w_s[2 * pc + j] = __ldg(reinterpret_cast<const uint4*>(p.in_norm) + j);
            }
        }
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised, the pair's TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // stages of a tile in the ring: a GEMM tile's K blocks
    auto tile_stages = [&](const Tile& tl) -> int {
        if (p.plain) return p.K / BK;
        return (tl.kind == TILE_F ? 2 * p.h : p.h) / BK;
    };
    // this CTA's 128-row block of GEMM tile tl, and whether the chunk has it (the last pair
    // block of a chunk with an odd number of row blocks has only rank 0's)
    auto own_block = [&](const Tile& tl) -> int { return 2 * tl.m + (int)rank; };
    auto has_block = [&](const Tile& tl) -> bool {
        return own_block(tl) < (p.plain ? (p.M + BM - 1) / BM : mt_of(p, tl.c));
    };

    if (warp == 0) {
        // ---------------- producer: (rank 0) claims tiles and announces them; both stage
        // their operands
        int s = 0;
        uint32_t ph = 0;
        int q = 0;
        uint32_t qph = 0;
        int64_t issued = 0;
        bool stop = false;
        // the plain GEMM (no dependencies) takes tiles pair, pair + pairs, ...; the prefill
        // claims every tile from the counter, so a claimed tile always belongs to a running
        // pair
        int64_t t = pair;
        if (leader && !p.plain && lane == 0) t = atomicAdd(p.ctr, 1u);
        t = __shfl_sync(0xffffffffu, t, 0);
        while (!stop) {
            bool end;
            if (leader) {
                // announce the tile (or the end) to both CTAs' readers
                end = t >= p.total;
                if (!mbar_wait_cluster_bounded(&qempty[q], qph ^ 1u, abort_flag)) break;
                if (lane == 0) {
                    const int v = end ? -1 : (int)t;
                    fifo[q] = v;
                    st_cluster_u32(map_rank(&fifo[q], 1), (uint32_t)v);
                    mbar_arrive(&qfull[q]);
                    mbar_arrive_cluster(map_rank(&qfull[q], 1));
                }
                __syncwarp();
            } else {
                // the tile rank 0 announced
                if (!mbar_wait_cluster_bounded(&qfull[q], qph, abort_flag)) break;
                const int v = fifo[q];
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(map_rank(&qempty[q], 0));
                end = v < 0;
                t = v;
            }
            if (++q == kFifo) {
                q = 0;
                qph ^= 1u;
            }
            if (end) break;
            const Tile tl = decode(p, t);
            const int m = own_block(tl);
            const bool has = has_block(tl);
            int64_t tn = t + npairs;  // rank 0's next claim, issued early
            if (leader && !p.plain && lane == 0) tn = atomicAdd(p.ctr, 1u);
            const int nst = tile_stages(tl);
            {
                // operands: F reads the chunk's concat rows, V its fc output rows; each only
                // once the tiles that write them are done. A block the chunk lacks stages
                // rank 0's rows instead (its products are never stored).
                const CUtensorMap* ma;
                const CUtensorMap* mb;
                const int arow = (has ? m : m - 1) * BM;
                int brow = tl.n * BN + (int)rank * BNH;
                if (p.plain) {
                    ma = &maps.a_concat[0];
                    mb = &maps.b_fc;
                } else if (tl.kind == TILE_F) {
                    ma = &maps.a_concat[tl.c % p.lanes];
                    mb = &maps.b_fc;
                    if (has && lane == 0 &&
                        !wait_counter(counter(p, TILE_P, tl.c, m),
                                      (uint32_t)((tl.c / kCtrSlots + 1) * kPParts), abort_flag))
                        stop = true;
                } else {
                    ma = &maps.a_y[tl.c % p.lanes];
                    mb = brow < kvd ? &maps.b_wk : &maps.b_wv;
                    if (brow >= kvd) brow -= kvd;
                    if (has && lane == 0 &&
                        !wait_counter(counter(p, TILE_F, tl.c, m),
                                      (uint32_t)((tl.c / kCtrSlots + 1) * p.nf), abort_flag))
                        stop = true;
                }
                stop = __shfl_sync(0xffffffffu, (int)stop, 0) != 0;
                if (!p.plain && lane == 0) fence_proxy_async_global();  // then async reads
                for (int kb = 0; kb < nst && !stop; ++kb) {
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    if (lane == 0) {
                        uint8_t* st = stages + (size_t)s * kGStageBytes;
                        const uint32_t fb = map_rank(&full[s], 0);
                        if (leader) mbar_arrive_expect_tx(&full[s], 2 * kGStageBytes);
                        tma_load_2d_pair(st, ma, kb * BK, arow, fb);
                        tma_load_2d_pair(st + kAStageBytes, mb, kb * BK, brow, fb);
                    }
                    __syncwarp();
                    ++issued;
                    if (++s == kGStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            t = __shfl_sync(0xffffffffu, tn, 0);
        }
        // no copy left in flight: rank 0's full barriers count both CTAs' copies; rank 1's
        // stages are free once the MMAs that read them completed
        for (int64_t j = issued > kGStages ? issued - kGStages : 0; j < issued; ++j) {
            const uint32_t par = (uint32_t)((j / kGStages) & 1);
            if (!mbar_wait_bounded(leader ? &full[j % kGStages] : &empty[j % kGStages], par, nullptr))
                break;
        }
        // if rank 0 stopped early, still tell every reader that no tile follows
        if (leader && stop && mbar_wait_cluster_bounded(&qempty[q], qph ^ 1u, nullptr) && lane == 0) {
            fifo[q] = -1;
            st_cluster_u32(map_rank(&fifo[q], 1), 0xFFFFFFFFu);
            mbar_arrive(&qfull[q]);
            mbar_arrive_cluster(map_rank(&qfull[q], 1));
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: one thread of rank 0, for the pair
        constexpr uint32_t idesc = idesc_bf16(2 * BM, BN);
        int s = 0;
        uint32_t ph = 0;
        int q = 0;
        uint32_t qph = 0;
        int local = 0;
        bool stop = !leader;
        while (!stop) {
            if (!mbar_wait_bounded(&qfull[q], qph, abort_flag)) break;
            const int t = fifo[q];
            __syncwarp();
            if (lane == 0) mbar_arrive(&qempty[q]);
            if (++q == kFifo) {
                q = 0;
                qph ^= 1u;
            }
            if (t < 0) break;
            const Tile tl = decode(p, t);
            const int nst = tile_stages(tl);
            const int buf = local & 1;
            const uint32_t tph = (uint32_t)((local >> 1) & 1);
            // both CTAs' epilogues have read this accumulator's previous tile
            if (!mbar_wait_cluster_bounded(&tempty[buf], tph ^ 1u, abort_flag)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
            for (int kb = 0; kb < nst; ++kb) {
                if (!mbar_wait_bounded(&full[s], ph, abort_flag)) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a0 = smem_u32(stages + s * kGStageBytes);
                    const uint32_t b0 = a0 + kAStageBytes;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_bf16_pair(d_tmem, sdesc_k128(a0 + k * 32), sdesc_k128(b0 + k * 32), idesc,
                                       (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit_pair(&empty[s], 3);  // frees both CTAs' stage once read
                }
                __syncwarp();
                if (++s == kGStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (lane == 0) umma_commit_pair(&tfull[buf], 3);  // both accumulators ready
            __syncwarp();
            ++local;
        }
        if (leader) {
            // every MMA this thread issued has completed before TMEM is released
            if (lane == 0) umma_commit_pair(done, 1);
            __syncwarp();
            mbar_wait_bounded(done, 0u, nullptr);
        }
    } else if (warp < 6) {
        // ---------------- epilogue warps 2..5: TMEM lane quarter = warp % 4
        const int qd = warp & 3;
        const int et = threadIdx.x - 64;  // 0..127
        const int ew = et >> 5;
        int q = 0;
        uint32_t qph = 0;
        int local = 0;
        while (true) {
            if (!mbar_wait_cluster_bounded(&qfull[q], qph, abort_flag)) break;
            const int t = fifo[q];
            named_sync(1, kEpiThreads);  // every epilogue thread has read the slot
            if (et == 0) {
                if (leader) mbar_arrive(&qempty[q]);
                else mbar_arrive_cluster(map_rank(&qempty[q], 0));
            }
            if (++q == kFifo) {
                q = 0;
                qph ^= 1u;
            }
            if (t < 0) break;
            const Tile tl = decode(p, t);
            const int m = own_block(tl);
            const bool has = !p.plain && has_block(tl);  // its counters exist
            const int64_t crow0 = (int64_t)tl.c * p.chunk;  // prompt row of the chunk's row 0
            const int64_t rows_c = p.plain ? p.M : min(p.chunk, p.R - crow0);
            const int buf = local & 1;
            const uint32_t tph = (uint32_t)((local >> 1) & 1);
            ++local;
            bool ok = mbar_wait_bounded(&tfull[buf], tph, abort_flag);
            // F writes the chunk lane's fc output rows: free once the chunk that used the
            // lane before has run its k/v tiles of these rows; V reads the RoPE rows
            if (et == 0 && ok && has) {
                if (tl.kind == TILE_F && tl.c >= p.lanes) {
                    const int ca = tl.c - p.lanes;
                    ok = wait_counter(counter(p, TILE_V, ca, m),
                                      (uint32_t)((ca / kCtrSlots + 1) * p.nv), abort_flag);
                } else if (tl.kind == TILE_V) {
                    ok = wait_counter(counter(p, TILE_P, tl.c, m),
                                      (uint32_t)((tl.c / kCtrSlots + 1) * kPParts), abort_flag);
                }
            }
            named_sync(1, kEpiThreads);
            ok = ok && !*abort_flag;
            tc_fence_after();
            const int row = m * BM + qd * 32 + lane;  // row of the chunk (of A)
            const bool row_ok = ok && row < rows_c;
            const uint32_t tb = tmem_base + ((uint32_t)(qd * 32) << 16) + (uint32_t)(buf * BN);
            if (tl.kind == TILE_F) {
                uint16_t* C = p.plain ? p.C : p.y[tl.c % p.lanes];
                const int64_t ldc = p.plain ? p.N : p.h;
                for (int cc = 0; cc < BN / 32; ++cc) {
                    uint32_t v[32];
                    tmem_ld32(tb + cc * 32, v);
                    tmem_ld_wait();
                    if (row_ok) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[i] = f32x2_to_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                        uint4* dst = reinterpret_cast<uint4*>(C + (int64_t)row * ldc + tl.n * BN + cc * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
                if (!p.plain) fence_proxy_async_global();  // read by the k/v tiles' TMA
            } else {
                const int col0 = tl.n * BN;
                const bool is_v = col0 >= kvd;
                int64_t slot = -1;
                if (row_ok) {
                    slot = cache_slot(p, crow0 + row);
                    if (slot < 0) raise_flag(p.dev_err, DEVFLAG_BAD_SLOT);
                }
                uint8_t* cache = is_v ? p.v_cache : p.k_cache;
                const float scale = is_v ? p.v_scale : p.k_scale;
                const float2* cs = p.rope[tl.c % (p.lanes + 1)] + (int64_t)row * half;
                const bool kn = !is_v && p.k_norm != nullptr;
                const float kadd = p.norm_mode ? 1.f : 0.f;
                for (int h0 = 0; h0 < BN; h0 += p.hd) {
                    const int head_i = ((is_v ? col0 - kvd : col0) + h0) / p.hd;
                    uint8_t* hdst = cache + (slot * p.nkv + head_i) * (int64_t)p.hd;
                    float kinv = 1.f;
                    if (kn) {  // per-head k norm: the head's sum of squares of bf16(k) first
                        float ss = 0.f;
                        for (int j0 = 0; j0 < p.hd; j0 += 32) {
                            uint32_t a[32];
                            tmem_ld32(tb + h0 + j0, a);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 32; i += 2) {
                                float v0 = __uint_as_float(a[i]), v1 = __uint_as_float(a[i + 1]);
                                round_bf16x2(v0, v1);
                                ss = fmaf(v0, v0, ss);
                                ss = fmaf(v1, v1, ss);
                            }
                        }
                        kinv = 1.0f / sqrtf(ss / (float)p.hd + p.eps);
                    }
                    for (int j0 = 0; j0 < half; j0 += 32) {
                        uint32_t a[32], b[32];
                        tmem_ld32(tb + h0 + j0, a);
                        tmem_ld32(tb + h0 + half + j0, b);
                        tmem_ld_wait();
                        float lo[32], hi[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            lo[i] = __uint_as_float(a[i]);
                            hi[i] = __uint_as_float(b[i]);
                            round_bf16x2(lo[i], hi[i]);
                        }
                        if (kn) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                lo[i] = lo[i] * kinv * (bf16_to_f32(kn_s[j0 + i]) + kadd);
                                hi[i] = hi[i] * kinv * (bf16_to_f32(kn_s[half + j0 + i]) + kadd);
                                round_bf16x2(lo[i], hi[i]);
                            }
                        }
                        if (!is_v && row_ok) rope32(lo, hi, cs + j0);
                        if (row_ok && slot >= 0) {
                            store_codes32(hdst + j0, lo, scale);
                            store_codes32(hdst + half + j0, hi, scale);
                        }
                    }
                }
            }
            tc_fence_before();
            named_sync(1, kEpiThreads);  // the accumulator is read, every store issued
            const bool norm_y = tl.kind == TILE_F && has && p.in_norm != nullptr;
            if (et == 0) {
                if (leader) mbar_arrive(&tempty[buf]);
                else mbar_arrive_cluster(map_rank(&tempty[buf], 0));
                if (has && !*abort_flag && !norm_y)
                    counter_release_add(counter(p, tl.kind, tl.c, m), 1u);
                if (norm_y) {
                    int last = 0;
                    if (!*abort_flag) {
                        fence_acq_rel_gpu();  // release this tile's y stores
                        const uint32_t old = atomicAdd(counter(p, kArrivals, tl.c, m), 1u);
                        last = old + 1u == (uint32_t)((tl.c / kCtrSlots + 1) * p.nf);
                        fence_acq_rel_gpu();  // acquire the other tiles' stores
                    }
                    *last_flag = last;
                }
            }
            if (norm_y) {
                named_sync(1, kEpiThreads);
                if (*last_flag) {
                    // the row block's input norm, in place: a warp per row, L2 loads (the
                    // rows were written by other SMs)
                    uint16_t* Y = p.y[tl.c % p.lanes];
                    const int h = p.h, pieces = h / 8;
                    const int nrow = (int)min((int64_t)BM, rows_c - (int64_t)m * BM);
                    const uint64_t wadd = f32x2_splat(p.norm_mode ? 1.f : 0.f);
                    const uint4* wn = p.w_in_smem ? w_s + 2 * pieces : reinterpret_cast<const uint4*>(p.in_norm);
                    for (int r = ew; r < nrow; r += kEpiThreads / 32) {
                        uint4* yr = reinterpret_cast<uint4*>(Y + ((int64_t)m * BM + r) * h);
                        uint64_t ss2 = 0;
#pragma unroll 4
                        for (int j = lane; j < pieces; j += 32) ss2 = sumsq8(__ldcg(yr + j), ss2);
                        float ss = hsum_f32x2(ss2);
#pragma unroll
                        for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                        const uint64_t inv = f32x2_splat(1.0f / sqrtf(ss / (float)h + p.eps));
#pragma unroll 4
                        for (int j = lane; j < pieces; j += 32)
                            __stcg(yr + j, norm8(__ldcg(yr + j), inv, wn[j], wadd));
                    }
                    fence_proxy_async_global();  // read by the k/v tiles' TMA
                    named_sync(1, kEpiThreads);
                    if (et == 0) counter_release_add(counter(p, TILE_F, tl.c, m), (uint32_t)p.nf);
                }
            }
        }
    } else {
        // ---------------- prologue warps 6..7: claim prologue tiles from their own counter
        // (every SM's pair takes the next one when it is free) and run them
        const int pt = threadIdx.x - 192;  // 0..63
        const int pw = pt >> 5;
        volatile int* pclaim = last_flag + 1;
        while (!p.plain) {
            if (pt == 0) *pclaim = (int)atomicAdd(p.ctr + 1, 1u);
            named_sync(2, kProThreads);
            const int64_t t = *pclaim;
            named_sync(2, kProThreads);  // everyone has read it before the next claim
            if (t >= p.p_total || *abort_flag) break;
            const Tile tl = decode_p(p, t);
            const int64_t crow0 = (int64_t)tl.c * p.chunk;  // prompt row of the chunk's row 0
            {
                // ---- rows m*128 + n*kPRows .. : the lanes' buffers are free once the chunks
                // that used them before are done with them
                const int lane_c = tl.c % p.lanes, slot_r = tl.c % (p.lanes + 1);
                bool ok = true;
                if (pt == 0) {
                    const int ca = tl.c - p.lanes, cr = tl.c - p.lanes - 1;
                    if (ca >= 0)
                        ok = wait_counter(counter(p, TILE_F, ca, tl.m),
                                          (uint32_t)((ca / kCtrSlots + 1) * p.nf), abort_flag);
                    if (ok && cr >= 0)
                        ok = wait_counter(counter(p, TILE_V, cr, tl.m),
                                          (uint32_t)((cr / kCtrSlots + 1) * p.nv), abort_flag);
                }
                named_sync(2, kProThreads);
                const int rows = p_tile_rows(p, tl);
                const int prow0 = tl.m * BM + tl.n * kPRows;  // the tile's first row of the chunk
                const int h = p.h, pieces = h / 8;  // 16-byte pieces of a row
                const uint64_t wadd = f32x2_splat(p.norm_mode ? 1.f : 0.f);
                // generic loads: shared memory when staged, else global
                const uint4* wne = p.w_in_smem ? w_s : reinterpret_cast<const uint4*>(p.w_ne);
                const uint4* wnh = p.w_in_smem ? w_s + pieces : reinterpret_cast<const uint4*>(p.w_nh);
                // warp pw takes rows pw, pw + 2, ...: each half of the concat row (embedding
                // row, hidden row) is loaded straight from global memory into registers (up
                // to 5,120 wide in one pass, else in two), reduced with warp shuffles and
                // written normalized
                for (int r = pw; r < rows; r += kProThreads / 32) {
                    const int64_t prow = crow0 + prow0 + r;  // prompt row
                    int64_t tok = p.tokens[prow];
                    if (tok < 0 || tok >= p.vocab) {
                        if (lane == 0) raise_flag(p.dev_err, DEVFLAG_BAD_TOKEN);
                        tok = -1;
                    }
                    uint4* crow = reinterpret_cast<uint4*>(p.concat[lane_c] + ((int64_t)prow0 + r) * 2 * h);
#pragma unroll 1
                    for (int side = 0; side < 2; ++side) {  // embedding half, then hidden half
                        const uint4* src = reinterpret_cast<const uint4*>(
                            side == 0 ? (tok >= 0 ? p.embed + tok * h : nullptr) : p.hidden + prow * h);
                        norm_row(src, side == 0 ? wne : wnh, crow + side * pieces, pieces, lane, p.eps, wadd);
                    }
                }
                // RoPE table of the rows: the angle pos * base^(-2j / hd) in turns, reduced to
                // [-1/2, 1/2] in double (exact to ~1e-12 turns), then cos and sin of the
                // remainder in fp32 (sincospif: no further range reduction)
                float2* cs = p.rope[slot_r] + (int64_t)prow0 * half;
                for (int k = pt; k < rows * half; k += kProThreads) {
                    const int r = k / half, j = k - r * half;
                    const double turns = (double)p.rope_pos[crow0 + prow0 + r] * inv_freq[j];
                    const float f = (float)(turns - rint(turns));
                    float sn, cn;
                    sincospif(2.0f * f, &sn, &cn);  // sin and cos of pi x: x in half turns
                    cs[k] = make_float2(cn, sn);
                }
                fence_proxy_async_global();  // the concat rows are read by TMA
                named_sync(2, kProThreads);
                if (pt == 0 && !*abort_flag) counter_release_add(counter(p, TILE_P, tl.c, tl.m), 1u);
            }
        }
    }
    tc_fence_before();
    cluster_sync();  // neither CTA leaves while an MMA, a copy or an arrival may reach it
    if (*abort_flag && threadIdx.x == 0) raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

// Stage check: bf16 k' (already rotated) and v rows -> E4M3 codes in the paged cache,
// through the same encode and slot code the k/v epilogue uses. One warp per row.
__global__ void kv_write_kernel(const uint16_t* __restrict__ k_rot, const uint16_t* __restrict__ v,
                                int64_t R, const PrefillParams p) {
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= R) return;
    const int64_t slot = cache_slot(p, r);
    if (slot < 0) {
        if (lane == 0) raise_flag(p.dev_err, DEVFLAG_BAD_SLOT);
        return;
    }
    const int kvd = p.nkv * p.hd;
    // lane handles 32-element pieces: (tensor, head, piece) flattened
    const int pieces = kvd / 32;
    for (int i = lane; i < 2 * pieces; i += 32) {
        const bool is_v = i >= pieces;
        const int pc = is_v ? i - pieces : i;
        const uint16_t* src = (is_v ? v : k_rot) + r * kvd + pc * 32;
        float vals[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) vals[j] = bf16_to_f32(src[j]);
        const int head = pc * 32 / p.hd, d0 = pc * 32 % p.hd;
        uint8_t* dst = (is_v ? p.v_cache : p.k_cache) + (slot * p.nkv + head) * (int64_t)p.hd + d0;
        store_codes32(dst, vals, is_v ? p.v_scale : p.k_scale);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// bf16 [rows, k] K-major operand, boxes of 64 x box_rows with the 128-byte swizzle.
cudaError_t make_operand_map(CUtensorMap* m, const void* base, int64_t rows, int64_t k,
                             int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(k * 2)};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int weight_smem_bytes(const PrefillParams& p) {
    return p.plain ? 0 : (p.in_norm ? 3 : 2) * 2 * p.h;
}

// CTA pairs that can be resident at once with `smem` bytes each (every SM pair of a TPC
// whose two SMs are both available), per device and size.
cudaError_t resident_pairs(int dev, int smem, int* out) {
    static std::mutex mu;
    static int cached[64][2] = {};  // [device] {smem, pairs}
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && cached[dev][0] == smem && cached[dev][1] > 0) {
        *out = cached[dev][1];
        return cudaSuccess;
    }
    int sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(sms & ~1), 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&n, prefill_kernel, &cfg)) != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64) {
        cached[dev][0] = smem;
        cached[dev][1] = n;
    }
    *out = n;
    return cudaSuccess;
}

cudaError_t launch(PrefillParams p, const Maps& maps, cudaStream_t s) {
    if (p.total < 1) return cudaSuccess;
    const int wb = weight_smem_bytes(p);
    p.w_in_smem = wb > 0 && kGemmSmem + wb <= kSmemMax;
    const int smem = kGemmSmem + (p.w_in_smem ? wb : 0);
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return e;
    int dev = 0, pairs = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = resident_pairs(dev, smem, &pairs)) != cudaSuccess) return e;
    // every pair is resident at once: a tile claimed from the counter always belongs to a
    // running pair, so every wait on another tile ends
    int64_t grid = pairs;
    if (grid > p.total) grid = p.total;
    prefill_kernel<<<(unsigned)(2 * grid), kGemmThreads, smem, s>>>(p, maps);
    return cudaGetLastError();
}

// Workspace layout: a counter header, then `lanes` x (concat rows, fc output rows), then
// lanes + 1 RoPE tables.
constexpr size_t kCtrHeader = 256;  // tile counter (and room), before the done counters
size_t up1k(size_t b) { return (b + 1023) & ~(size_t)1023; }
size_t header_bytes(int64_t chunk_rows) {
    const size_t mt = (size_t)((chunk_rows + BM - 1) / BM);
    return up1k(kCtrHeader + 4 * kCtrSlots * mt * sizeof(uint32_t));
}
size_t concat_bytes(int64_t c, int32_t h) { return up1k((size_t)c * 2 * h * 2); }
size_t y_bytes(int64_t c, int32_t h) { return up1k((size_t)c * h * 2); }
size_t rope_bytes(int64_t c, int32_t hd) { return up1k((size_t)c * (hd / 2) * sizeof(float2)); }

}  // namespace

size_t prefill_ws_bytes_lanes(int64_t chunk_rows, int32_t h, int32_t hd, int lanes) {
    return header_bytes(chunk_rows) +
           (size_t)lanes * (concat_bytes(chunk_rows, h) + y_bytes(chunk_rows, h)) +
           (size_t)(lanes + 1) * rope_bytes(chunk_rows, hd);
}

size_t prefill_lane_bytes(int64_t chunk_rows, int32_t h, int32_t nkv, int32_t hd) {
    (void)nkv;
    return prefill_ws_bytes_lanes(chunk_rows, h, hd, 1);  // the minimum: one lane
}

size_t prefill_ws_bytes(int64_t chunk_rows, int32_t h, int32_t nkv, int32_t hd) {
    (void)nkv;
    // twice the one-lane minimum (which covers the two-lane layout), so that half of the
    // full size is always a valid one-lane workspace
    return 2 * prefill_ws_bytes_lanes(chunk_rows, h, hd, 1);
}

// The widest hidden size the prefill takes (the fc GEMM's K is twice it).
int prefill_max_hidden() { return 12288; }

cudaError_t prefill_launch(const PrefillArgs& a, cudaStream_t s) {
    const int kvd = a.nkv * a.hd;
    PrefillParams p{};
    p.embed = a.embed;
    p.vocab = a.vocab;
    p.tokens = a.tokens;
    p.hidden = a.hidden;
    p.R = a.R;
    p.h = a.h;
    p.w_ne = a.w_norm_embed;
    p.w_nh = a.w_norm_hidden;
    p.eps = a.eps;
    p.norm_mode = a.norm_mode;
    p.k_norm = a.k_norm;
    p.in_norm = a.in_norm;
    p.nkv = a.nkv;
    p.hd = a.hd;
    p.rope_base = a.rope_base;
    p.rope_pos = a.rope_pos;
    p.cache_start = a.cache_start;
    p.block_table = a.block_table;
    p.n_table = a.n_table;
    p.block_size = a.block_size;
    p.num_blocks = a.num_blocks;
    p.k_cache = a.k_cache;
    p.v_cache = a.v_cache;
    p.k_scale = a.k_scale;
    p.v_scale = a.v_scale;
    p.dev_err = a.dev_err;
    p.chunk = a.chunk_rows;
    p.n_chunks = (int)((a.R + a.chunk_rows - 1) / a.chunk_rows);
    p.mt_full = (int)((a.chunk_rows + BM - 1) / BM);
    const int64_t last_rows = a.R - (int64_t)(p.n_chunks - 1) * a.chunk_rows;
    p.mt_last = (int)((last_rows + BM - 1) / BM);
    p.mp_full = (p.mt_full + 1) / 2;
    p.mp_last = (p.mt_last + 1) / 2;
    p.nf = a.h / BN;
    p.nv = 2 * kvd / BN;
    p.lanes = (a.R > a.chunk_rows && a.ws_bytes >= prefill_ws_bytes_lanes(a.chunk_rows, a.h, a.hd, 2))
                  ? 2 : 1;
    p.total = 0;
    p.p_total = 0;
    for (int c = 0; c < p.n_chunks; ++c) {
        const int mt = c == p.n_chunks - 1 ? p.mt_last : p.mt_full;
        const int mp = c == p.n_chunks - 1 ? p.mp_last : p.mp_full;
        p.total += (int64_t)mp * (p.nf + p.nv);
        p.p_total += (int64_t)mt * kPParts;
    }
    if (a.hd / 2 > 128) return cudaErrorInvalidValue;
    // workspace carving
    uint8_t* w = static_cast<uint8_t*>(a.ws);
    p.ctr = reinterpret_cast<uint32_t*>(w);
    size_t off = header_bytes(a.chunk_rows);
    for (int l = 0; l < p.lanes; ++l) {
        p.concat[l] = reinterpret_cast<uint16_t*>(w + off);
        off += concat_bytes(a.chunk_rows, a.h);
        p.y[l] = reinterpret_cast<uint16_t*>(w + off);
        off += y_bytes(a.chunk_rows, a.h);
    }
    for (int l = 0; l < p.lanes + 1; ++l) {
        p.rope[l] = reinterpret_cast<float2*>(w + off);
        off += rope_bytes(a.chunk_rows, a.hd);
    }
    Maps maps{};
    cudaError_t e;
    for (int l = 0; l < p.lanes; ++l) {
        if ((e = make_operand_map(&maps.a_concat[l], p.concat[l], a.chunk_rows, 2 * (int64_t)a.h, BM)) !=
            cudaSuccess)
            return e;
        if ((e = make_operand_map(&maps.a_y[l], p.y[l], a.chunk_rows, a.h, BM)) != cudaSuccess) return e;
    }
    if ((e = make_operand_map(&maps.b_fc, a.fc, a.h, 2 * (int64_t)a.h, BNH)) != cudaSuccess) return e;
    if ((e = make_operand_map(&maps.b_wk, a.wk, kvd, a.h, BNH)) != cudaSuccess) return e;
    if ((e = make_operand_map(&maps.b_wv, a.wv, kvd, a.h, BNH)) != cudaSuccess) return e;
    // the counters start at zero on every call (a memset node in the caller's stream)
    if ((e = cudaMemsetAsync(p.ctr, 0, header_bytes(a.chunk_rows), s)) != cudaSuccess) return e;
    return launch(p, maps, s);
}

cudaError_t gemm_bf16_launch(const uint16_t* A, const uint16_t* B, uint16_t* C, int M, int N,
                             int K, int32_t* dev_err, cudaStream_t s) {
    PrefillParams p{};
    p.plain = 1;
    p.M = M;
    p.N = N;
    p.K = K;
    p.C = C;
    p.R = M;
    p.chunk = M;
    p.n_chunks = 1;
    p.lanes = 1;
    p.nf = N / BN;
    p.total = (int64_t)((M + 2 * BM - 1) / (2 * BM)) * (N / BN);
    p.dev_err = dev_err;
    Maps maps{};
    cudaError_t e;
    if ((e = make_operand_map(&maps.a_concat[0], A, M, K, BM)) != cudaSuccess) return e;
    if ((e = make_operand_map(&maps.b_fc, B, N, K, BNH)) != cudaSuccess) return e;
    return launch(p, maps, s);
}

cudaError_t kv_write_launch(const uint16_t* k_rot, const uint16_t* v, int64_t R, int nkv, int hd,
                            int64_t cache_start, const int32_t* block_table, int64_t n_table,
                            int block_size, int64_t num_blocks, uint8_t* k_cache, uint8_t* v_cache,
                            float k_scale, float v_scale, int32_t* dev_err, cudaStream_t s) {
    PrefillParams p{};
    p.nkv = nkv;
    p.hd = hd;
    p.cache_start = cache_start;
    p.block_table = block_table;
    p.n_table = n_table;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.dev_err = dev_err;
    const int64_t blocks = (R + 7) / 8;
    kv_write_kernel<<<(unsigned)blocks, 256, 0, s>>>(k_rot, v, R, p);
    return cudaGetLastError();
}

int gemm_tile_n() { return BN; }
int gemm_tile_k() { return BK; }

}  // namespace mtp
