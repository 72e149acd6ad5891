// Drafter-context prefill: the K/V cache rows of the MTP drafter for a whole prompt.
//
// What it computes (spark_model/layers/mtp_head.rs, the drafter-prefill docs and
// MtpPrefillScratch: the drafter's K/V for prompt row i depend only on
// (embed(token_{i+1}), target_hidden_i), so no attention runs; block size 16 and the
// FP8 cache in metrale_model_layers/layers/mtp_head/new.rs; the slot rule of
// metrale_model_arch/deepseek_v4_mtp.rs forward_one step 4). Per prompt row r:
//   c  = [bf16(rms(embed[tok_r]) w_e) || bf16(rms(hidden_r) w_h)]          (prologue)
//   y  = bf16(fc . c)                                           (GEMM 1, tcgen05)
//   k  = bf16(Wk . y), v = bf16(Wv . y)                         (GEMM 2, tcgen05)
//   k' = bf16(RoPE_neox(k, pos_r)) per head, codes = e4m3(k' / k_scale), e4m3(v / v_scale)
//   cache row p = cache_start + r, slot = block_table[p / bs] * bs + p % bs,
//   element (slot, head, d) of a [num_blocks, bs, nkv, hd] cache.        (GEMM 2 epilogue)
//
// Design (B200): rows are processed in chunks (the reference's PREFILL_CHUNK). The two
// projections are the only dense contractions, so they run on the 5th-generation tensor
// cores: one persistent kernel per GEMM, 128 x 256 output tiles, a 4-stage TMA ring
// (128-byte swizzle, K-major A and B), tcgen05.mma issued by one thread into a
// double-buffered 512-column TMEM accumulator, and four epilogue warps that read it back
// with tcgen05.ld while the next tile accumulates. GEMM 2's epilogue applies RoPE from a
// per-row cos/sin table (computed in double by the prologue), encodes E4M3 and scatters
// each row's 32-byte pieces straight into the paged cache: K/V never round-trip through
// HBM in bf16. All waits are bounded (abort flag + MTP_DEVFLAG_TIMEOUT).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace mtp {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kGStages = 4;
constexpr int kAStageBytes = BM * BK * 2;  // 16 KB
constexpr int kBStageBytes = BN * BK * 2;  // 32 KB
constexpr int kGStageBytes = kAStageBytes + kBStageBytes;
constexpr int kGemmThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kTmemCols = 2 * BN;  // two fp32 accumulators of 128 lanes x 256 columns
constexpr int kGemmSmem = kGStages * kGStageBytes + 1024 /* barriers */ + 1024 /* align */;
constexpr int kPrologueThreads = 256;

struct GemmParams {
    int M, N, K;        // rows of A (valid), columns of the output, reduction length
    int m_tiles, n_tiles;
    // epilogue 0: bf16 output
    uint16_t* C;
    int64_t ldc;
    // epilogue 1: k/v -> RoPE (k) -> E4M3 -> paged cache
    int nkv, hd;
    const float2* rope_cs;  // [M][hd/2] (cos, sin)
    int64_t row0;           // prompt row of this chunk's first row
    int64_t cache_start;
    const int32_t* block_table;
    int64_t n_table;
    int block_size;
    int64_t num_blocks;
    uint8_t* k_cache;
    uint8_t* v_cache;
    float k_scale, v_scale;
    int32_t* dev_err;
};

// Cache slot of prompt row (row0 + r), or -1 when its block is missing / out of range.
__device__ __forceinline__ int64_t cache_slot(const GemmParams& p, int64_t prompt_row) {
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

__device__ __forceinline__ float round_bf16(float f) { return bf16_to_f32(f32_to_bf16(f)); }

// NeoX rotation of one head's pair block: lo = k[j], hi = k[j + hd/2] for 32 j's.
__device__ __forceinline__ void rope32(float (&lo)[32], float (&hi)[32], const float2* cs) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float2 t = cs[j];
        const float a = lo[j], b = hi[j];
        lo[j] = round_bf16(fmaf(a, t.x, -b * t.y));
        hi[j] = round_bf16(fmaf(b, t.x, a * t.y));
    }
}

// ------------------------------------------------------------------------------ prologue
// One CTA per chunk row: the combiner's concat row c[r] = [ne || nh] and the RoPE table.
__global__ void __launch_bounds__(kPrologueThreads) prefill_prologue_kernel(
    const uint16_t* __restrict__ embed, int64_t vocab, const int32_t* __restrict__ tokens,
    const uint16_t* __restrict__ hidden, int h, const uint16_t* __restrict__ w_ne,
    const uint16_t* __restrict__ w_nh, float eps, const int32_t* __restrict__ rope_pos,
    double rope_base, int hd, int64_t row0, uint16_t* __restrict__ c_out,
    float2* __restrict__ cs_out, int32_t* dev_err) {
    __shared__ float red[2][kPrologueThreads / 32];
    const int r = blockIdx.x, tid = threadIdx.x;
    const int64_t pr = row0 + r;
    const int64_t tok = tokens[pr];
    const bool bad = tok < 0 || tok >= vocab;
    if (bad && tid == 0) raise_flag(dev_err, DEVFLAG_BAD_TOKEN);
    const uint16_t* e = bad ? nullptr : embed + tok * h;
    const uint16_t* x = hidden + pr * h;
    float se = 0.f, sx = 0.f;
    for (int j = tid; j < h; j += kPrologueThreads) {
        const float ev = e ? bf16_to_f32(e[j]) : 0.f;
        const float xv = bf16_to_f32(x[j]);
        se += ev * ev;
        sx += xv * xv;
    }
    for (int o = 16; o; o >>= 1) {
        se += __shfl_xor_sync(0xffffffffu, se, o);
        sx += __shfl_xor_sync(0xffffffffu, sx, o);
    }
    if ((tid & 31) == 0) {
        red[0][tid >> 5] = se;
        red[1][tid >> 5] = sx;
    }
    __syncthreads();
    se = 0.f;
    sx = 0.f;
#pragma unroll
    for (int w = 0; w < kPrologueThreads / 32; ++w) {
        se += red[0][w];
        sx += red[1][w];
    }
    const float inv_e = 1.0f / sqrtf(se / (float)h + eps);
    const float inv_x = 1.0f / sqrtf(sx / (float)h + eps);
    uint16_t* row = c_out + (int64_t)r * 2 * h;
    for (int j = tid; j < h; j += kPrologueThreads) {
        const float ev = e ? bf16_to_f32(e[j]) : 0.f;
        row[j] = f32_to_bf16(ev * inv_e * bf16_to_f32(w_ne[j]));
        row[h + j] = f32_to_bf16(bf16_to_f32(x[j]) * inv_x * bf16_to_f32(w_nh[j]));
    }
    const int half = hd / 2;
    for (int j = tid; j < half; j += kPrologueThreads) {
        const double inv_freq = pow(rope_base, -2.0 * (double)j / (double)hd);
        const double th = (double)rope_pos[pr] * inv_freq;
        double s, c;
        sincos(th, &s, &c);
        cs_out[(int64_t)r * half + j] = make_float2((float)c, (float)s);
    }
}

// ------------------------------------------------------------------------------ GEMM
// out[M, N] = A[M, K] . B[N, K]^T with A, B bf16 K-major. EPI 0 stores bf16; EPI 1 is
// the k/v epilogue (B rows [0, nkv*hd) from map_b0 = Wk, the rest from map_b1 = Wv).
template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap map_a,
                const __grid_constant__ CUtensorMap map_b0,
                const __grid_constant__ CUtensorMap map_b1) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* stages = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStageBytes);
    uint64_t* empty = full + kGStages;
    uint64_t* tfull = empty + kGStages;   // [2]
    uint64_t* tempty = tfull + 2;         // [2]
    uint64_t* done = tempty + 2;          // MMA drain at exit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = p.m_tiles * p.n_tiles;
    const int kb_count = p.K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
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

    if (warp == 0) {
        // ---------------- TMA producer
        int s = 0;
        uint32_t ph = 0;
        bool stop = false;
        int64_t issued = 0;
        for (int t = blockIdx.x; t < total && !stop; t += gridDim.x) {
            const int m = t % p.m_tiles, n = t / p.m_tiles;
            const int brow = n * BN;
            const bool second = EPI == 1 && brow >= p.nkv * p.hd;
            for (int kb = 0; kb < kb_count; ++kb) {
                if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag)) {
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    uint8_t* st = stages + s * kGStageBytes;
                    mbar_arrive_expect_tx(&full[s], kGStageBytes);
                    tma_load_2d_g(st, &map_a, kb * BK, m * BM, &full[s]);
                    tma_load_2d_g(st + kAStageBytes, second ? &map_b1 : &map_b0, kb * BK,
                                  second ? brow - p.nkv * p.hd : brow, &full[s]);
                }
                __syncwarp();
                ++issued;
                if (++s == kGStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        for (int64_t j = issued > kGStages ? issued - kGStages : 0; j < issued; ++j)
            if (!mbar_wait_bounded(&full[j % kGStages], (uint32_t)((j / kGStages) & 1), nullptr)) break;
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread)
        constexpr uint32_t idesc = idesc_bf16(BM, BN);
        int s = 0;
        uint32_t ph = 0;
        int local = 0;
        bool stop = false;
        for (int t = blockIdx.x; t < total && !stop; t += gridDim.x, ++local) {
            const int buf = local & 1;
            const uint32_t tph = (uint32_t)((local >> 1) & 1);
            if (!mbar_wait_bounded(&tempty[buf], tph ^ 1u, abort_flag)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
            for (int kb = 0; kb < kb_count; ++kb) {
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
                        umma_bf16(d_tmem, sdesc_k128(a0 + k * 32), sdesc_k128(b0 + k * 32), idesc,
                                  (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);  // frees the stage once these MMAs have read it
                }
                __syncwarp();
                if (++s == kGStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (lane == 0) umma_commit(&tfull[buf]);  // accumulator ready for the epilogue
            __syncwarp();
        }
        // every MMA this thread issued has completed before TMEM is released
        if (lane == 0) umma_commit(done);
        __syncwarp();
        mbar_wait_bounded(done, 0u, nullptr);
    } else {
        // ---------------- epilogue warps 2..5: TMEM lane quarter = warp % 4
        const int q = warp & 3;
        const int r_in_tile = q * 32 + lane;
        int local = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++local) {
            const int m = t % p.m_tiles, n = t / p.m_tiles;
            const int buf = local & 1;
            const uint32_t tph = (uint32_t)((local >> 1) & 1);
            const bool ok = mbar_wait_bounded(&tfull[buf], tph, abort_flag);
            tc_fence_after();
            const int row = m * BM + r_in_tile;  // row of A / of this chunk
            const bool row_ok = ok && row < p.M;
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);
            if (EPI == 0) {
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tb + c * 32, v);
                    tmem_ld_wait();
                    if (row_ok) {
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[i] = (uint32_t)f32_to_bf16(__uint_as_float(v[2 * i])) |
                                    ((uint32_t)f32_to_bf16(__uint_as_float(v[2 * i + 1])) << 16);
                        uint4* dst = reinterpret_cast<uint4*>(p.C + (int64_t)row * p.ldc + n * BN + c * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            } else {
                const int kvd = p.nkv * p.hd;
                const int col0 = n * BN;
                const bool is_v = col0 >= kvd;
                const int half = p.hd / 2;
                int64_t slot = -1;
                if (row_ok) {
                    slot = cache_slot(p, p.row0 + row);
                    if (slot < 0) raise_flag(p.dev_err, DEVFLAG_BAD_SLOT);
                }
                uint8_t* cache = is_v ? p.v_cache : p.k_cache;
                const float scale = is_v ? p.v_scale : p.k_scale;
                for (int h0 = 0; h0 < BN; h0 += p.hd) {
                    const int head = ((is_v ? col0 - kvd : col0) + h0) / p.hd;
                    uint8_t* hdst = cache + (slot * p.nkv + head) * (int64_t)p.hd;
                    for (int j0 = 0; j0 < half; j0 += 32) {
                        uint32_t a[32], b[32];
                        tmem_ld32(tb + h0 + j0, a);
                        tmem_ld32(tb + h0 + half + j0, b);
                        tmem_ld_wait();
                        float lo[32], hi[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            lo[i] = round_bf16(__uint_as_float(a[i]));
                            hi[i] = round_bf16(__uint_as_float(b[i]));
                        }
                        if (!is_v && row_ok) rope32(lo, hi, p.rope_cs + (int64_t)row * half + j0);
                        if (row_ok && slot >= 0) {
                            store_codes32(hdst + j0, lo, scale);
                            store_codes32(hdst + half + j0, hi, scale);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
        }
    }
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Stage check: bf16 k' (already rotated) and v rows -> E4M3 codes in the paged cache,
// through the same encode and slot code the GEMM epilogue uses. One warp per row.
__global__ void kv_write_kernel(const uint16_t* __restrict__ k_rot, const uint16_t* __restrict__ v,
                                int64_t R, const GemmParams p) {
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

int sm_count_now() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int EPI>
cudaError_t launch_gemm(const GemmParams& p0, const CUtensorMap& ma, const CUtensorMap& mb0,
                        const CUtensorMap& mb1, cudaStream_t s) {
    GemmParams p = p0;
    p.m_tiles = (p.M + BM - 1) / BM;
    p.n_tiles = p.N / BN;
    const int total = p.m_tiles * p.n_tiles;
    if (total < 1) return cudaSuccess;
    auto kern = gemm_kernel<EPI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
    if (e != cudaSuccess) return e;
    int grid = sm_count_now();
    if (grid > total) grid = total;
    kern<<<grid, kGemmThreads, kGemmSmem, s>>>(p, ma, mb0, mb1);
    return cudaGetLastError();
}

}  // namespace

size_t prefill_lane_bytes(int64_t chunk_rows, int32_t h, int32_t nkv, int32_t hd) {
    (void)nkv;
    auto up = [](size_t b) { return (b + 1023) & ~(size_t)1023; };
    return up((size_t)chunk_rows * 2 * h * 2) + up((size_t)chunk_rows * h * 2) +
           up((size_t)chunk_rows * (hd / 2) * sizeof(float2));
}

size_t prefill_ws_bytes(int64_t chunk_rows, int32_t h, int32_t nkv, int32_t hd) {
    return 2 * prefill_lane_bytes(chunk_rows, h, nkv, hd);
}

namespace {

// Two streams per device on which alternate chunks run: a chunk's fc GEMM (320 tiles of
// 128 x 256 at 2,048 rows x hidden 5,120) ends in a partial wave on 148 SMs, and the k/v
// GEMM and the prologue leave SMs idle too; chunks are independent, so the next chunk's
// kernels fill those SMs. Created on first use and kept for the life of the process.
struct ChunkLanes {
    cudaStream_t s[2] = {nullptr, nullptr};
    cudaEvent_t fork = nullptr, join[2] = {nullptr, nullptr};
};
constexpr int kMaxLaneDevices = 64;
ChunkLanes g_lanes[kMaxLaneDevices];
std::mutex g_lane_mutex;  // held while a call forks and joins (events are shared)

cudaError_t lanes_for_current_device(ChunkLanes** out) {
    int dev = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxLaneDevices) return cudaErrorInvalidDevice;
    ChunkLanes& L = g_lanes[dev];
    if (!L.fork) {
        for (int i = 0; i < 2; ++i) {
            if ((e = cudaStreamCreateWithFlags(&L.s[i], cudaStreamNonBlocking)) != cudaSuccess) return e;
            if ((e = cudaEventCreateWithFlags(&L.join[i], cudaEventDisableTiming)) != cudaSuccess)
                return e;
        }
        if ((e = cudaEventCreateWithFlags(&L.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    *out = &L;
    return cudaSuccess;
}

// One chunk: prologue (gather, norms, concat, RoPE table), fc GEMM, k/v GEMM with the
// RoPE + E4M3 + paged-write epilogue, using one lane of the workspace.
cudaError_t prefill_chunk(const PrefillArgs& a, int64_t r0, int rows, uint8_t* lane,
                          const CUtensorMap& m_fc, const CUtensorMap& m_wk, const CUtensorMap& m_wv,
                          cudaStream_t s) {
    auto up = [](size_t b) { return (b + 1023) & ~(size_t)1023; };
    uint16_t* cbuf = reinterpret_cast<uint16_t*>(lane);
    uint16_t* ybuf = reinterpret_cast<uint16_t*>(lane + up((size_t)a.chunk_rows * 2 * a.h * 2));
    float2* csbuf = reinterpret_cast<float2*>(reinterpret_cast<uint8_t*>(ybuf) +
                                              up((size_t)a.chunk_rows * a.h * 2));
    const int kvd = a.nkv * a.hd;
    cudaError_t e;
    prefill_prologue_kernel<<<rows, kPrologueThreads, 0, s>>>(
        a.embed, a.vocab, a.tokens, a.hidden, a.h, a.w_norm_embed, a.w_norm_hidden, a.eps,
        a.rope_pos, a.rope_base, a.hd, r0, cbuf, csbuf, a.dev_err);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    CUtensorMap m_c, m_y;
    if ((e = make_operand_map(&m_c, cbuf, rows, 2 * (int64_t)a.h, BM)) != cudaSuccess) return e;
    if ((e = make_operand_map(&m_y, ybuf, rows, a.h, BM)) != cudaSuccess) return e;
    GemmParams g1{};
    g1.M = rows;
    g1.N = a.h;
    g1.K = 2 * a.h;
    g1.C = ybuf;
    g1.ldc = a.h;
    g1.dev_err = a.dev_err;
    if ((e = launch_gemm<0>(g1, m_c, m_fc, m_fc, s)) != cudaSuccess) return e;
    GemmParams g2{};
    g2.M = rows;
    g2.N = 2 * kvd;
    g2.K = a.h;
    g2.nkv = a.nkv;
    g2.hd = a.hd;
    g2.rope_cs = csbuf;
    g2.row0 = r0;
    g2.cache_start = a.cache_start;
    g2.block_table = a.block_table;
    g2.n_table = a.n_table;
    g2.block_size = a.block_size;
    g2.num_blocks = a.num_blocks;
    g2.k_cache = a.k_cache;
    g2.v_cache = a.v_cache;
    g2.k_scale = a.k_scale;
    g2.v_scale = a.v_scale;
    g2.dev_err = a.dev_err;
    return launch_gemm<1>(g2, m_y, m_wk, m_wv, s);
}

}  // namespace

cudaError_t prefill_launch(const PrefillArgs& a, cudaStream_t s) {
    const int kvd = a.nkv * a.hd;
    CUtensorMap m_fc, m_wk, m_wv;
    cudaError_t e;
    if ((e = make_operand_map(&m_fc, a.fc, a.h, 2 * (int64_t)a.h, BN)) != cudaSuccess) return e;
    if ((e = make_operand_map(&m_wk, a.wk, kvd, a.h, BN)) != cudaSuccess) return e;
    if ((e = make_operand_map(&m_wv, a.wv, kvd, a.h, BN)) != cudaSuccess) return e;
    const size_t lane_bytes = prefill_lane_bytes(a.chunk_rows, a.h, a.nkv, a.hd);
    uint8_t* ws = static_cast<uint8_t*>(a.ws);
    const bool two = a.R > a.chunk_rows && a.ws_bytes >= 2 * lane_bytes;
    if (!two) {  // one lane: the chunks in order on the caller's stream
        for (int64_t r0 = 0; r0 < a.R; r0 += a.chunk_rows) {
            const int rows = (int)((a.R - r0) < a.chunk_rows ? (a.R - r0) : a.chunk_rows);
            if ((e = prefill_chunk(a, r0, rows, ws, m_fc, m_wk, m_wv, s)) != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    // two lanes: chunk i runs on lane stream i % 2 with workspace lane i % 2, forked from
    // and joined back into the caller's stream (the same pattern works under capture)
    std::lock_guard<std::mutex> lock(g_lane_mutex);
    ChunkLanes* L = nullptr;
    if ((e = lanes_for_current_device(&L)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(L->fork, s)) != cudaSuccess) return e;
    for (int i = 0; i < 2; ++i)
        if ((e = cudaStreamWaitEvent(L->s[i], L->fork, 0)) != cudaSuccess) return e;
    cudaError_t err = cudaSuccess;
    int64_t i = 0;
    for (int64_t r0 = 0; r0 < a.R && err == cudaSuccess; r0 += a.chunk_rows, ++i) {
        const int rows = (int)((a.R - r0) < a.chunk_rows ? (a.R - r0) : a.chunk_rows);
        err = prefill_chunk(a, r0, rows, ws + (size_t)(i & 1) * lane_bytes, m_fc, m_wk, m_wv,
                            L->s[i & 1]);
    }
    // join even after a failed launch, so the caller's stream stays ordered after both lanes
    for (int j = 0; j < 2; ++j) {
        if ((e = cudaEventRecord(L->join[j], L->s[j])) != cudaSuccess) return e;
        if ((e = cudaStreamWaitEvent(s, L->join[j], 0)) != cudaSuccess) return e;
    }
    return err;
}

cudaError_t gemm_bf16_launch(const uint16_t* A, const uint16_t* B, uint16_t* C, int M, int N,
                             int K, int32_t* dev_err, cudaStream_t s) {
    CUtensorMap ma, mb;
    cudaError_t e;
    if ((e = make_operand_map(&ma, A, M, K, BM)) != cudaSuccess) return e;
    if ((e = make_operand_map(&mb, B, N, K, BN)) != cudaSuccess) return e;
    GemmParams g{};
    g.M = M;
    g.N = N;
    g.K = K;
    g.C = C;
    g.ldc = N;
    g.dev_err = dev_err;
    return launch_gemm<0>(g, ma, mb, mb, s);
}

cudaError_t kv_write_launch(const uint16_t* k_rot, const uint16_t* v, int64_t R, int nkv, int hd,
                            int64_t cache_start, const int32_t* block_table, int64_t n_table,
                            int block_size, int64_t num_blocks, uint8_t* k_cache, uint8_t* v_cache,
                            float k_scale, float v_scale, int32_t* dev_err, cudaStream_t s) {
    GemmParams p{};
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
