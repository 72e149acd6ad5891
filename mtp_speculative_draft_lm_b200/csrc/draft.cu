// One whole draft step for a small, L2-resident draft head in a single launch: the
// embed+hidden combiner (embedding gather, two RMSNorms, concat, fc projection) and the
// lm_head sweep fused with the (masked) argmax.
//
// What it computes is mtp_combine followed by mtp_lm_head_argmax (metrale_model_arch/
// deepseek_v4_mtp.rs, forward_one steps 1-2 and 6-7; spark_model/layers/mtp_head.rs, the
// embed+hidden concat -> fc order):
//   c  = [bf16(rms(embed[tok]) w_e) || bf16(rms(hidden) w_h)],  y = bf16(fc . c)
//   l[r] = sum_j head[r, j] y[j] (fp32),  idx = lowest allowed r with the largest l[r]
//
// Design (B200): for a head of a few MB, the separate launches and a grid-wide fold cost
// more than the bytes. One thread-block cluster (16 CTAs where the device allows, else 8)
// does it all, exchanging data through distributed shared memory: every CTA builds the
// concat rows itself (a few KB), CTA r computes fc output rows [r h/CL, (r+1) h/CL) and the
// CTAs then read each other's slices of y; the head's rows are split over the cluster, each
// warp keeping 16 rows' 16-byte loads in flight; per input the CTAs' (max, lowest row)
// partials go to CTA 0's shared memory and CTA 0 writes the result. Two cluster barriers,
// no global workspace. Launched with programmatic stream serialization, so in a chain of
// drafts the next step's launch overlaps this one's end: it first copies its fc and head
// rows into shared memory (bulk copies, when they fit in about 192 KB; else it pulls them
// into L1) and waits for the previous step only before reading the token and hidden rows
// that step writes.
#include <cuda_runtime.h>
#include <stdint.h>

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace mtp {
namespace {

constexpr int kDThreads = 512;  // 16 warps
constexpr int kDWarps = kDThreads / 32;
constexpr int kDRowsPerWarp = 16;  // head rows whose loads a warp keeps in flight (one input;
                                   // half that with more, for registers)
constexpr int kDMaxM = 4;
constexpr int kDMaxH = 1024;
constexpr int kDMaxCluster = 16;

struct DraftParams {
    const uint16_t* embed;
    int64_t vocab;
    const int32_t* tokens;  // [M]
    const uint16_t* hidden; // [M, h]
    int M, h;
    const uint16_t* w_ne;
    const uint16_t* w_nh;
    float eps;
    int norm_mode;          // 0: weights w, 1: weights 1 + w
    const uint16_t* fc;     // bf16 [h, 2h]
    const uint16_t* head;   // bf16 [n, h]
    int64_t n;              // rows swept
    const int32_t* mask;
    int64_t mask_words, mask_stride;
    uint16_t* out_y;        // [M, h] or null
    int32_t* out_idx;
    float* out_val;
    int32_t* dev_err;
    int staged;             // 1: the CTA's fc and head rows are copied into shared memory
};

__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_cluster_v2(uint32_t addr, float a, int32_t b) {
    asm volatile("st.shared::cluster.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(__float_as_uint(a)),
                 "r"(b)
                 : "memory");
}

__device__ __forceinline__ bool allowed(const DraftParams& p, int m, int64_t row) {
    if (!p.mask) return true;
    const int64_t w = row >> 5;
    if (w >= p.mask_words) return false;
    return (__ldg(p.mask + (int64_t)m * p.mask_stride + w) >> (row & 31)) & 1;
}

__device__ __forceinline__ float dot8(uint4 a, const uint16_t* y) {
    const uint4 b = lds128(y);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        s = fmaf(bf16_lo(av[i]), bf16_lo(bv[i]), s);
        s = fmaf(bf16_hi(av[i]), bf16_hi(bv[i]), s);
    }
    return s;
}

// MM: the most inputs this instance serves (1, or up to kDMaxM), which sizes its registers.
template <int MM>
__global__ void __launch_bounds__(kDThreads, 1) draft_step_kernel(const __grid_constant__ DraftParams p) {
    __shared__ __align__(16) uint16_t cs[kDMaxM][2 * kDMaxH];  // concat rows
    __shared__ __align__(16) uint16_t ys[kDMaxM][kDMaxH];      // fc output rows
    __shared__ float red[2][kDWarps];
    __shared__ float wv[kDWarps][kDMaxM];
    __shared__ int32_t wi[kDWarps][kDMaxM];
    __shared__ __align__(8) float2 cpart[kDMaxCluster][kDMaxM];  // CTA 0: (value, row bits)
    __shared__ __align__(8) uint64_t wbar;                        // the staged weights landed
    extern __shared__ __align__(128) uint8_t dsm[];               // staged fc rows, head rows
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int RPW = MM == 1 ? kDRowsPerWarp : kDRowsPerWarp / 2;
    const uint32_t rank = cluster_rank(), CL = cluster_size();
    const int M = p.M, h = p.h, h2 = 2 * h;
    pdl_launch_dependents();
    // The weights never change: this CTA's fc rows and head rows are fetched before waiting
    // for the previous step, so that their latency overlaps its end -- copied into shared
    // memory by bulk copies when they fit (staged), else pulled into L1.
    const int rows_per = (h + (int)CL - 1) / (int)CL;
    const int f0 = (int)rank * rows_per, f1 = min(h, f0 + rows_per);
    const int64_t per = (p.n + CL - 1) / CL;
    const int64_t q0 = (int64_t)rank * per, q1 = min(p.n, q0 + per);
    const uint32_t fbytes = (uint32_t)max(0, f1 - f0) * (uint32_t)h2 * 2u;
    const uint32_t hbytes = (uint32_t)max((int64_t)0, q1 - q0) * (uint32_t)h * 2u;
    const uint32_t hoff = (fbytes + 127u) & ~127u;  // head rows after the fc rows
    const uint16_t* fc_s = reinterpret_cast<const uint16_t*>(dsm);
    const uint16_t* head_s = reinterpret_cast<const uint16_t*>(dsm + hoff);
    if (p.staged) {
        if (tid == 0) {
            mbar_init(&wbar, 1);
            mbar_fence_init();
        }
        __syncthreads();
        if (warp == 0) {
            constexpr uint32_t kPiece = 16384;
            const uint32_t nf = (fbytes + kPiece - 1) / kPiece, nh = (hbytes + kPiece - 1) / kPiece;
            if (lane == 0) mbar_arrive_expect_tx(&wbar, fbytes + hbytes);
            __syncwarp();
            const uint8_t* fb = reinterpret_cast<const uint8_t*>(p.fc + (int64_t)f0 * h2);
            const uint8_t* hb = reinterpret_cast<const uint8_t*>(p.head + q0 * h);
            for (uint32_t i = lane; i < nf + nh; i += 32) {
                const bool isf = i < nf;
                const uint32_t o = (isf ? i : i - nf) * kPiece;
                const uint32_t n = min(kPiece, (isf ? fbytes : hbytes) - o);
                bulk_copy_g2s(dsm + (isf ? 0u : hoff) + o, (isf ? fb : hb) + o, n, &wbar);
            }
        }
    } else {
        const int64_t fl = fbytes / 128, hl = hbytes / 128;  // 128-byte lines
        const uint8_t* fb = reinterpret_cast<const uint8_t*>(p.fc + (int64_t)f0 * h2);
        const uint8_t* hb = reinterpret_cast<const uint8_t*>(p.head + q0 * h);
        for (int64_t i = tid; i < fl + hl; i += kDThreads) {
            const uint8_t* a = i < fl ? fb + 128 * i : hb + 128 * (i - fl);
            asm volatile("prefetch.global.L1 [%0];" ::"l"(a));
        }
    }
    pdl_wait();  // tokens and hidden rows may come from the previous step

    // 1. concat rows (every CTA): two RMSNorms with plain weights, bf16 rounding
    for (int m = 0; m < M; ++m) {
        const int64_t tok = p.tokens[m];
        const bool bad = tok < 0 || tok >= p.vocab;
        if (bad && tid == 0 && rank == 0) raise_flag(p.dev_err, DEVFLAG_BAD_TOKEN);
        const uint16_t* e = bad ? nullptr : p.embed + tok * h;
        const uint16_t* x = p.hidden + (int64_t)m * h;
        float se = 0.f, sx = 0.f;
        for (int j = tid; j < h; j += kDThreads) {
            const float ev = e ? bf16_to_f32(e[j]) : 0.f, xv = bf16_to_f32(x[j]);
            se += ev * ev;
            sx += xv * xv;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            se += __shfl_xor_sync(0xffffffffu, se, o);
            sx += __shfl_xor_sync(0xffffffffu, sx, o);
        }
        if (lane == 0) {
            red[0][warp] = se;
            red[1][warp] = sx;
        }
        __syncthreads();
        se = sx = 0.f;
#pragma unroll
        for (int w = 0; w < kDWarps; ++w) {
            se += red[0][w];
            sx += red[1][w];
        }
        const float inv_e = 1.0f / sqrtf(se / (float)h + p.eps);
        const float inv_x = 1.0f / sqrtf(sx / (float)h + p.eps);
        const float add = p.norm_mode ? 1.f : 0.f;  // weights w or 1 + w
        for (int j = tid; j < h; j += kDThreads) {
            const float ev = e ? bf16_to_f32(e[j]) : 0.f;
            cs[m][j] = f32_to_bf16(ev * inv_e * (bf16_to_f32(p.w_ne[j]) + add));
            cs[m][h + j] = f32_to_bf16(bf16_to_f32(x[j]) * inv_x * (bf16_to_f32(p.w_nh[j]) + add));
        }
        __syncthreads();
    }

    // 2. this CTA's slice of y = bf16(fc . c): a warp per fc row, 16-byte pieces per lane
    if (p.staged && !mbar_wait_bounded(&wbar, 0u, nullptr) && tid == 0)
        raise_flag(p.dev_err, DEVFLAG_TIMEOUT);  // (the copies' bytes never arrived)
    const int r0 = f0, r1 = f1;
    for (int r = r0 + warp; r < r1; r += kDWarps) {
        const uint16_t* frow = p.staged ? fc_s + (int64_t)(r - r0) * h2 : p.fc + (int64_t)r * h2;
        float acc[MM];
#pragma unroll
        for (int m = 0; m < MM; ++m) acc[m] = 0.f;
        for (int c = lane; c < h2 / 8; c += 32) {
            const uint4 a = p.staged ? lds128(frow + 8 * c) : __ldg(reinterpret_cast<const uint4*>(frow + 8 * c));
#pragma unroll
            for (int m = 0; m < MM; ++m)
                if (m < M) acc[m] += dot8(a, &cs[m][8 * c]);
        }
#pragma unroll
        for (int m = 0; m < MM; ++m) {
            if (m >= M) break;
            float s = acc[m];
#pragma unroll
            for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) ys[m][r] = f32_to_bf16(s);
        }
    }
    cluster_sync();  // every slice of y is in its CTA's shared memory
    // gather the other CTAs' slices (32-bit pieces; slices are whole rows of y, and h is even)
    for (int i = tid; i < M * (h / 2); i += kDThreads) {
        const int m = i / (h / 2), j = 2 * (i - m * (h / 2));
        const uint32_t owner = (uint32_t)(j / rows_per);
        if (owner == rank) continue;
        if (j / rows_per != (j + 1) / rows_per) {  // a slice boundary inside the pair
            const uint32_t o2 = (uint32_t)((j + 1) / rows_per);
            const uint32_t lo = ld_cluster_u32(map_rank(&ys[m][j], owner)) & 0xFFFFu;
            const uint32_t hi = ld_cluster_u32(map_rank(&ys[m][j], o2)) & 0xFFFF0000u;
            if (owner != rank) ys[m][j] = (uint16_t)lo;
            if (o2 != rank) ys[m][j + 1] = (uint16_t)(hi >> 16);
            continue;
        }
        *reinterpret_cast<uint32_t*>(&ys[m][j]) = ld_cluster_u32(map_rank(&ys[m][j], owner));
    }
    __syncthreads();
    if (rank == 0 && p.out_y)
        for (int i = tid; i < M * h; i += kDThreads) p.out_y[i] = ys[i / h][i % h];

    // 3. this CTA's rows of the head: warp w takes 16-row groups; lane l holds 16-byte piece
    // l (and l + 32, ...) of each row; each lane keeps a running (max, lowest row) per input
    float bv[MM];
    int32_t bi[MM];
#pragma unroll
    for (int m = 0; m < MM; ++m) {
        bv[m] = -INFINITY;
        bi[m] = INT_MAX;
    }
    const int64_t n0 = q0, n1 = q1;
    const int pieces = h / 8;
    for (int64_t g = n0 + (int64_t)warp * RPW; g < n1; g += (int64_t)kDWarps * RPW) {
        float acc[RPW][MM];
#pragma unroll
        for (int j = 0; j < RPW; ++j)
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[j][m] = 0.f;
        for (int c0 = 0; c0 < pieces; c0 += 32) {
            const int c = c0 + lane;
            uint4 a[RPW];
#pragma unroll
            for (int j = 0; j < RPW; ++j)
                a[j] = (c < pieces && g + j < n1)
                           ? (p.staged ? lds128(head_s + (g + j - n0) * h + 8 * c)
                                       : __ldg(reinterpret_cast<const uint4*>(p.head + (g + j) * h + 8 * c)))
                           : make_uint4(0, 0, 0, 0);
            if (c < pieces) {
#pragma unroll
                for (int j = 0; j < RPW; ++j)
#pragma unroll
                    for (int m = 0; m < MM; ++m)
                        if (m < M) acc[j][m] += dot8(a[j], &ys[m][8 * c]);
            }
        }
#pragma unroll
        for (int j = 0; j < RPW; ++j) {
            const int64_t row = g + j;
#pragma unroll
            for (int m = 0; m < MM; ++m) {
                if (m >= M) break;
                float s = acc[j][m];
#pragma unroll
                for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                // rows arrive in increasing order within the warp: the first wins a tie
                if (row < n1 && allowed(p, m, row) && s > bv[m]) {
                    bv[m] = s;
                    bi[m] = (int32_t)row;
                }
            }
        }
    }
    if (lane == 0)
#pragma unroll
        for (int m = 0; m < MM; ++m) {
            wv[warp][m] = bv[m];
            wi[warp][m] = bi[m];
        }
    __syncthreads();
    if (warp == 0 && lane < M) {  // fold the warps; ties to the lowest row
        float v = -INFINITY;
        int32_t i = INT_MAX;
        for (int w = 0; w < kDWarps; ++w)
            if (wv[w][lane] > v || (wv[w][lane] == v && wi[w][lane] < i)) {
                v = wv[w][lane];
                i = wi[w][lane];
            }
        st_cluster_v2(map_rank(&cpart[rank][lane], 0), v, i);
    }
    cluster_sync();  // every CTA's partial is in CTA 0's shared memory
    if (rank == 0 && warp == 0 && lane < M) {
        float v = -INFINITY;
        int32_t i = INT_MAX;
        for (uint32_t r = 0; r < CL; ++r) {
            const float pv = cpart[r][lane].x;
            const int32_t pi = __float_as_int(cpart[r][lane].y);
            if (pv > v || (pv == v && pi < i)) {
                v = pv;
                i = pi;
            }
        }
        if (i == INT_MAX) {  // nothing allowed
            i = 0;
            v = -INFINITY;
            raise_flag(p.dev_err, DEVFLAG_EMPTY_MASK);
        }
        p.out_idx[lane] = i;
        if (p.out_val) p.out_val[lane] = v;
    }
}

}  // namespace

int draft_step_max_m() { return kDMaxM; }
int draft_step_max_h() { return kDMaxH; }

cudaError_t draft_step_launch(const uint16_t* embed, int64_t vocab, const int32_t* tokens,
                              const uint16_t* hidden, int M, int h, const uint16_t* w_ne,
                              const uint16_t* w_nh, float eps, int norm_mode, const uint16_t* fc,
                              const uint16_t* head, int64_t n, const int32_t* mask,
                              int64_t mask_words, int64_t mask_stride, uint16_t* out_y,
                              int32_t* out_idx, float* out_val, int32_t* dev_err, cudaStream_t s) {
    DraftParams p{};
    p.embed = embed;
    p.vocab = vocab;
    p.tokens = tokens;
    p.hidden = hidden;
    p.M = M;
    p.h = h;
    p.w_ne = w_ne;
    p.w_nh = w_nh;
    p.eps = eps;
    p.norm_mode = norm_mode;
    p.fc = fc;
    p.head = head;
    p.n = n;
    p.mask = mask;
    p.mask_words = mask ? mask_words : 0;
    p.mask_stride = mask ? mask_stride : 0;
    p.out_y = out_y;
    p.out_idx = out_idx;
    p.out_val = out_val;
    p.dev_err = dev_err;
    // 16 CTAs per cluster where the device allows it, else the portable 8; each CTA's fc
    // and head rows staged in shared memory when they fit beside the static arrays
    auto kern = M == 1 ? draft_step_kernel<1> : draft_step_kernel<kDMaxM>;
    auto staged_bytes = [&](int clusters) -> size_t {
        const size_t rows_per = (size_t)((h + clusters - 1) / clusters);
        const size_t per = (size_t)((n + clusters - 1) / clusters);
        return ((rows_per * 2 * (size_t)h * 2 + 127) & ~(size_t)127) + per * (size_t)h * 2;
    };
    constexpr size_t kStageLimit = 192 * 1024;  // beside ~26 KB of static shared memory
    static int cl_cached[2][64] = {{0}};  // per instance and device: the cluster size used
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int inst = M == 1 ? 0 : 1;
    // the cluster size is the same for every head: it is chosen with the staging limit
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStageLimit) !=
        cudaSuccess)
        cudaGetLastError();
    int cl = dev >= 0 && dev < 64 ? cl_cached[inst][dev] : 0;
    if (cl == 0) {
        cl = 8;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
            cudaSuccess) {
            cudaLaunchConfig_t q{};
            q.gridDim = dim3(kDMaxCluster);
            q.blockDim = dim3(kDThreads);
            q.dynamicSmemBytes = kStageLimit;
            cudaLaunchAttribute qa[1];
            qa[0].id = cudaLaunchAttributeClusterDimension;
            qa[0].val.clusterDim.x = kDMaxCluster;
            qa[0].val.clusterDim.y = 1;
            qa[0].val.clusterDim.z = 1;
            q.attrs = qa;
            q.numAttrs = 1;
            int maxc = 0;
            if (cudaOccupancyMaxPotentialClusterSize(&maxc, kern, &q) == cudaSuccess &&
                maxc >= kDMaxCluster)
                cl = kDMaxCluster;
        }
        cudaGetLastError();  // a refused attribute or query leaves nothing behind
        if (dev >= 0 && dev < 64) cl_cached[inst][dev] = cl;
    }
    const size_t sb = staged_bytes(cl);
    p.staged = sb <= kStageLimit;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)cl);
    cfg.blockDim = dim3(kDThreads);
    cfg.dynamicSmemBytes = p.staged ? sb : 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if ((e = cudaLaunchKernelEx(&cfg, kern, p)) != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace mtp
