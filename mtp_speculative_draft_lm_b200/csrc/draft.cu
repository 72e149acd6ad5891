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
// concat rows itself (a few KB), CTA r computes an even slice of fc output rows and stores
// each finished pair of y elements into every CTA's shared memory (st.async, the bytes
// completing on that CTA's mbarrier, so that each CTA waits only for its own copy of y, not
// for a cluster barrier); the head's rows are split over the cluster and swept on the
// tensor cores (mma.sync, 16 rows by 8 columns, column j being input j, so the k sum needs
// no shuffles); per input the warps' and then the CTAs' (max, lowest row) partials are
// folded across lanes, the CTAs' sent to CTA 0 the same way, and CTA 0 writes the result.
// No global workspace. Launched with
// programmatic stream serialization, so in a chain of drafts the next step's launch
// overlaps this one's end: it first copies its fc and head rows into shared memory (bulk
// copies, when they fit in about 192 KB; else it pulls them into L1), loads the norm
// weights, and waits for the previous step only before reading the token and hidden rows
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
constexpr int kDMaxM = 4;
constexpr int kDMaxH = 1024;
constexpr int kDMaxCluster = 16;
constexpr int kResMaxH = 256;                  // register form: h (8 steps of 32 columns)
constexpr int kResSteps = kResMaxH / 32;
constexpr int kResMaxRowsPerCta = 16 * kDWarps;  // register form: one 16-row tile per warp

// Staged head row pitch in bytes: 2h rounded up to 64 modulo 128.
__host__ __device__ constexpr uint32_t head_pitch(int h) {
    return (uint32_t)(2 * h) + ((64u - ((uint32_t)(2 * h) & 127u)) & 127u);
}

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
// Stores into CTA-of-the-cluster shared memory whose bytes complete on that CTA's mbarrier
// `bar` (both shared::cluster addresses in the same CTA).
__device__ __forceinline__ void st_async_u32(uint32_t addr, uint32_t v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(addr),
                 "r"(v), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v2u(uint32_t addr, uint32_t a, uint32_t b, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(addr),
                 "r"(a), "r"(b), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v4(uint32_t addr, uint4 v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     addr),
                 "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t addr, float a, int32_t b, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(
                     addr),
                 "r"(__float_as_uint(a)), "r"(b), "r"(bar)
                 : "memory");
}
// The cluster barrier in two halves: arrive (no ordering) early, wait before the first
// access to another CTA's shared memory, which must not come before that CTA runs.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
// A 16-byte load that stays where it is written: the register form fetches its weights
// before the wait for the previous step. A non-coherent (read-only) load may legally be
// issued again where its value is used -- with registers at their cap it was, putting an L2
// round trip back on the step's critical path (about 1.6 us per draft) -- so this one is a
// plain coherent load, which cannot be.
__device__ __forceinline__ uint4 ldg_here(const void* p) {
    uint4 r;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
// Wait for phase `parity` of this CTA's mbarrier `bar`, which other CTAs of the cluster
// complete, by polling (no suspend: these waits are short and on the step's critical path);
// gives up after kWaitLimitCycles.
__device__ __forceinline__ bool spin_wait_cluster(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity, 0u)) return true;
        if (clock64() - t0 > kWaitLimitCycles) return false;
    }
}
// Fold (value, row) over the warp: the largest value, ties to the lowest row, in every lane.
// Values map to unsigned keys in the same order (-0 taken as +0; values are never NaN here:
// a NaN logit never becomes a best), so two warp reductions do it.
__device__ __forceinline__ void warp_fold_max(float& v, int32_t& i) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    const uint32_t key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    uint32_t km, im;
    asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(km) : "r"(key));
    asm volatile("redux.sync.min.u32 %0, %1, 0xffffffff;" : "=r"(im) : "r"(key == km ? (uint32_t)i : 0xffffffffu));
    v = __uint_as_float((km & 0x80000000u) ? (km & 0x7fffffffu) : ~km);
    i = (int32_t)im;
}
// Keep (v, i) or take (ov, oi): the larger value, ties to the lower row.
__device__ __forceinline__ void fold_max(float& v, int32_t& i, float ov, int32_t oi) {
    if (ov > v || (ov == v && oi < i)) {
        v = ov;
        i = oi;
    }
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

// Keep the per-input best of a 16-row tile's results (lane (g, t): rows ra = tile + g and
// rb = ra + 8, inputs 2t and 2t + 1), rows in increasing order: the first of equal wins.
__device__ __forceinline__ void tile_best(const DraftParams& p, const float (&c0)[4], const float (&c1)[4],
                                          int64_t ra, int64_t rb, int64_t q1, int t, float& bv0,
                                          int32_t& bi0, float& bv1, int32_t& bi1) {
    const int M = p.M, m0 = 2 * t, m1 = 2 * t + 1;
    const bool va = ra < q1, vb = rb < q1;
    const float la0 = c0[0] + c1[0], la1 = c0[1] + c1[1];
    const float lb0 = c0[2] + c1[2], lb1 = c0[3] + c1[3];
    if (m0 < M) {
        if (va && allowed(p, m0, ra) && la0 > bv0) { bv0 = la0; bi0 = (int32_t)ra; }
        if (vb && allowed(p, m0, rb) && lb0 > bv0) { bv0 = lb0; bi0 = (int32_t)rb; }
    }
    if (m1 < M) {
        if (va && allowed(p, m1, ra) && la1 > bv1) { bv1 = la1; bi1 = (int32_t)ra; }
        if (vb && allowed(p, m1, rb) && lb1 > bv1) { bv1 = lb1; bi1 = (int32_t)rb; }
    }
}

// MM: the most inputs this instance serves (1, or up to kDMaxM), which sizes its registers.
// RES (one input, h <= kResMaxH, at most 16 head rows per warp): the weights live in
// registers -- each warp loads its pair of fc rows and its 16-row tile of the head as MMA
// fragments before waiting for the previous step, and builds the concat pieces it needs
// itself (no shared-memory concat rows, no block barrier); otherwise they are staged in
// shared memory (or read through L1) and the warps loop over tiles.
template <int MM, bool RES>
__global__ void __launch_bounds__(kDThreads, 1) draft_step_kernel(const __grid_constant__ DraftParams p) {
    static_assert(!RES || MM == 1, "the register-resident form serves one input");
    __shared__ __align__(16) uint16_t cs[RES ? 1 : kDMaxM][RES ? 8 : 2 * kDMaxH];  // concat rows
    __shared__ __align__(16) uint16_t ys[kDMaxM][kDMaxH];  // y rows (all of y, every CTA)
    __shared__ float red[2][kDMaxM][kDWarps];
    __shared__ float wv[kDWarps][kDMaxM];
    __shared__ int32_t wi[kDWarps][kDMaxM];
    __shared__ __align__(8) float2 cpart[kDMaxCluster][kDMaxM];  // CTA 0: (value, row bits)
    __shared__ __align__(8) uint64_t wbar;  // the staged weights landed
    __shared__ __align__(8) uint64_t ybar;  // all of y landed (M h 2 bytes from the CTAs)
    __shared__ __align__(8) uint64_t cbar;  // CTA 0: every CTA's partials landed
    extern __shared__ __align__(128) uint8_t dsm[];  // staged fc rows, head rows
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
    const uint32_t rank = cluster_rank(), CL = cluster_size();
    const int M = p.M, h = p.h, h2 = 2 * h;
    const int chunks = h >> 3, ksteps = (chunks + 3) >> 2;  // 16-byte pieces, 32-column steps
    pdl_launch_dependents();
    if (tid == 0) {
        mbar_init(&wbar, 1);
        mbar_init(&ybar, 1);
        mbar_init(&cbar, 1);
        mbar_fence_init();
        mbar_arrive_expect_tx(&ybar, (uint32_t)M * (uint32_t)h * 2u);
        if (rank == 0) mbar_arrive_expect_tx(&cbar, CL * (uint32_t)M * 8u);  // a partial per CTA, input
    }
    // this CTA runs and its barriers are initialised: the others may write its shared memory
    cluster_arrive_relaxed();
    const int rows_per = 2 * ((h + 2 * (int)CL - 1) / (2 * (int)CL));  // even: y goes in words
    const int f0 = (int)rank * rows_per, f1 = min(h, f0 + rows_per);
    const int64_t per = (p.n + CL - 1) / CL;
    const int64_t q0 = (int64_t)rank * per, q1 = min(p.n, q0 + per);
    const int64_t nrows = max((int64_t)0, q1 - q0);
    const uint32_t fbytes = (uint32_t)max(0, f1 - f0) * (uint32_t)h2 * 2u;
    const uint32_t hrow = (uint32_t)h * 2u, hpitch = head_pitch(h);
    const uint32_t hoff = (fbytes + 127u) & ~127u;  // head rows after the fc rows
    const uint16_t* fc_s = reinterpret_cast<const uint16_t*>(dsm);
    const uint16_t* head_s = reinterpret_cast<const uint16_t*>(dsm + hoff);
    const float add = p.norm_mode ? 1.f : 0.f;  // weights w or 1 + w

    // The weights never change: they are fetched before waiting for the previous step, so
    // that their latency overlaps its end.
    constexpr int kPer = kDMaxH / kDThreads;
    float wne[kPer], wnh[kPer];                      // staged form: this thread's norm weights
    uint4 fr[2][2], ha[kResSteps], hb[kResSteps];    // register form: fc pair, head fragments
    const int fr0 = f0 + 2 * warp;                   // register form: this warp's fc pair
    const int64_t ra = q0 + 16 * warp + g, rb = ra + 8;  // register form: this lane's head rows
    if constexpr (RES) {
        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int c = lane + 32 * i;
                fr[r][i] = fr0 + r < f1 && c < h2 / 8 ? ldg_here(p.fc + (int64_t)(fr0 + r) * h2 + 8 * c) : z;
            }
#pragma unroll
        for (int s = 0; s < kResSteps; ++s) {
            const int ch = 4 * s + t;
            ha[s] = ch < chunks && ra < q1 ? ldg_here(p.head + ra * h + 8 * ch) : z;
            hb[s] = ch < chunks && rb < q1 ? ldg_here(p.head + rb * h + 8 * ch) : z;
        }
    } else {
        // copied into shared memory by bulk copies when they fit (staged; head rows at a
        // pitch of 64 bytes modulo 128, so that the two rows that one quarter-warp's
        // fragment loads touch fall in different banks), else pulled into L1
        if (p.staged) {
            if (warp == 0) {  // (wbar was initialised by lane 0)
                constexpr uint32_t kPiece = 16384;
                const uint32_t nf = (fbytes + kPiece - 1) / kPiece;
                if (lane == 0) mbar_arrive_expect_tx(&wbar, fbytes + (uint32_t)nrows * hrow);
                __syncwarp();
                const uint8_t* fb = reinterpret_cast<const uint8_t*>(p.fc + (int64_t)f0 * h2);
                const uint8_t* hbp = reinterpret_cast<const uint8_t*>(p.head + q0 * h);
                for (uint32_t i = lane; i < nf + (uint32_t)nrows; i += 32) {
                    if (i < nf) {
                        const uint32_t o = i * kPiece;
                        bulk_copy_g2s(dsm + o, fb + o, min(kPiece, fbytes - o), &wbar);
                    } else {
                        const uint32_t r = i - nf;
                        bulk_copy_g2s(dsm + hoff + r * hpitch, hbp + (int64_t)r * hrow, hrow, &wbar);
                    }
                }
            }
        } else {
            const int64_t fl = fbytes / 128, hl = nrows * hrow / 128;  // 128-byte lines
            const uint8_t* fb = reinterpret_cast<const uint8_t*>(p.fc + (int64_t)f0 * h2);
            const uint8_t* hbp = reinterpret_cast<const uint8_t*>(p.head + q0 * h);
            for (int64_t i = tid; i < fl + hl; i += kDThreads) {
                const uint8_t* a = i < fl ? fb + 128 * i : hbp + 128 * (i - fl);
                asm volatile("prefetch.global.L1 [%0];" ::"l"(a));
            }
        }
        // the norm weights: this thread's elements j = tid + i kDThreads
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int j = tid + i * kDThreads;
            wne[i] = j < h ? bf16_to_f32(p.w_ne[j]) + add : 0.f;
            wnh[i] = j < h ? bf16_to_f32(p.w_nh[j]) + add : 0.f;
        }
    }
    pdl_wait();  // tokens and hidden rows may come from the previous step

    if constexpr (RES) {
        // 1+2. a warp with an fc pair builds the concat pieces its lanes take in the fc dot
        // products (pieces lane and lane + 32 of [e-part || x-part]), with both RMS sums
        // reduced over the warp, and writes its pair of y here (and into out_y); then warp 0
        // stores the CTA's slice into every CTA's copy of y in pieces of up to 16 bytes
        const int npairs = (f1 - f0) / 2;  // warps with an fc pair (f0, f1 even)
        if (fr0 < f1) {
            const int64_t tok = p.tokens[0];
            const bool bad = tok < 0 || tok >= p.vocab;
            if (bad && lane == 0 && rank == 0 && warp == 0) raise_flag(p.dev_err, DEVFLAG_BAD_TOKEN);
            const uint16_t* e = bad ? nullptr : p.embed + tok * h;
            uint4 v[2], w[2];
            float se = 0.f, sx = 0.f;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int c = lane + 32 * i;
                const bool ise = c < chunks, isx = !ise && c < 2 * chunks;
                v[i] = make_uint4(0, 0, 0, 0);
                w[i] = v[i];
                if (ise) {
                    if (e) v[i] = __ldg(reinterpret_cast<const uint4*>(e + 8 * c));
                    w[i] = __ldg(reinterpret_cast<const uint4*>(p.w_ne + 8 * c));
                } else if (isx) {
                    v[i] = *reinterpret_cast<const uint4*>(p.hidden + 8 * (c - chunks));
                    w[i] = __ldg(reinterpret_cast<const uint4*>(p.w_nh + 8 * (c - chunks)));
                }
                const uint32_t vv[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                float q = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    q += bf16_lo(vv[k]) * bf16_lo(vv[k]);
                    q += bf16_hi(vv[k]) * bf16_hi(vv[k]);
                }
                if (ise) se += q;
                else sx += q;
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                se += __shfl_xor_sync(0xffffffffu, se, o);
                sx += __shfl_xor_sync(0xffffffffu, sx, o);
            }
            const float inv_e = 1.0f / sqrtf(se / (float)h + p.eps);
            const float inv_x = 1.0f / sqrtf(sx / (float)h + p.eps);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int c = lane + 32 * i;
                const float inv = c < chunks ? inv_e : inv_x;
                const uint32_t vv[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                const uint32_t ww[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
                const uint32_t a0[4] = {fr[0][i].x, fr[0][i].y, fr[0][i].z, fr[0][i].w};
                const uint32_t a1[4] = {fr[1][i].x, fr[1][i].y, fr[1][i].z, fr[1][i].w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float clo = bf16_to_f32(f32_to_bf16(bf16_lo(vv[k]) * inv * (bf16_lo(ww[k]) + add)));
                    const float chi = bf16_to_f32(f32_to_bf16(bf16_hi(vv[k]) * inv * (bf16_hi(ww[k]) + add)));
                    s0 = fmaf(bf16_lo(a0[k]), clo, s0);
                    s0 = fmaf(bf16_hi(a0[k]), chi, s0);
                    s1 = fmaf(bf16_lo(a1[k]), clo, s1);
                    s1 = fmaf(bf16_hi(a1[k]), chi, s1);
                }
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                s0 += __shfl_xor_sync(0xffffffffu, s0, o);
                s1 += __shfl_xor_sync(0xffffffffu, s1, o);
            }
            const uint16_t y0 = f32_to_bf16(s0), y1 = f32_to_bf16(s1);
            if (lane == 0) {
                *reinterpret_cast<uint32_t*>(&ys[0][fr0]) = (uint32_t)y0 | ((uint32_t)y1 << 16);
                if (p.out_y) {
                    p.out_y[fr0] = y0;
                    p.out_y[fr0 + 1] = y1;
                }
            }
            named_sync(1, npairs * 32);  // the CTA's slice of y is complete
        }
        cluster_wait();  // every CTA of the cluster has started
        if (warp == 0 && npairs > 0) {
            // piece size: the largest of 16, 8, 4 bytes dividing the slice pitch, so that
            // every slice starts and ends on a piece
            const int pitch = rows_per * 2;
            const int chunk = pitch % 16 == 0 ? 16 : (pitch % 8 == 0 ? 8 : 4);
            const int npieces = (f1 - f0) * 2 / chunk;
            const uint8_t* slice = reinterpret_cast<const uint8_t*>(&ys[0][f0]);
            for (int q = lane; q < (int)CL * npieces; q += 32) {
                const uint32_t dst = (uint32_t)(q / npieces);
                const int off = (q % npieces) * chunk;
                const uint32_t a = map_rank(slice + off, dst), b = map_rank(&ybar, dst);
                if (chunk == 16) {
                    st_async_v4(a, *reinterpret_cast<const uint4*>(slice + off), b);
                } else if (chunk == 8) {
                    const uint2 v = *reinterpret_cast<const uint2*>(slice + off);
                    st_async_v2u(a, v.x, v.y, b);
                } else {
                    st_async_u32(a, *reinterpret_cast<const uint32_t*>(slice + off), b);
                }
            }
        }
    } else {
        // 1. concat rows (every CTA): two RMSNorms per input, bf16 rounding; every input's
        // rows are read at once and reduced with one block barrier
        float ev[MM][kPer], xv[MM][kPer];
#pragma unroll
        for (int m = 0; m < MM; ++m) {
            if (m >= M) break;
            const int64_t tok = p.tokens[m];
            const bool bad = tok < 0 || tok >= p.vocab;
            if (bad && tid == 0 && rank == 0) raise_flag(p.dev_err, DEVFLAG_BAD_TOKEN);
            const uint16_t* e = bad ? nullptr : p.embed + tok * h;
            const uint16_t* x = p.hidden + (int64_t)m * h;
            float se = 0.f, sx = 0.f;
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int j = tid + i * kDThreads;
                ev[m][i] = (j < h && e) ? bf16_to_f32(e[j]) : 0.f;
                xv[m][i] = j < h ? bf16_to_f32(x[j]) : 0.f;
                se += ev[m][i] * ev[m][i];
                sx += xv[m][i] * xv[m][i];
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                se += __shfl_xor_sync(0xffffffffu, se, o);
                sx += __shfl_xor_sync(0xffffffffu, sx, o);
            }
            if (lane == 0) {
                red[0][m][warp] = se;
                red[1][m][warp] = sx;
            }
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < MM; ++m) {
            if (m >= M) break;
            float se = 0.f, sx = 0.f;
#pragma unroll
            for (int w = 0; w < kDWarps; ++w) {
                se += red[0][m][w];
                sx += red[1][m][w];
            }
            const float inv_e = 1.0f / sqrtf(se / (float)h + p.eps);
            const float inv_x = 1.0f / sqrtf(sx / (float)h + p.eps);
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int j = tid + i * kDThreads;
                if (j < h) {
                    cs[m][j] = f32_to_bf16(ev[m][i] * inv_e * wne[i]);
                    cs[m][h + j] = f32_to_bf16(xv[m][i] * inv_x * wnh[i]);
                }
            }
        }
        __syncthreads();

        // 2. this CTA's slice of y = bf16(fc . c): a warp per pair of fc rows, 16-byte
        // pieces per lane; each finished pair of y is stored into every CTA's copy of y
        if (p.staged && !mbar_wait_bounded(&wbar, 0u, nullptr) && tid == 0)
            raise_flag(p.dev_err, DEVFLAG_TIMEOUT);  // (the copies' bytes never arrived)
        cluster_wait();  // every CTA of the cluster has started
        for (int r = f0 + 2 * warp; r < f1; r += 2 * kDWarps) {  // r + 1 < f1: f0, f1 even
            const uint16_t* frow = p.staged ? fc_s + (int64_t)(r - f0) * h2 : p.fc + (int64_t)r * h2;
            float acc[2][MM];
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[0][m] = acc[1][m] = 0.f;
            for (int c = lane; c < h2 / 8; c += 32) {
                const uint4 a0 = p.staged ? lds128(frow + 8 * c) : __ldg(reinterpret_cast<const uint4*>(frow + 8 * c));
                const uint4 a1 = p.staged ? lds128(frow + h2 + 8 * c)
                                          : __ldg(reinterpret_cast<const uint4*>(frow + h2 + 8 * c));
#pragma unroll
                for (int m = 0; m < MM; ++m)
                    if (m < M) {
                        acc[0][m] += dot8(a0, &cs[m][8 * c]);
                        acc[1][m] += dot8(a1, &cs[m][8 * c]);
                    }
            }
#pragma unroll
            for (int m = 0; m < MM; ++m) {
                if (m >= M) break;
                float s0 = acc[0][m], s1 = acc[1][m];
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    s0 += __shfl_xor_sync(0xffffffffu, s0, o);
                    s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                }
                const uint16_t y0 = f32_to_bf16(s0), y1 = f32_to_bf16(s1);
                if (lane < (int)CL)
                    st_async_u32(map_rank(&ys[m][r], (uint32_t)lane), (uint32_t)y0 | ((uint32_t)y1 << 16),
                                 map_rank(&ybar, (uint32_t)lane));
                if (lane == 0 && p.out_y) {
                    p.out_y[(int64_t)m * h + r] = y0;
                    p.out_y[(int64_t)m * h + r + 1] = y1;
                }
            }
        }
    }
    if (!spin_wait_cluster(&ybar, 0u) && tid == 0)
        raise_flag(p.dev_err, DEVFLAG_TIMEOUT);  // all of y is in this CTA's shared memory

    // 3. this CTA's rows of the head on the tensor cores (mma.sync m16n8k16, bf16 operands,
    // fp32 sums): a warp takes 16-row tiles, column j of the product is input j (zero for
    // j >= M). Lane (g, t) = (lane / 4, lane % 4) holds tile rows g and g + 8; of every 32
    // columns of k it loads the 16 bytes at 8 t of both rows and of y[g], and the MMA's k
    // slots (2t, 2t+1, 2t+8, 2t+9) take elements 0-3 of them in the first MMA and 4-7 in
    // the second: rows and y pair the same k, and each k of the 32 is taken once.
    float bv0 = -INFINITY, bv1 = -INFINITY;
    int32_t bi0 = INT_MAX, bi1 = INT_MAX;
    if constexpr (RES) {
        float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s = 0; s < kResSteps; ++s) {
            if (s >= ksteps) break;
            const int ch = 4 * s + t;
            const uint4 y = ch < chunks && g == 0 ? lds128(&ys[0][8 * ch]) : make_uint4(0, 0, 0, 0);
            mma_bf16_16816(c0, ha[s].x, hb[s].x, ha[s].y, hb[s].y, y.x, y.y);
            mma_bf16_16816(c1, ha[s].z, hb[s].z, ha[s].w, hb[s].w, y.z, y.w);
        }
        tile_best(p, c0, c1, ra, rb, q1, t, bv0, bi0, bv1, bi1);
    } else {
        const int64_t hpe = hpitch / 2;  // staged pitch in elements
        for (int64_t r0 = q0 + 16 * warp; r0 < q1; r0 += 16 * kDWarps) {
            const int64_t ta = r0 + g, tb = ta + 8;
            const bool va = ta < q1, vb = tb < q1;
            const uint16_t* pa = p.staged ? head_s + (ta - q0) * hpe : p.head + ta * h;
            const uint16_t* pb = p.staged ? head_s + (tb - q0) * hpe : p.head + tb * h;
            float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int s = 0; s < ksteps; ++s) {
                const int ch = 4 * s + t;
                uint4 a = make_uint4(0, 0, 0, 0), b = a, y = a;
                if (ch < chunks) {
                    if (va) a = p.staged ? lds128(pa + 8 * ch) : __ldg(reinterpret_cast<const uint4*>(pa + 8 * ch));
                    if (vb) b = p.staged ? lds128(pb + 8 * ch) : __ldg(reinterpret_cast<const uint4*>(pb + 8 * ch));
                    if (g < M) y = lds128(&ys[g][8 * ch]);
                }
                mma_bf16_16816(c0, a.x, b.x, a.y, b.y, y.x, y.y);
                mma_bf16_16816(c1, a.z, b.z, a.w, b.w, y.z, y.w);
            }
            tile_best(p, c0, c1, ta, tb, q1, t, bv0, bi0, bv1, bi1);
        }
    }
    if constexpr (RES) {
        // one input (lanes t != 0 hold nothing): fold the warp, then the CTA's warps, and send
        // the CTA's partial to CTA 0, which folds the CTAs'
        warp_fold_max(bv0, bi0);
        if (lane == 0) {
            wv[warp][0] = bv0;
            wi[warp][0] = bi0;
        }
        __syncthreads();
        if (warp == 0) {
            float v = lane < kDWarps ? wv[lane][0] : -INFINITY;
            int32_t i = lane < kDWarps ? wi[lane][0] : INT_MAX;
            warp_fold_max(v, i);
            if (lane == 0) st_async_v2(map_rank(&cpart[rank][0], 0), v, i, map_rank(&cbar, 0));
            if (rank == 0) {
                if (!spin_wait_cluster(&cbar, 0u) && lane == 0) raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
                v = lane < (int)CL ? cpart[lane][0].x : -INFINITY;
                i = lane < (int)CL ? __float_as_int(cpart[lane][0].y) : INT_MAX;
                warp_fold_max(v, i);
                if (lane == 0) {
                    if (i == INT_MAX) {  // nothing allowed
                        i = 0;
                        v = -INFINITY;
                        raise_flag(p.dev_err, DEVFLAG_EMPTY_MASK);
                    }
                    p.out_idx[0] = i;
                    if (p.out_val) p.out_val[0] = v;
                }
            }
        }
        return;
    }
    // fold over the lanes of equal t (ties to the lowest row), then over the warps
    const int m0 = 2 * t, m1 = 2 * t + 1;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        fold_max(bv0, bi0, __shfl_xor_sync(0xffffffffu, bv0, o), __shfl_xor_sync(0xffffffffu, bi0, o));
        fold_max(bv1, bi1, __shfl_xor_sync(0xffffffffu, bv1, o), __shfl_xor_sync(0xffffffffu, bi1, o));
    }
    if (g == 0) {
        if (m0 < M) {
            wv[warp][m0] = bv0;
            wi[warp][m0] = bi0;
        }
        if (m1 < M) {
            wv[warp][m1] = bv1;
            wi[warp][m1] = bi1;
        }
    }
    __syncthreads();
    if (warp < M) {  // warp m folds input m over this CTA's warps and sends it to CTA 0
        float v = lane < kDWarps ? wv[lane][warp] : -INFINITY;
        int32_t i = lane < kDWarps ? wi[lane][warp] : INT_MAX;
#pragma unroll
        for (int o = 16; o; o >>= 1)
            fold_max(v, i, __shfl_xor_sync(0xffffffffu, v, o), __shfl_xor_sync(0xffffffffu, i, o));
        if (lane == 0) st_async_v2(map_rank(&cpart[rank][warp], 0), v, i, map_rank(&cbar, 0));
        // CTA 0 waits for every CTA's partials; the others are done (every store into their
        // shared memory has landed: they waited for all of y)
        if (rank == 0) {
            if (!spin_wait_cluster(&cbar, 0u) && lane == 0)
                raise_flag(p.dev_err, DEVFLAG_TIMEOUT);
            v = lane < (int)CL ? cpart[lane][warp].x : -INFINITY;
            i = lane < (int)CL ? __float_as_int(cpart[lane][warp].y) : INT_MAX;
#pragma unroll
            for (int o = 16; o; o >>= 1)
                fold_max(v, i, __shfl_xor_sync(0xffffffffu, v, o), __shfl_xor_sync(0xffffffffu, i, o));
            if (lane == 0) {
                if (i == INT_MAX) {  // nothing allowed
                    i = 0;
                    v = -INFINITY;
                    raise_flag(p.dev_err, DEVFLAG_EMPTY_MASK);
                }
                p.out_idx[warp] = i;
                if (p.out_val) p.out_val[warp] = v;
            }
        }
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
    auto staged_bytes = [&](int clusters) -> size_t {
        const size_t rows_per = (size_t)(2 * ((h + 2 * clusters - 1) / (2 * clusters)));
        const size_t per = (size_t)((n + clusters - 1) / clusters);
        return ((rows_per * 2 * (size_t)h * 2 + 127) & ~(size_t)127) + per * (size_t)head_pitch(h);
    };
    constexpr size_t kStageLimit = 192 * 1024;  // beside ~26 KB of static shared memory
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // The cluster size of an instance: 16 CTAs where the device allows it, else the portable
    // 8 (the same for every head; queried once per instance and device).
    static int cl_cached[3][64] = {{0}};
    auto cluster_of = [&](int inst, void (*kern)(DraftParams), size_t smem) -> int {
        int cl = dev >= 0 && dev < 64 ? cl_cached[inst][dev] : 0;
        if (cl != 0) return cl;
        cl = 8;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
                cudaSuccess &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                cudaSuccess) {
            cudaLaunchConfig_t q{};
            q.gridDim = dim3(kDMaxCluster);
            q.blockDim = dim3(kDThreads);
            q.dynamicSmemBytes = smem;
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
        return cl;
    };
    // one input and a head slice of at most one 16-row tile per warp, h <= 256: the
    // register form; otherwise the staged form
    void (*kern)(DraftParams) = nullptr;
    int cl = 0;
    // (its norm weights are read as 16-byte pieces: both 16-byte aligned)
    const bool w16 = ((reinterpret_cast<uintptr_t>(w_ne) | reinterpret_cast<uintptr_t>(w_nh)) & 15u) == 0;
    if (M == 1 && h <= kResMaxH && w16) {
        cl = cluster_of(2, draft_step_kernel<1, true>, 0);
        if ((n + cl - 1) / cl <= kResMaxRowsPerCta) kern = draft_step_kernel<1, true>;
    }
    if (!kern) {
        kern = M == 1 ? draft_step_kernel<1, false> : draft_step_kernel<kDMaxM, false>;
        cl = cluster_of(M == 1 ? 0 : 1, kern, kStageLimit);
    }
    const bool res = kern == draft_step_kernel<1, true>;
    const size_t sb = res ? 0 : staged_bytes(cl);
    p.staged = !res && sb <= kStageLimit;
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
