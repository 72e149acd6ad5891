// Device helpers shared by the draft-head kernels (sm_100a only).
//
// Number formats: bf16 is the top half of an fp32; E4M3 is OCP E4M3FN (largest
// finite 448, no infinities); E2M1 is OCP FP4 ({0,.5,1,1.5,2,3,4,6} and sign).
// Conversions to the narrow formats use the hardware's round-to-nearest-even,
// saturating ("satfinite") converts; conversions from them are exact.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#ifndef __CUDACC_RTC__
#include <cstddef>
#endif

namespace mtp {

// ---------------------------------------------------------------- bf16 / fp32 bits
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

// fp32 -> bf16, round to nearest even (hardware convert).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

// Two fp32 -> bf16x2 (`lo` in bits 0..15), round to nearest even: one packed convert.
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// fp32 -> f16, round to nearest even.
__device__ __forceinline__ uint16_t f32_to_f16(float f) {
    uint16_t r;
    asm("cvt.rn.f16.f32 %0, %1;" : "=h"(r) : "f"(f));
    return r;
}

// ---------------------------------------------------------------- narrow formats
// Two fp32 -> two E4M3 codes; `lo` lands in bits 0..7, `hi` in bits 8..15.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two fp32 -> two E2M1 codes in one byte; `lo` in bits 0..3, `hi` in bits 4..7.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 q;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q, %1, %2;\n\t"
        "cvt.u32.u8 %0, q;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Exact decode of one E4M3 code to fp32 (used off the hot path).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    uint16_t c = (uint16_t)(code & 0xFF);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    float f;
    asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, lo;\n\t}"
        : "=f"(f) : "r"(h2));
    return f;
}

// Two E4M3 codes (bits 0..7 and 8..15) -> f16x2 (low half from bits 0..7). Exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
    return r;
}

// Eight E2M1 codes packed in a word (element 2j in the low nibble of byte j) ->
// four f16x2 registers, element order preserved (low half = lower element). Exact.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&o)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]) : "r"(w));
}

// Packed f16x2 multiply (round to nearest). Used only where the product is exact.
// f16x2 -> two floats (exact).
__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t v) {
    float2 r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "cvt.f32.f16 %0, lo;\n\t"
        "cvt.f32.f16 %1, hi;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "r"(v));
    return r;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// ---------------------------------------------------------------- tensor-core MMA
// D[16x8] += A[16x16] * B[16x8], fp32 accumulate. Fragment layout (lane = 4g + c):
//   A: a0 = (row g,   k 2c..2c+1), a1 = (row g+8, k 2c..2c+1),
//      a2 = (row g,   k 2c+8..+9), a3 = (row g+8, k 2c+8..+9)
//   B: b0 = (k 2c..2c+1, col g),   b1 = (k 2c+8..+9, col g)
//   D: d0,d1 = (row g, cols 2c, 2c+1), d2,d3 = (row g+8, cols 2c, 2c+1)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- memory
// Streaming 16-byte load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ldg_u16(const void* p) {
    unsigned short r;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 lds128(const void* p) {
    return *reinterpret_cast<const uint4*>(p);
}

// Release/acquire fence at GPU scope (orders this thread's memory accesses around a
// relaxed atomic used as a flag).
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Atomic add with release (earlier writes visible first) and acquire (later reads see
// what the releases before it published) semantics at GPU scope; returns the old value.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Programmatic dependent launch: let the next kernel in the stream start its prologue
// (it still waits for this grid before reading anything this grid may write), and wait
// for the previous grid to complete with its writes visible. Both are no-ops when the
// launch carries no programmatic-serialization attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Device error word bits (a copy of the public MTP_DEVFLAG_* values).
enum : int32_t { DEVFLAG_BAD_TOKEN = 1, DEVFLAG_EMPTY_MASK = 2, DEVFLAG_BAD_SLOT = 4,
                 DEVFLAG_TIMEOUT = 8 };

__device__ __forceinline__ void raise_flag(int32_t* dev_err, int32_t f) {
    if (dev_err) atomicOr(dev_err, f);
}

}  // namespace mtp

namespace mtp {

// ---------------------------------------------------------------- shared-memory sync
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// Makes initialised mbarriers visible to the async (TMA) proxy.
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Like mbar_try_wait, but the thread may sleep in hardware for up to `ns` nanoseconds
// waiting for the phase (no issue slots spent spinning).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// About one second at the B200's clock: a wait this long means the pipeline is broken.
constexpr long long kWaitLimitCycles = 2000000000LL;

// Waits for `bar` to complete the phase with `parity`, sleeping in hardware between
// checks. Gives up after kWaitLimitCycles -- or at once when *abort is already set --
// sets *abort and returns false; the caller then runs on without the data so that every
// thread still reaches the end of the kernel. With abort == nullptr only the time limit
// applies (used to drain copies in flight at exit).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort,
                                                  long long limit = kWaitLimitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 2000u)) return true;
        if (abort && *abort) return false;
        if (clock64() - t0 > limit) {
            if (abort) *abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* a) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
    return v;
}

// Waits until the global counter *a reaches `target` (GPU-scope acquire loads), sleeping
// between checks; gives up like mbar_wait_bounded (at once when *abort is set, or after
// `limit` cycles, setting *abort).
__device__ __forceinline__ bool counter_wait_bounded(const uint32_t* a, uint32_t target,
                                                     volatile int* abort,
                                                     long long limit = kWaitLimitCycles) {
    if (ld_acquire_gpu(a) >= target) return true;
    const long long t0 = clock64();
    while (true) {
        __nanosleep(500);
        if (ld_acquire_gpu(a) >= target) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            *abort = 1;
            return false;
        }
    }
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar` (no multicast).
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Pull `bytes` (a multiple of 16, 16-byte aligned) of global memory into L2, asynchronously.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster: release this CTA's shared-memory writes,
// acquire the others'.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// The address of this CTA's shared variable `p` in CTA `rank`'s shared memory.
__device__ __forceinline__ uint32_t map_rank(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Arrive on the mbarrier at shared::cluster address `addr` (this CTA's or another's of the
// cluster), releasing this thread's earlier writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
// mbar_wait_bounded with a cluster-scope acquire: for barriers that threads of other CTAs
// of the cluster arrive on, after writing what the waiter then reads.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity,
                                                          volatile int* abort,
                                                          long long limit = kWaitLimitCycles) {
    if (mbar_try_wait_cluster(bar, parity, 0u)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity, 2000u)) return true;
        if (abort && *abort) return false;
        if (clock64() - t0 > limit) {
            if (abort) *abort = 1;
            return false;
        }
    }
}

// Named barrier over the first `threads` threads of the CTA (id 1; id 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace mtp
