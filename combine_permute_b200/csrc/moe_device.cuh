// Device-side helpers shared by the sm_100a kernels of libmoe.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kWarp = 32;

// ---------------------------------------------------------------------------
// Programmatic dependent launch (PTX griddepcontrol, sm_90+).  Every kernel
// waits for its stream predecessor before touching global memory the
// predecessor may write or read, and lets its dependents launch before it
// ends: the short kernels (prepare, layouts) at their start, the streaming
// ones (dispatch, combine, gathers, memset) only after their work loop.
// Measured on B200: with the early signal, the next kernel's blocks sit on
// the SMs for the whole of a long streaming kernel and slowed the large
// workload's step by about 80 us in 1.3 ms; signalled after the loop, the
// next launch still overlaps the tail.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Memory access helpers.
// ---------------------------------------------------------------------------

// 16-byte read of data that stays constant for the whole kernel, not kept in
// L1 (each row is read once per block).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(void *p, const uint4 &v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void st_release_u32(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Atomic add with acquire-release semantics at GPU scope; returns the old value.
__device__ __forceinline__ unsigned atom_add_acq_rel_u32(unsigned *p, unsigned v) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
                 : "memory");
    return old;
}

// Atomic add with release semantics at GPU scope, no result.
__device__ __forceinline__ void red_add_release_u32(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Wrapping increment (atomicInc semantics) with acquire-release semantics.
__device__ __forceinline__ unsigned atom_inc_acq_rel_u32(unsigned *p, unsigned limit) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(limit)
                 : "memory");
    return old;
}

// Nanoseconds of the GPU's global timer: the clock behind every bounded wait.
__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ---------------------------------------------------------------------------
// Element conversions (CUDA intrinsics, round to nearest even).
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ static float to_f32(float v) { return v; }
    __device__ static float from_f32(float v) { return v; }
};
template <> struct Elem<__half> {
    __device__ static float to_f32(__half v) { return __half2float(v); }
    __device__ static __half from_f32(float v) { return __float2half_rn(v); }
};
template <> struct Elem<__nv_bfloat16> {
    __device__ static float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ static __nv_bfloat16 from_f32(float v) { return __float2bfloat16_rn(v); }
};

// Two fp32 values -> two OCP E4M3 bytes (round to nearest even, finite
// results saturate to +-448).  `lo` lands in the low byte.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// a / b rounded to nearest even, given rb = the correctly rounded 1/b
// (__frcp_rn(b), taken once per divisor).  Markstein's division (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): q0 = RN(a * rb) is within one
// ulp of a/b, the remainder a - q0*b is exact in one fma, and one fma
// correction RN(q0 + r*rb) is the correctly rounded quotient, provided that
// nothing underflows or overflows.  Callers keep b in [2^-60, 2^60] and
// only use the result where |a/b| >= 2^-12 matters; below that the result
// still has |value| < 2^-11 and the sign of a.  copysignf keeps the sign of
// a zero dividend (the fma chain turns -0 into +0).
__device__ __forceinline__ float div_rn_recip(float a, float b, float rb) {
    const float q0 = __fmul_rn(a, rb);
    const float r = __fmaf_rn(-q0, b, a);
    return copysignf(__fmaf_rn(r, rb, q0), a);
}

// Two fp32 values -> two FP4 E2M1 codes (round to nearest even, saturating
// to +-6), `lo` in bits 0..3 and `hi` in bits 4..7.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
        "cvt.u32.u8 %0, b;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// The value of an E4M3 byte, exactly, as fp32 (every E4M3 value is an fp16).
__device__ __forceinline__ float e4m3_to_f32(uint16_t byte) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(byte));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

// ---------------------------------------------------------------------------
// Two exclusive scans in one pass over n <= 32 * blockDim.x counts held in
// shared memory: a[] in place, and pad[] <- exclusive scan of a[] each
// rounded up to a multiple of A.  Returns the total of a; *pad_total gets
// the total of the rounded counts.  Needs blockDim.x a multiple of 32 and
// at most 1024; warp_tmp needs 66 ints.  All threads must call it.
__device__ __forceinline__ int block_exclusive_scan2(int *a, int *pad, int n, int A, int *warp_tmp,
                                                     int *pad_total) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int nw = nt >> 5;
    const int per = (n + nt - 1) / nt;
    const int beg = min(n, tid * per), end = min(n, beg + per);
    int la = 0, lp = 0;
    for (int i = beg; i < end; ++i) {
        la += a[i];
        lp += (a[i] + A - 1) / A * A;
    }
    int va = la, vp = lp;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ua = __shfl_up_sync(0xffffffffu, va, o);
        const int up = __shfl_up_sync(0xffffffffu, vp, o);
        if (lane >= o) {
            va += ua;
            vp += up;
        }
    }
    if (lane == 31) {
        warp_tmp[warp] = va;
        warp_tmp[33 + warp] = vp;
    }
    __syncthreads();
    int ba = 0, bp = 0, ta = 0, tp = 0;
    for (int w = 0; w < nw; ++w) {  // warp totals: a short broadcast read
        const int xa = warp_tmp[w], xp = warp_tmp[33 + w];
        if (w < warp) {
            ba += xa;
            bp += xp;
        }
        ta += xa;
        tp += xp;
    }
    int ra = va - la + ba, rp = vp - lp + bp;
    for (int i = beg; i < end; ++i) {
        const int c = a[i];
        a[i] = ra;
        pad[i] = rp;
        ra += c;
        rp += (c + A - 1) / A * A;
    }
    __syncthreads();
    *pad_total = tp;
    return ta;
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// Bulk asynchronous copies (TMA engine, non-tensor form) and mbarriers.
// All addresses are 16-byte aligned and sizes multiples of 16 bytes.  No
// cluster-wide form is used anywhere.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Bounded wait for the phase with parity `parity` of an mbarrier to
// complete.  Returns false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t max_polls) {
    const uint32_t a = smem_addr(bar);
    for (uint32_t i = 0; i < max_polls; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// global -> shared bulk copy completing on an mbarrier (transaction bytes)
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// shared -> global bulk copy, tracked by bulk async-groups
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_addr(src_smem)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed bulk groups still read shared memory.
template <int N> __device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group has completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace moe
