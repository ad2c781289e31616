// Combine: gather the k expert-output rows of every token, scale each by its
// router weight and reduce in fp32 (sglang PR #19058, "Changes", item 3
// apply_shuffle_mul_sum: gather + scale + reduce, FP32 accumulation,
// fp16 / bf16 / fp32).
//
// A persistent grid-stride kernel over tokens.  Per token every thread holds
// the k row indices and weights in registers; per 16-byte column vector it
// issues the loads from all k rows (kBatch at a time) before using any, then
// accumulates in ascending slot order with separately rounded products and
// sums (__fmul_rn / __fadd_rn, which the compiler never contracts into an
// FMA; the packed fp32-pair instructions were contracted and lost bit
// parity), and rounds once to the output type with packed conversions.
#include "kernels.h"
#include "launch.h"
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 128;
constexpr int kBatch = 8;  // slots whose loads are in flight together

typedef unsigned long long f32x2;  // two fp32 values, low word = first element

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
    return ((f32x2)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float lo_of(f32x2 v) { return __uint_as_float((unsigned)v); }
__device__ __forceinline__ float hi_of(f32x2 v) { return __uint_as_float((unsigned)(v >> 32)); }

// 16 bytes of the expert-output type as fp32 pairs (exact conversions).
template <typename YT> struct Unpack;
template <> struct Unpack<__nv_bfloat16> {
    static constexpr int kPairs = 4;
    __device__ static void run(const uint4 &v, f32x2 *out) {
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)  // a bf16 is the high half of its fp32
            out[i] = ((f32x2)(w[i] & 0xffff0000u) << 32) | (f32x2)(w[i] << 16);
    }
};
template <> struct Unpack<__half> {
    static constexpr int kPairs = 4;
    __device__ static void run(const uint4 &v, f32x2 *out) {
        const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            out[i] = pack2(f.x, f.y);
        }
    }
};
template <> struct Unpack<float> {
    static constexpr int kPairs = 2;
    __device__ static void run(const uint4 &v, f32x2 *out) {
        out[0] = ((f32x2)v.y << 32) | v.x;
        out[1] = ((f32x2)v.w << 32) | v.z;
    }
};

// fp32 pairs rounded (to nearest even) to the output type and stored.
template <typename OT, int P> struct Store;
template <int P> struct Store<__nv_bfloat16, P> {
    __device__ static void run(void *dst, const f32x2 *acc) {
        unsigned w[P];
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(lo_of(acc[i]), hi_of(acc[i]));
            w[i] = *reinterpret_cast<const unsigned *>(&h);
        }
        if (P == 4) st_v4(dst, make_uint4(w[0], w[1], w[2], w[P > 3 ? 3 : 0]));
        else asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(dst), "r"(w[0]), "r"(w[P > 1 ? 1 : 0]) : "memory");
    }
};
template <int P> struct Store<__half, P> {
    __device__ static void run(void *dst, const f32x2 *acc) {
        unsigned w[P];
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const __half2 h = __floats2half2_rn(lo_of(acc[i]), hi_of(acc[i]));
            w[i] = *reinterpret_cast<const unsigned *>(&h);
        }
        if (P == 4) st_v4(dst, make_uint4(w[0], w[1], w[2], w[P > 3 ? 3 : 0]));
        else asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(dst), "r"(w[0]), "r"(w[P > 1 ? 1 : 0]) : "memory");
    }
};
template <int P> struct Store<float, P> {
    __device__ static void run(void *dst, const f32x2 *acc) {
#pragma unroll
        for (int i = 0; i < P; i += 2)
            st_v4((char *)dst + 8 * i,
                  make_uint4((unsigned)acc[i], (unsigned)(acc[i] >> 32), (unsigned)acc[i + 1],
                             (unsigned)(acc[i + 1] >> 32)));
    }
};

// Row indices and weights of slots j0 .. j0+kBatch-1 of one token; an
// invalid or out-of-range slot gets row -1 and contributes nothing.
__device__ __forceinline__ void load_batch(int64_t S, const int32_t *rows, const float *wt, int j0,
                                           int k, int (&row)[kBatch], float (&wj)[kBatch]) {
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
        const int p = (j0 + b < k) ? __ldg(rows + j0 + b) : -1;
        row[b] = (p >= 0 && p < S) ? p : -1;
        wj[b] = row[b] >= 0 ? __ldg(wt + j0 + b) : 0.0f;
    }
}

// acc += w_j * y_j for one batch of slots, in slot order, at byte offset
// `coff` of the rows.
template <typename YT, int P>
__device__ __forceinline__ void accumulate_batch(f32x2 (&acc)[P], const char *y, int64_t row_bytes,
                                                 const int (&row)[kBatch],
                                                 const float (&wj)[kBatch], int64_t coff) {
    uint4 v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
        if (row[b] >= 0) v[b] = ld_stream_v4(y + (int64_t)row[b] * row_bytes + coff);
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
        if (row[b] < 0) continue;
        f32x2 yv[P];
        Unpack<YT>::run(v[b], yv);
#pragma unroll
        for (int i = 0; i < P; ++i) {
            const float lo = __fadd_rn(lo_of(acc[i]), __fmul_rn(wj[b], lo_of(yv[i])));
            const float hi = __fadd_rn(hi_of(acc[i]), __fmul_rn(wj[b], hi_of(yv[i])));
            acc[i] = pack2(lo, hi);
        }
    }
}

// Work unit: (token, part): part covers `vpu` consecutive 16-byte column
// vectors of the token's row; the host picks the split so that the units
// spread evenly over the persistent grid.  kSmallK: k <= kBatch, and every
// slot's row and weight stay in registers for the unit; otherwise they are
// re-read (L1) per column vector.
template <typename YT, typename OT, bool kSmallK>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const YT *__restrict__ y, int64_t T, int64_t H, int k,
                   const int32_t *__restrict__ out_perm, const float *__restrict__ w,
                   OT *__restrict__ out, int64_t nsplit, int64_t vpu) {
    constexpr int VE = 16 / sizeof(YT);    // elements per 16-byte load
    constexpr int P = Unpack<YT>::kPairs;  // fp32 pairs per load
    pdl_wait();
    pdl_launch_dependents();
    const int64_t nvec = H / VE;
    const int64_t S = T * k;
    const int64_t row_bytes = H * (int64_t)sizeof(YT);
    const char *yb = reinterpret_cast<const char *>(y);
    const int64_t units = T * nsplit;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t t = u / nsplit;
        const int64_t cbeg = (u - t * nsplit) * vpu;
        const int64_t cend = min(nvec, cbeg + vpu);
        const int32_t *rows = out_perm + t * k;
        const float *wt = w + t * k;
        char *orow = reinterpret_cast<char *>(out + t * H);
        int row[kBatch];
        float wj[kBatch];
        if (kSmallK) load_batch(S, rows, wt, 0, k, row, wj);
        for (int64_t c = cbeg + threadIdx.x; c < cend; c += kCombineThreads) {
            f32x2 acc[P];
#pragma unroll
            for (int i = 0; i < P; ++i) acc[i] = 0ull;  // +0.0f, +0.0f
            if (kSmallK) {
                accumulate_batch<YT, P>(acc, yb, row_bytes, row, wj, c * 16);
            } else {
                for (int j0 = 0; j0 < k; j0 += kBatch) {
                    load_batch(S, rows, wt, j0, k, row, wj);
                    accumulate_batch<YT, P>(acc, yb, row_bytes, row, wj, c * 16);
                }
            }
            Store<OT, P>::run(orow + c * (int64_t)(VE * sizeof(OT)), acc);
        }
    }
}

// Column split of the token rows: the number of parts that minimises
// (units per block) x (vectors per unit + a per-unit overhead).
inline int64_t combine_split(int64_t T, int64_t nvec, int64_t grid_max) {
    constexpr int64_t kUnitOverheadVectors = 32;
    int64_t best_n = 1, best_cost = -1;
    for (int64_t n = 1; n <= 16; ++n) {
        const int64_t vpu = (nvec + n - 1) / n;
        if (n > 1 && vpu < kCombineThreads) break;  // keep every thread busy
        const int64_t parts = (nvec + vpu - 1) / vpu;
        const int64_t units = T * parts;
        const int64_t grid = units < grid_max ? units : grid_max;
        const int64_t per = (units + grid - 1) / grid;
        const int64_t cost = per * (vpu + kUnitOverheadVectors);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best_n = n;
        }
    }
    return best_n;
}

template <typename YT, typename OT>
cudaError_t launch_combine(const void *y, int64_t T, int64_t H, int k, const int32_t *out_perm,
                           const float *w, void *out, int64_t nsplit, cudaStream_t stream) {
    auto kern = k <= kBatch ? combine_kernel<YT, OT, true> : combine_kernel<YT, OT, false>;
    const int64_t nvec = H / (16 / (int64_t)sizeof(YT));
    const int64_t grid_max = (int64_t)sm_count() * blocks_per_sm(kern, kCombineThreads, 0);
    if (nsplit <= 0) nsplit = combine_split(T, nvec, grid_max);
    const int64_t vpu = (nvec + nsplit - 1) / nsplit;
    const int64_t parts = (nvec + vpu - 1) / vpu;
    const int64_t grid = persistent_grid(kern, kCombineThreads, 0, T * parts);
    return launch(kern, grid, kCombineThreads, 0, stream, (const YT *)y, T, H, k, out_perm, w,
                  (OT *)out, parts, vpu);
}

template <typename YT>
cudaError_t dispatch_out(DType out_dtype, const void *y, int64_t T, int64_t H, int k,
                         const int32_t *out_perm, const float *w, void *out, int64_t nsplit,
                         cudaStream_t stream) {
    switch (out_dtype) {
    case DType::F32: return launch_combine<YT, float>(y, T, H, k, out_perm, w, out, nsplit, stream);
    case DType::F16: return launch_combine<YT, __half>(y, T, H, k, out_perm, w, out, nsplit, stream);
    default:
        return launch_combine<YT, __nv_bfloat16>(y, T, H, k, out_perm, w, out, nsplit, stream);
    }
}

}  // namespace

cudaError_t run_combine_split(const void *y, DType y_dtype, int64_t T, int64_t H, int k,
                              const int32_t *out_perm, const float *w, void *out,
                              DType out_dtype, int64_t nsplit, cudaStream_t stream) {
    switch (y_dtype) {
    case DType::F32:
        return dispatch_out<float>(out_dtype, y, T, H, k, out_perm, w, out, nsplit, stream);
    case DType::F16:
        return dispatch_out<__half>(out_dtype, y, T, H, k, out_perm, w, out, nsplit, stream);
    default:
        return dispatch_out<__nv_bfloat16>(out_dtype, y, T, H, k, out_perm, w, out, nsplit, stream);
    }
}

cudaError_t run_combine(const void *y, DType y_dtype, int64_t T, int64_t H, int k,
                        const int32_t *out_perm, const float *w, void *out, DType out_dtype,
                        cudaStream_t stream) {
    return run_combine_split(y, y_dtype, T, H, k, out_perm, w, out, out_dtype, 0, stream);
}

}  // namespace moe
