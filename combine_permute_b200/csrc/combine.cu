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

// Where the expert output of each slot is read.  LocalRows: row
// output_permutation[i] of this GPU's y.  PeerRows: the row each slot's
// destination rank holds in its grouped buffer (the fused exchange between
// GPUs; a buffer may be another GPU's memory mapped into this process, read
// with plain loads).  A slot without a valid row contributes nothing.  A
// slot's row is read in two steps, pre() (loads) and finish() (checks and
// the address); for PeerRows, whose checks need the rank's row count and
// buffer, a batch of up to kBatch slots issues all its loads before any
// check.
struct LocalRows {
    using Ref = int;
    using Pre = int;
    static constexpr bool kLocal = true;
    const char *y;
    const int32_t *perm;
    int64_t S, row_bytes;
    __device__ Pre pre(int64_t i) const { return __ldg(perm + i); }
    __device__ Ref finish(Pre p) const { return p >= 0 && p < S ? p : -1; }
    __device__ static Ref none() { return -1; }
    __device__ static bool valid(Ref r) { return r >= 0; }
    __device__ const char *addr(Ref r, int64_t coff) const {
        return y + (int64_t)r * row_bytes + coff;
    }
};

struct PeerRows {
    using Ref = const char *;
    using Pre = int2;  // (rank, row)
    static constexpr bool kLocal = false;
    const char *const *bufs;  // [R] each rank's grouped buffer of expert outputs
    const int32_t *rank;      // [S] destination rank of every slot (-1: none)
    const int32_t *row;       // [S] and its row there
    const int32_t *nrows;     // [R] rows of each buffer
    int R;
    int64_t row_bytes;
    __device__ Pre pre(int64_t i) const { return make_int2(__ldg(rank + i), __ldg(row + i)); }
    __device__ Ref finish(Pre v) const {
        if (v.x < 0 || v.x >= R) return nullptr;
        if (v.y < 0 || v.y >= __ldg(nrows + v.x)) return nullptr;
        return bufs[v.x] + (int64_t)v.y * row_bytes;
    }
    __device__ static Ref none() { return nullptr; }
    __device__ static bool valid(Ref r) { return r != nullptr; }
    __device__ const char *addr(Ref r, int64_t coff) const { return r + coff; }
};

// Rows and weights of slots j0 .. j0+kBatch-1 of one token (slot index
// `first` + j); a slot without a valid row gets weight 0 and is skipped.
template <bool kTwoStep, typename Rows>
__device__ __forceinline__ void load_batch(const Rows &rows, int64_t first, const float *wt, int j0,
                                           int k, typename Rows::Ref (&row)[kBatch],
                                           float (&wj)[kBatch]) {
    if constexpr (!kTwoStep) {
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            row[b] = (j0 + b < k) ? rows.finish(rows.pre(first + j0 + b)) : Rows::none();
            wj[b] = Rows::valid(row[b]) ? __ldg(wt + j0 + b) : 0.0f;
        }
    } else {
        // every slot's rank, row and weight loads first, then the checks
        // (measured: 2-3 % faster for peer rows, 0.5-1.5 % slower for local
        // ones; with k > kBatch it spills)
        typename Rows::Pre v[kBatch];
        float wv[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (j0 + b < k) {
                v[b] = rows.pre(first + j0 + b);
                wv[b] = __ldg(wt + j0 + b);
            }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            row[b] = (j0 + b < k) ? rows.finish(v[b]) : Rows::none();
            wj[b] = Rows::valid(row[b]) ? wv[b] : 0.0f;
        }
    }
}

// acc += w_j * y_j for one batch of slots, in slot order, at byte offset
// `coff` of the rows.
template <typename YT, int P, typename Rows>
__device__ __forceinline__ void accumulate_batch(f32x2 (&acc)[P], const Rows &rows,
                                                 const typename Rows::Ref (&row)[kBatch],
                                                 const float (&wj)[kBatch], int64_t coff) {
    uint4 v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
        if (Rows::valid(row[b])) v[b] = ld_stream_v4(rows.addr(row[b], coff));
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
        if (!Rows::valid(row[b])) continue;
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
// Resident blocks per SM the compiler must leave room for, for rows read from
// this GPU: eight for 16-bit expert outputs summed into fp32 (at most 64
// registers a thread), seven for the others (72); six for rows in other
// ranks' buffers.  The kernels the workloads use spill nothing.
template <typename YT, typename OT, typename Rows> constexpr int combine_min_blocks() {
    return !Rows::kLocal ? 6 : (sizeof(YT) == 2 && sizeof(OT) == 4 ? 8 : 7);
}

template <typename YT, typename OT, bool kSmallK, typename Rows>
__global__ void __launch_bounds__(kCombineThreads, combine_min_blocks<YT, OT, Rows>())
    combine_kernel(const Rows rows, int64_t T, int64_t H, int k, const float *__restrict__ w,
                   OT *__restrict__ out, int64_t nsplit, int64_t vpu) {
    constexpr int VE = 16 / sizeof(YT);    // elements per 16-byte load
    constexpr int P = Unpack<YT>::kPairs;  // fp32 pairs per load
    pdl_wait();
    const int64_t nvec = H / VE;
    const int64_t units = T * nsplit;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t t = u / nsplit;
        const int64_t cbeg = (u - t * nsplit) * vpu;
        const int64_t cend = min(nvec, cbeg + vpu);
        const float *wt = w + t * k;
        char *orow = reinterpret_cast<char *>(out + t * H);
        typename Rows::Ref row[kBatch];
        float wj[kBatch];
        if (kSmallK) load_batch<!Rows::kLocal>(rows, t * k, wt, 0, k, row, wj);
        for (int64_t c = cbeg + threadIdx.x; c < cend; c += kCombineThreads) {
            f32x2 acc[P];
#pragma unroll
            for (int i = 0; i < P; ++i) acc[i] = 0ull;  // +0.0f, +0.0f
            if (kSmallK) {
                accumulate_batch<YT, P>(acc, rows, row, wj, c * 16);
            } else {
                for (int j0 = 0; j0 < k; j0 += kBatch) {
                    load_batch<false>(rows, t * k, wt, j0, k, row, wj);
                    accumulate_batch<YT, P>(acc, rows, row, wj, c * 16);
                }
            }
            Store<OT, P>::run(orow + c * (int64_t)(VE * sizeof(OT)), acc);
        }
    }
    pdl_launch_dependents();  // after the work loop: see pdl_launch_dependents
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

template <typename YT, typename OT, typename Rows>
cudaError_t launch_combine(const Rows &rows, int64_t T, int64_t H, int k, const float *w,
                           void *out, int64_t nsplit, cudaStream_t stream) {
    auto kern =
        k <= kBatch ? combine_kernel<YT, OT, true, Rows> : combine_kernel<YT, OT, false, Rows>;
    const int64_t nvec = H / (16 / (int64_t)sizeof(YT));
    const int64_t grid_max = (int64_t)sm_count() * blocks_per_sm(kern, kCombineThreads, 0);
    if (nsplit <= 0) nsplit = combine_split(T, nvec, grid_max);
    const int64_t vpu = (nvec + nsplit - 1) / nsplit;
    const int64_t parts = (nvec + vpu - 1) / vpu;
    const int64_t grid = persistent_grid(kern, kCombineThreads, 0, T * parts);
    const Start start = streaming_start(T * k * H * (int64_t)sizeof(YT));
    return launch(kern, grid, kCombineThreads, 0, stream, start, rows, T, H, k, w, (OT *)out, parts,
                  vpu);
}

// The combine of element types (y_dtype, out_dtype) over rows made by
// make_rows(sizeof the y element).
template <typename MakeRows>
cudaError_t combine_typed(DType y_dtype, DType out_dtype, int64_t T, int64_t H, int k,
                          const float *w, void *out, int64_t nsplit, cudaStream_t stream,
                          MakeRows make_rows) {
    auto by_out = [&](auto yt) -> cudaError_t {
        using YT = decltype(yt);
        const auto rows = make_rows((int64_t)sizeof(YT));
        switch (out_dtype) {
        case DType::F32: return launch_combine<YT, float>(rows, T, H, k, w, out, nsplit, stream);
        case DType::F16: return launch_combine<YT, __half>(rows, T, H, k, w, out, nsplit, stream);
        default: return launch_combine<YT, __nv_bfloat16>(rows, T, H, k, w, out, nsplit, stream);
        }
    };
    switch (y_dtype) {
    case DType::F32: return by_out(float{});
    case DType::F16: return by_out(__half{});
    default: return by_out(__nv_bfloat16{});
    }
}

}  // namespace

cudaError_t run_combine_split(const void *y, DType y_dtype, int64_t T, int64_t H, int k,
                              const int32_t *out_perm, const float *w, void *out,
                              DType out_dtype, int64_t nsplit, cudaStream_t stream) {
    return combine_typed(y_dtype, out_dtype, T, H, k, w, out, nsplit, stream, [&](int64_t elt) {
        return LocalRows{(const char *)y, out_perm, T * k, H * elt};
    });
}

cudaError_t run_combine(const void *y, DType y_dtype, int64_t T, int64_t H, int k,
                        const int32_t *out_perm, const float *w, void *out, DType out_dtype,
                        cudaStream_t stream) {
    return run_combine_split(y, y_dtype, T, H, k, out_perm, w, out, out_dtype, 0, stream);
}

cudaError_t run_combine_peer(const void *const *bufs, const int32_t *nrows, int R, DType y_dtype,
                             int64_t T, int64_t H, int k, const int32_t *dest_rank,
                             const int32_t *dest_row, const float *w, void *out, DType out_dtype,
                             cudaStream_t stream) {
    return combine_typed(y_dtype, out_dtype, T, H, k, w, out, 0, stream, [&](int64_t elt) {
        return PeerRows{(const char *const *)bufs, dest_rank, dest_row, nrows, R, H * elt};
    });
}

}  // namespace moe
