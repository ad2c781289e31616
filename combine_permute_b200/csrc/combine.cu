// Combine: gather the k expert-output rows of every token, scale each by its
// router weight and reduce in fp32 (sglang PR #19058, "Changes", item 3
// apply_shuffle_mul_sum: gather + scale + reduce, FP32 accumulation,
// fp16 / bf16 / fp32).
//
// A persistent grid-stride kernel over tokens.  Each thread owns one
// 16-byte column vector of the token row: it issues the loads of that
// vector from all k rows before consuming any of them (up to kBatch loads
// in flight), then accumulates in ascending slot order with separately
// rounded products and sums (__fmul_rn / __fadd_rn: no FMA contraction),
// and rounds once to the output type.
#include "kernels.h"
#include "launch.h"
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int kCombineThreads = 128;
constexpr int kBatch = 8;  // slots whose loads are in flight together

template <int N> struct Bytes;
template <> struct Bytes<8> {
    __device__ static void store(void *p, const void *src) {
        const uint2 v = *reinterpret_cast<const uint2 *>(src);
        asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
    }
};
template <> struct Bytes<16> {
    __device__ static void store(void *p, const void *src) {
        st_v4(p, *reinterpret_cast<const uint4 *>(src));
    }
};
template <> struct Bytes<32> {
    __device__ static void store(void *p, const void *src) {
        st_v4(p, *reinterpret_cast<const uint4 *>(src));
        st_v4((char *)p + 16, *(reinterpret_cast<const uint4 *>(src) + 1));
    }
};

template <typename YT, typename OT>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const YT *__restrict__ y, int64_t T, int64_t H, int k,
                   const int32_t *__restrict__ out_perm, const float *__restrict__ w,
                   OT *__restrict__ out) {
    constexpr int VE = 16 / sizeof(YT);  // elements per 16-byte load
    pdl_wait();
    pdl_launch_dependents();
    const int64_t nvec = H / VE;
    const int64_t S = T * k;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        const int32_t *rows = out_perm + t * k;
        const float *wt = w + t * k;
        for (int64_t c = threadIdx.x; c < nvec; c += kCombineThreads) {
            float acc[VE];
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[e] = 0.0f;
            for (int j0 = 0; j0 < k; j0 += kBatch) {
                uint4 v[kBatch];
                int p[kBatch];
#pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    p[b] = (j0 + b < k) ? __ldg(rows + j0 + b) : -1;
                    if (p[b] >= S) p[b] = -1;  // a corrupt entry contributes nothing
                    if (p[b] >= 0) v[b] = ld_stream_v4(y + (int64_t)p[b] * H + c * VE);
                }
#pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    if (p[b] < 0) continue;
                    const float wj = __ldg(wt + j0 + b);
                    const YT *h = reinterpret_cast<const YT *>(&v[b]);
#pragma unroll
                    for (int e = 0; e < VE; ++e)
                        acc[e] = __fadd_rn(acc[e], __fmul_rn(wj, Elem<YT>::to_f32(h[e])));
                }
            }
            OT o[VE];
#pragma unroll
            for (int e = 0; e < VE; ++e) o[e] = Elem<OT>::from_f32(acc[e]);
            Bytes<VE * sizeof(OT)>::store(out + t * H + c * VE, o);
        }
    }
}

template <typename YT, typename OT>
cudaError_t launch_combine(const void *y, int64_t T, int64_t H, int k, const int32_t *out_perm,
                           const float *w, void *out, cudaStream_t stream) {
    auto kern = combine_kernel<YT, OT>;
    const int64_t grid = persistent_grid(kern, kCombineThreads, 0, T);
    return launch(kern, grid, kCombineThreads, 0, stream, (const YT *)y, T, H, k, out_perm, w,
                  (OT *)out);
}

template <typename YT>
cudaError_t dispatch_out(DType out_dtype, const void *y, int64_t T, int64_t H, int k,
                         const int32_t *out_perm, const float *w, void *out, cudaStream_t stream) {
    switch (out_dtype) {
    case DType::F32: return launch_combine<YT, float>(y, T, H, k, out_perm, w, out, stream);
    case DType::F16: return launch_combine<YT, __half>(y, T, H, k, out_perm, w, out, stream);
    default: return launch_combine<YT, __nv_bfloat16>(y, T, H, k, out_perm, w, out, stream);
    }
}

}  // namespace

cudaError_t run_combine(const void *y, DType y_dtype, int64_t T, int64_t H, int k,
                        const int32_t *out_perm, const float *w, void *out, DType out_dtype,
                        cudaStream_t stream) {
    switch (y_dtype) {
    case DType::F32: return dispatch_out<float>(out_dtype, y, T, H, k, out_perm, w, out, stream);
    case DType::F16: return dispatch_out<__half>(out_dtype, y, T, H, k, out_perm, w, out, stream);
    default: return dispatch_out<__nv_bfloat16>(out_dtype, y, T, H, k, out_perm, w, out, stream);
    }
}

}  // namespace moe
