// moe_prepare_no_alloc: moe_prepare for callers that cannot allocate device
// memory.  The scratch that the tiled prepare path needs (its look-back
// words) lives in a file-scope device array instead of a caller-provided
// workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "moe.h"

namespace moe {
moe_status_t status_from_cuda(cudaError_t e);  // capi.cu: records the error text
}

namespace {

constexpr size_t kScratchBytes = MOE_PREPARE_NO_ALLOC_SCRATCH_BYTES;

// One copy per GPU that loads the library, held until the process exits.
// In host code this name is only a host-side stand-in: kernels get the
// device address returned by cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_prepare_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // device address of g_prepare_scratch, per device

// Device address of the scratch array on the current device (with that
// device current).  Outside stream capture it is looked up on every call and
// the cache refreshed, so that a context torn down and created again (after
// cudaDeviceReset, say) never leaves a stale address behind; while a stream
// is being captured the cached address is used, since the first call on the
// device came before any capture.
cudaError_t scratch_address(int dev, cudaStream_t stream, void **out) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> g(g_mu);
    if (cap == cudaStreamCaptureStatusNone || g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_prepare_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" moe_status_t moe_prepare_no_alloc(const int32_t *topk_ids, int64_t num_tokens,
                                             int32_t top_k, int32_t num_experts,
                                             int32_t *expert_counts, int32_t *expert_offsets,
                                             int32_t *blockscale_offsets, int32_t blockscale_align,
                                             int32_t *input_permutation,
                                             int32_t *output_permutation, int32_t *diag,
                                             moe_stream_t stream) {
    if (num_tokens < 0 || top_k < 1 || num_experts < 1) return MOE_ERR_INVALID_ARG;
    if (num_tokens > 0 && num_tokens * (int64_t)top_k >= ((int64_t)1 << 31))
        return MOE_ERR_UNSUPPORTED;
    if (num_experts > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
    const int64_t S = num_tokens * (int64_t)top_k;
    if (!expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!topk_ids || !input_permutation || !output_permutation))
        return MOE_ERR_INVALID_ARG;
    if (blockscale_offsets && blockscale_align < 1) return MOE_ERR_INVALID_ARG;
    const size_t need = moe::prepare_workspace_bytes(S, num_experts);
    if (need > kScratchBytes) return MOE_ERR_UNSUPPORTED;  // larger than the static scratch

    void *scratch = nullptr;
    if (need > 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return moe::status_from_cuda(e);
        if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
        e = scratch_address(dev, (cudaStream_t)stream, &scratch);
        if (e != cudaSuccess) return moe::status_from_cuda(e);
        // the array keeps whatever the last call left: the look-back words
        // must start at zero
        e = cudaMemsetAsync(scratch, 0, need, (cudaStream_t)stream);
        if (e != cudaSuccess) return moe::status_from_cuda(e);
    }
    return moe::status_from_cuda(moe::run_prepare(
        topk_ids, false, 0, S, num_experts, blockscale_offsets ? blockscale_align : 1, expert_counts,
        expert_offsets, blockscale_offsets, input_permutation, output_permutation, diag, scratch,
        (cudaStream_t)stream));
}
