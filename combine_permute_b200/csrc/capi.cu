// extern "C" entry points of libmoe: host-side argument validation, then the
// launchers in prepare.cu / dispatch.cu / combine.cu.  Contracts are stated
// in include/moe.h.  No entry point allocates memory or synchronises.
#include <cuda_runtime.h>
#include <stdio.h>

#include "moe.h"
#include "kernels.h"
#include "launch.h"

namespace {

constexpr int64_t kMaxSlots = (int64_t)1 << 31;

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

inline bool io_dtype(moe_dtype_t d) { return d == MOE_F32 || d == MOE_F16 || d == MOE_BF16; }

// The CUDA error behind the calling thread's last MOE_ERR_CUDA.
thread_local cudaError_t t_last_cuda_error = cudaSuccess;
thread_local char t_last_error_text[256] = "no CUDA error";

inline moe_status_t from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    t_last_cuda_error = e;
    snprintf(t_last_error_text, sizeof t_last_error_text, "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return MOE_ERR_CUDA;
}

inline moe::DType dt(moe_dtype_t d) { return static_cast<moe::DType>(static_cast<int>(d)); }

// Checks shared by every call that takes (T, k).
inline moe_status_t check_tk(int64_t T, int32_t k) {
    if (T < 0 || k < 1) return MOE_ERR_INVALID_ARG;
    if (T > 0 && T * (int64_t)k >= kMaxSlots) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace

namespace moe {
// Status of a CUDA result, recording the error text like every entry point.
moe_status_t status_from_cuda(cudaError_t e) { return from_cuda(e); }
}  // namespace moe

extern "C" {

const char *moe_status_string(moe_status_t s) {
    switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: outside the supported sizes or types";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA launch or runtime call failed";
    }
    return "unknown moe_status_t";
}

int32_t moe_version(void) { return 10000; }

const char *moe_last_cuda_error(void) { return t_last_error_text; }

size_t moe_prepare_workspace_bytes(int64_t num_tokens, int32_t top_k, int32_t num_experts) {
    if (num_tokens < 0 || top_k < 1 || num_experts < 1) return 0;
    return moe::prepare_workspace_bytes(num_tokens * (int64_t)top_k, num_experts);
}

moe_status_t moe_prepare(const int32_t *topk_ids, int64_t num_tokens, int32_t top_k,
                         int32_t num_experts, int32_t *expert_counts, int32_t *expert_offsets,
                         int32_t *blockscale_offsets, int32_t blockscale_align,
                         int32_t *input_permutation, int32_t *output_permutation, int32_t *diag,
                         void *workspace, size_t workspace_bytes, moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (num_experts < 1) return MOE_ERR_INVALID_ARG;
    if (num_experts > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
    const int64_t S = num_tokens * (int64_t)top_k;
    if (!expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!topk_ids || !input_permutation || !output_permutation))
        return MOE_ERR_INVALID_ARG;
    if (blockscale_offsets && blockscale_align < 1) return MOE_ERR_INVALID_ARG;
    const size_t need = moe::prepare_workspace_bytes(S, num_experts);
    if (need > 0 && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)))
        return MOE_ERR_WORKSPACE;
    return from_cuda(moe::run_prepare(topk_ids, false, 0, S, num_experts,
                                      blockscale_offsets ? blockscale_align : 1, expert_counts,
                                      expert_offsets, blockscale_offsets, input_permutation,
                                      output_permutation, diag, workspace,
                                      (cudaStream_t)stream));
}

moe_status_t moe_prepare_local(const void *topk_ids, moe_index_t id_type, int64_t num_tokens,
                               int32_t top_k, int64_t local_expert_offset,
                               int32_t num_local_experts, int32_t *expert_counts,
                               int32_t *expert_offsets, int32_t *blockscale_offsets,
                               int32_t blockscale_align, int32_t *input_permutation,
                               int32_t *output_permutation, int32_t *diag, void *workspace,
                               size_t workspace_bytes, moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (id_type != MOE_I32 && id_type != MOE_I64) return MOE_ERR_INVALID_ARG;
    if (num_local_experts < 1) return MOE_ERR_INVALID_ARG;
    if (num_local_experts > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
    const int64_t S = num_tokens * (int64_t)top_k;
    if (!expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!topk_ids || !input_permutation || !output_permutation))
        return MOE_ERR_INVALID_ARG;
    if (blockscale_offsets && blockscale_align < 1) return MOE_ERR_INVALID_ARG;
    const size_t need = moe::prepare_workspace_bytes(S, num_local_experts);
    if (need > 0 && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)))
        return MOE_ERR_WORKSPACE;
    return from_cuda(moe::run_prepare(topk_ids, id_type == MOE_I64, local_expert_offset, S,
                                      num_local_experts, blockscale_offsets ? blockscale_align : 1,
                                      expert_counts, expert_offsets, blockscale_offsets,
                                      input_permutation, output_permutation, diag, workspace,
                                      (cudaStream_t)stream));
}

moe_status_t moe_output_memset(void *out, moe_dtype_t dtype, int64_t num_tokens, int64_t hidden,
                               int32_t top_k, const int32_t *output_permutation,
                               moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (!io_dtype(dtype) || hidden < 1) return MOE_ERR_INVALID_ARG;
    const int64_t row_bytes = hidden * moe::dtype_bytes(dt(dtype));
    if (row_bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (num_tokens == 0) return MOE_OK;
    if (!out || !output_permutation || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_output_memset(out, num_tokens, row_bytes, top_k, output_permutation,
                                            (cudaStream_t)stream));
}

moe_status_t moe_dispatch_rows(const void *x, moe_dtype_t dtype, int64_t num_tokens,
                               int64_t hidden, int32_t top_k, const int32_t *input_permutation,
                               const int32_t *output_permutation, void *out,
                               moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (!io_dtype(dtype) || hidden < 1) return MOE_ERR_INVALID_ARG;
    const int64_t row_bytes = hidden * moe::dtype_bytes(dt(dtype));
    if (row_bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (num_tokens == 0) return MOE_OK;
    if (!x || !out || (!input_permutation && !output_permutation)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if (output_permutation)
        return from_cuda(moe::run_dispatch_scatter(x, num_tokens, row_bytes, top_k,
                                                   output_permutation, out, (cudaStream_t)stream));
    return from_cuda(moe::run_dispatch_gather(x, num_tokens, row_bytes, top_k, input_permutation,
                                              out, (cudaStream_t)stream));
}

moe_status_t moe_dispatch_error(int32_t *error, moe_stream_t stream) {
    if (!error) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_dispatch_error(error, (cudaStream_t)stream));
}

moe_status_t moe_set_wait_limits(int64_t prepare_wait_us, int64_t dispatch_polls) {
    moe::prepare_wait_ns().store(prepare_wait_us < 0 ? moe::kDefaultPrepareWaitNs
                                                     : (uint64_t)prepare_wait_us * 1000ull);
    moe::dispatch_polls().store(dispatch_polls < 0 ? moe::kDefaultDispatchPolls
                                : dispatch_polls > 0xffffffffll ? 0xffffffffu
                                                                : (uint32_t)dispatch_polls);
    return MOE_OK;
}

moe_status_t moe_dispatch_rows_fp8(const void *x, moe_dtype_t x_dtype, int64_t num_tokens,
                                   int64_t hidden, int32_t top_k, int32_t num_experts,
                                   const int32_t *output_permutation,
                                   const int32_t *expert_offsets,
                                   const int32_t *blockscale_offsets, uint8_t *out_q,
                                   float *out_scales, moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (x_dtype != MOE_BF16 && x_dtype != MOE_F16) return MOE_ERR_UNSUPPORTED;
    if (hidden < 1 || hidden % 128 != 0 || num_experts < 1) return MOE_ERR_INVALID_ARG;
    if (num_experts > 4 * moe::kMaxExperts || top_k > 4096) return MOE_ERR_UNSUPPORTED;
    if (num_tokens == 0) return MOE_OK;
    if (!x || !output_permutation || !expert_offsets || !blockscale_offsets || !out_q ||
        !out_scales)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out_q) || ((uintptr_t)out_scales & 3u))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_dispatch_fp8(x, dt(x_dtype), num_tokens, hidden, top_k, num_experts,
                                           output_permutation, expert_offsets, blockscale_offsets,
                                           out_q, out_scales, (cudaStream_t)stream));
}

moe_status_t moe_dispatch_rows_nvfp4(const void *x, moe_dtype_t x_dtype, int64_t num_tokens,
                                     int64_t hidden, int32_t top_k, int32_t num_experts,
                                     const int32_t *output_permutation,
                                     const int32_t *expert_offsets,
                                     const int32_t *blockscale_offsets, uint8_t *out_q,
                                     uint8_t *out_scales, moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (x_dtype != MOE_BF16 && x_dtype != MOE_F16) return MOE_ERR_UNSUPPORTED;
    if (hidden < 1 || hidden % 16 != 0 || num_experts < 1) return MOE_ERR_INVALID_ARG;
    if (num_experts > 4 * moe::kMaxExperts || top_k > 4096) return MOE_ERR_UNSUPPORTED;
    if (num_tokens == 0) return MOE_OK;
    if (!x || !output_permutation || !expert_offsets || !blockscale_offsets || !out_q ||
        !out_scales)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || ((uintptr_t)out_q & 7u)) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_dispatch_nvfp4(x, dt(x_dtype), num_tokens, hidden, top_k,
                                             num_experts, output_permutation, expert_offsets,
                                             blockscale_offsets, out_q, out_scales,
                                             (cudaStream_t)stream));
}

moe_status_t moe_combine(const void *y, moe_dtype_t y_dtype, int64_t num_tokens, int64_t hidden,
                         int32_t top_k, const int32_t *output_permutation, const float *weights,
                         void *out, moe_dtype_t out_dtype, moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (!io_dtype(y_dtype) || !io_dtype(out_dtype) || hidden < 1) return MOE_ERR_INVALID_ARG;
    if ((hidden * moe::dtype_bytes(dt(y_dtype))) % 16 != 0 ||
        (hidden * moe::dtype_bytes(dt(out_dtype))) % 16 != 0)
        return MOE_ERR_INVALID_ARG;
    if (num_tokens == 0) return MOE_OK;
    if (!y || !output_permutation || !weights || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out) || ((uintptr_t)weights & 3u)) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_combine(y, dt(y_dtype), num_tokens, hidden, top_k,
                                      output_permutation, weights, out, dt(out_dtype),
                                      (cudaStream_t)stream));
}

moe_status_t moe_prepare_dispatch(const int32_t *topk_ids, int64_t num_tokens, int32_t top_k,
                                  int32_t num_experts, int32_t *expert_counts,
                                  int32_t *expert_offsets, int32_t *blockscale_offsets,
                                  int32_t blockscale_align, int32_t *input_permutation,
                                  int32_t *output_permutation, int32_t *diag, const void *x,
                                  moe_dtype_t dtype, int64_t hidden, void *out,
                                  moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (num_experts < 1 || !io_dtype(dtype) || hidden < 1) return MOE_ERR_INVALID_ARG;
    if (num_experts > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
    const int64_t S = num_tokens * (int64_t)top_k;
    if (S > moe::kFusedMaxSlots) return MOE_ERR_UNSUPPORTED;
    const int64_t row_bytes = hidden * moe::dtype_bytes(dt(dtype));
    if (row_bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (!expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if (blockscale_offsets && blockscale_align < 1) return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!topk_ids || !x || !out || !input_permutation || !output_permutation))
        return MOE_ERR_INVALID_ARG;
    if (num_tokens > 0 && (!aligned16(x) || !aligned16(out))) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_prepare_dispatch(
        topk_ids, num_tokens, top_k, num_experts, blockscale_offsets ? blockscale_align : 1,
        expert_counts, expert_offsets, blockscale_offsets, input_permutation, output_permutation,
        diag, x, row_bytes, out, (cudaStream_t)stream));
}

moe_status_t moe_problem_sizes(const int32_t *expert_counts, int32_t num_experts, int32_t n1,
                               int32_t k1, int32_t n2, int32_t k2, int32_t *problem_sizes1,
                               int32_t *problem_sizes2, moe_stream_t stream) {
    if (num_experts < 1 || !expert_counts || !problem_sizes1) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_problem_sizes(expert_counts, num_experts, n1, k1, n2, k2,
                                            problem_sizes1, problem_sizes2, (cudaStream_t)stream));
}

moe_status_t moe_tile_layout(int64_t num_tokens, int32_t top_k, int32_t num_experts,
                             int32_t tile_size, const int32_t *expert_counts,
                             const int32_t *expert_offsets, const int32_t *output_permutation,
                             int32_t max_tiles, int32_t *padded_offsets,
                             int32_t *tile_idx_to_group_idx, int32_t *tile_idx_to_mn_limit,
                             int32_t *expanded_idx_to_permuted_idx,
                             int32_t *permuted_idx_to_expanded_idx,
                             int32_t *num_non_exiting_tiles, int32_t *total_num_padded_tokens,
                             moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (num_experts < 1 || tile_size < 1 || max_tiles < 1) return MOE_ERR_INVALID_ARG;
    if (num_experts > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if ((int64_t)max_tiles * tile_size >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    const int64_t S = num_tokens * (int64_t)top_k;
    if (!expert_counts || !expert_offsets || !padded_offsets || !tile_idx_to_group_idx ||
        !tile_idx_to_mn_limit || !permuted_idx_to_expanded_idx || !num_non_exiting_tiles ||
        !total_num_padded_tokens)
        return MOE_ERR_INVALID_ARG;
    if (S > 0 && (!output_permutation || !expanded_idx_to_permuted_idx)) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_tile_layout(
        S, num_experts, tile_size, expert_counts, expert_offsets, output_permutation, max_tiles,
        padded_offsets, tile_idx_to_group_idx, tile_idx_to_mn_limit, expanded_idx_to_permuted_idx,
        permuted_idx_to_expanded_idx, num_non_exiting_tiles, total_num_padded_tokens,
        (cudaStream_t)stream));
}

moe_status_t moe_ep_recv_layout(const int32_t *recv_expert_counts, int32_t num_ranks,
                                int32_t num_local_experts, int64_t capacity,
                                int32_t *recv_offsets, int32_t *local_offsets,
                                int32_t *recv_to_local, int32_t *local_to_recv,
                                int32_t *num_recv, moe_stream_t stream) {
    if (num_ranks < 1 || num_local_experts < 1 || capacity < 0) return MOE_ERR_INVALID_ARG;
    if ((int64_t)num_ranks * num_local_experts > moe::kMaxEpGroups) return MOE_ERR_UNSUPPORTED;
    if (!recv_expert_counts || !recv_offsets || !local_offsets || !num_recv)
        return MOE_ERR_INVALID_ARG;
    if (capacity > 0 && (!recv_to_local || !local_to_recv)) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_ep_recv_layout(recv_expert_counts, num_ranks, num_local_experts,
                                             capacity, recv_offsets, local_offsets, recv_to_local,
                                             local_to_recv, num_recv, (cudaStream_t)stream));
}

moe_status_t moe_ep_peer_layout(const int32_t *all_expert_counts, int32_t num_ranks,
                                int32_t rank, int32_t num_experts, const int32_t *topk_ids,
                                int64_t num_tokens, int32_t top_k,
                                const int32_t *expert_offsets,
                                const int32_t *output_permutation, int32_t *dest_rank,
                                int32_t *dest_row, int32_t *recv_rows, int32_t *local_offsets,
                                moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (num_ranks < 1 || rank < 0 || rank >= num_ranks || num_experts < 1 ||
        num_experts % num_ranks != 0)
        return MOE_ERR_INVALID_ARG;
    if (num_experts > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if (!all_expert_counts || !expert_offsets || !recv_rows || !local_offsets)
        return MOE_ERR_INVALID_ARG;
    const int64_t S = num_tokens * (int64_t)top_k;
    if (S > 0 && (!topk_ids || !output_permutation || !dest_rank || !dest_row))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_ep_peer_layout(all_expert_counts, num_ranks, rank, num_experts,
                                             topk_ids, S, expert_offsets, output_permutation,
                                             dest_rank, dest_row, recv_rows, local_offsets,
                                             (cudaStream_t)stream));
}

moe_status_t moe_ep_dispatch_peer(const void *x, moe_dtype_t dtype, int64_t num_tokens,
                                  int64_t hidden, int32_t top_k, const int32_t *dest_rank,
                                  const int32_t *dest_row, void *const *recv_buffers,
                                  const int32_t *recv_rows, int32_t num_ranks,
                                  moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (!io_dtype(dtype) || hidden < 1 || num_ranks < 1) return MOE_ERR_INVALID_ARG;
    const int64_t row_bytes = hidden * moe::dtype_bytes(dt(dtype));
    if (row_bytes % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (num_tokens == 0) return MOE_OK;
    if (!x || !dest_rank || !dest_row || !recv_buffers || !recv_rows || !aligned16(x))
        return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_dispatch_peer(x, num_tokens, row_bytes, top_k, dest_rank, dest_row,
                                            recv_buffers, recv_rows, num_ranks,
                                            (cudaStream_t)stream));
}

moe_status_t moe_ep_combine_peer(const void *const *out_buffers, const int32_t *recv_rows,
                                 int32_t num_ranks, moe_dtype_t y_dtype, int64_t num_tokens,
                                 int64_t hidden, int32_t top_k, const int32_t *dest_rank,
                                 const int32_t *dest_row, const float *weights, void *out,
                                 moe_dtype_t out_dtype, moe_stream_t stream) {
    moe_status_t st = check_tk(num_tokens, top_k);
    if (st != MOE_OK) return st;
    if (!io_dtype(y_dtype) || !io_dtype(out_dtype) || hidden < 1 || num_ranks < 1)
        return MOE_ERR_INVALID_ARG;
    if ((hidden * moe::dtype_bytes(dt(y_dtype))) % 16 != 0 ||
        (hidden * moe::dtype_bytes(dt(out_dtype))) % 16 != 0)
        return MOE_ERR_INVALID_ARG;
    if (num_tokens == 0) return MOE_OK;
    if (!out_buffers || !recv_rows || !dest_rank || !dest_row || !weights || !out)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(out) || ((uintptr_t)weights & 3u)) return MOE_ERR_INVALID_ARG;
    return from_cuda(moe::run_combine_peer(out_buffers, recv_rows, num_ranks, dt(y_dtype),
                                           num_tokens, hidden, top_k, dest_rank, dest_row,
                                           weights, out, dt(out_dtype), (cudaStream_t)stream));
}

}  // extern "C"
