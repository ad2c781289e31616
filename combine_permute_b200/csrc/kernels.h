// Internal launchers behind the C ABI (see include/moe.h for the contracts).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

enum class DType : int { F32 = 0, F16 = 1, BF16 = 2, FP8_E4M3 = 3 };

inline int dtype_bytes(DType d) {
    return d == DType::F32 ? 4 : (d == DType::FP8_E4M3 ? 1 : 2);
}

// Prepare: a problem with at most kSingleBlockSlots slots runs as one block;
// larger ones as tiles of kTileSlots slots over the whole GPU.
constexpr int kSingleBlockSlots = 4096;
constexpr int kTileSlots = 2048;  // slots per tile
constexpr int kMaxExperts = 1024;
constexpr int kFusedMaxSlots = 4096;
constexpr int kMaxEpGroups = 8192;  // ranks x local experts of one exchange layout

size_t prepare_workspace_bytes(int64_t S, int E);

// ids are int32 (ids64 false) or int64; slot i's expert is ids[i] - base when
// that lies in [0, E), else the slot is excluded like an invalid id.
cudaError_t run_prepare(const void *ids, bool ids64, int64_t base, int64_t S, int E, int A,
                        int32_t *counts, int32_t *offsets, int32_t *bso, int32_t *in_perm,
                        int32_t *out_perm, int32_t *diag, void *workspace, cudaStream_t stream);

cudaError_t run_prepare_dispatch(const int32_t *ids, int64_t T, int k, int E, int A,
                                 int32_t *counts, int32_t *offsets, int32_t *bso,
                                 int32_t *in_perm, int32_t *out_perm, int32_t *diag,
                                 const void *x, int64_t row_bytes, void *out,
                                 cudaStream_t stream);

cudaError_t run_dispatch_scatter(const void *x, int64_t T, int64_t row_bytes, int k,
                                 const int32_t *out_perm, void *out, cudaStream_t stream);

// The same with an explicit number of chunks per row (for tuning).
cudaError_t run_dispatch_scatter_split(const void *x, int64_t T, int64_t row_bytes, int k,
                                       const int32_t *out_perm, void *out, int64_t nsplit,
                                       cudaStream_t stream);

// Writes the bulk dispatch's error word (1: a bounded wait gave up since
// the last query) to *out and clears it.
cudaError_t run_dispatch_error(int32_t *out, cudaStream_t stream);

cudaError_t run_dispatch_gather(const void *x, int64_t T, int64_t row_bytes, int k,
                                const int32_t *in_perm, void *out, cudaStream_t stream);

cudaError_t run_dispatch_fp8(const void *x, DType x_dtype, int64_t T, int64_t H, int k, int E,
                             const int32_t *out_perm, const int32_t *offsets, const int32_t *bso,
                             uint8_t *q, float *scales, cudaStream_t stream);
// NVFP4 dispatch: E2M1 codes two per byte ([T*k, H/2]) and one E4M3 scale
// byte per 16 elements ([rows, H/16], rows placed by the block-scale offsets).
cudaError_t run_dispatch_nvfp4(const void *x, DType x_dtype, int64_t T, int64_t H, int k, int E,
                               const int32_t *out_perm, const int32_t *offsets, const int32_t *bso,
                               uint8_t *q, uint8_t *scales, cudaStream_t stream);

cudaError_t run_output_memset(void *out, int64_t T, int64_t row_bytes, int k,
                              const int32_t *out_perm, cudaStream_t stream);

cudaError_t run_combine(const void *y, DType y_dtype, int64_t T, int64_t H, int k,
                        const int32_t *out_perm, const float *w, void *out, DType out_dtype,
                        cudaStream_t stream);

cudaError_t run_problem_sizes(const int32_t *counts, int E, int n1, int k1, int n2, int k2,
                              int32_t *ps1, int32_t *ps2, cudaStream_t stream);

cudaError_t run_tile_layout(int64_t S, int E, int tile, const int32_t *counts,
                            const int32_t *offsets, const int32_t *out_perm, int max_tiles,
                            int32_t *padded_offsets, int32_t *tile_group, int32_t *tile_limit,
                            int32_t *exp2perm, int32_t *perm2exp, int32_t *num_tiles,
                            int32_t *total_padded, cudaStream_t stream);

// The fused exchange between GPUs: every slot's destination rank and row in
// the owners' grouped buffers (from all ranks' expert counts [R][E]), the
// dispatch that stores rows there (bufs: device array of R row pointers,
// nrows: rows of each buffer) and the combine that reads the expert outputs
// back from them.
cudaError_t run_ep_peer_layout(const int32_t *all_counts, int R, int rank, int E,
                               const int32_t *ids, int64_t S, const int32_t *offsets,
                               const int32_t *out_perm, int32_t *dest_rank, int32_t *dest_row,
                               int32_t *recv_rows, int32_t *local_offsets, cudaStream_t stream);
cudaError_t run_dispatch_peer(const void *x, int64_t T, int64_t row_bytes, int k,
                              const int32_t *dest_rank, const int32_t *dest_row,
                              void *const *bufs, const int32_t *nrows, int R, cudaStream_t stream);
cudaError_t run_combine_peer(const void *const *bufs, const int32_t *nrows, int R, DType y_dtype,
                             int64_t T, int64_t H, int k, const int32_t *dest_rank,
                             const int32_t *dest_row, const float *w, void *out, DType out_dtype,
                             cudaStream_t stream);

// Receiving rank's layout of the expert-parallel exchange: counts [R][El]
// -> recv_offsets [R+1], local_offsets [El+1], the two row maps (written when
// the number of received rows is at most `capacity`) and that number.
cudaError_t run_ep_recv_layout(const int32_t *counts, int R, int El, int64_t capacity,
                               int32_t *recv_offsets, int32_t *local_offsets,
                               int32_t *recv_to_local, int32_t *local_to_recv,
                               int32_t *num_recv, cudaStream_t stream);

}  // namespace moe
