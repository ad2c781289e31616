// Grouped-GEMM metadata, the step after prepare: per-expert problem sizes
// (sglang PR #19058, "Changes", item 1: compute_problem_sizes_kernel fills
// problem_sizes1 / problem_sizes2) and the tile-padded layout that a tiled
// grouped GEMM consumes (TensorRT-LLM PR #9592, the moe_sort outputs
// tile_idx_to_group_idx, tile_idx_to_mn_limit, expanded_idx_to_permuted_idx,
// permuted_idx_to_expanded_idx, total_num_padded_tokens,
// num_non_exiting_tiles).
//
// tile_layout_kernel is one grid-stride pass: every block turns the E counts
// into padded offsets in shared memory (a block-wide scan of the counts
// rounded up to the tile), then the grid writes the tile owners and row
// limits, the padded row of every valid slot (its expert found from the
// expert offsets, so any id type or expert window works) and its inverse,
// and -1 on padding rows.  The valid rows and the padding rows are disjoint, so the
// writes never race.
#include "kernels.h"
#include "launch.h"
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int kLayoutThreads = 256;

__global__ void __launch_bounds__(kLayoutThreads)
    problem_sizes_kernel(const int32_t *__restrict__ counts, int E, int n1, int k1, int n2, int k2,
                         int32_t *ps1, int32_t *ps2) {
    pdl_wait();
    pdl_launch_dependents();
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
        const int c = __ldg(counts + e);
        ps1[3 * e + 0] = c;
        ps1[3 * e + 1] = n1;
        ps1[3 * e + 2] = k1;
        if (ps2) {
            ps2[3 * e + 0] = c;
            ps2[3 * e + 1] = n2;
            ps2[3 * e + 2] = k2;
        }
    }
}

// Expert whose padded row range [poff[e], poff[e+1]) holds `row`
// (0 <= row < poff[E]): the last e with poff[e] <= row.
__device__ __forceinline__ int owner_of(const int *poff, int E, int64_t row) {
    int lo = 0, hi = E;  // poff[lo] <= row < poff[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (poff[mid] <= row) lo = mid;
        else hi = mid;
    }
    return lo;
}

// The same search over the unpadded offsets (off[e] <= p < off[e] + cnt[e]).
__device__ __forceinline__ int owner_of_rows(const int *off, int E, int p) {
    int lo = 0, hi = E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= p) lo = mid;
        else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kLayoutThreads)
    tile_layout_kernel(int64_t S, int E, int tile,
                       const int32_t *__restrict__ counts, const int32_t *__restrict__ offsets,
                       const int32_t *__restrict__ out_perm, int max_tiles,
                       int32_t *padded_offsets, int32_t *tile_group, int32_t *tile_limit,
                       int32_t *exp2perm, int32_t *perm2exp, int32_t *num_tiles,
                       int32_t *total_padded) {
    extern __shared__ int smem[];
    __shared__ int warp_tmp[66];
    int *cnt = smem;           // [E]
    int *off = cnt + E;        // [E]
    int *tmp = off + E;        // [E] scratch
    int *poff = tmp + E;       // [E+1] padded offsets
    const int tid = threadIdx.x;
    pdl_wait();
    pdl_launch_dependents();
    for (int e = tid; e < E; e += kLayoutThreads) {
        cnt[e] = __ldg(counts + e);
        off[e] = __ldg(offsets + e);
        tmp[e] = cnt[e];
    }
    __syncthreads();
    int total = 0;
    block_exclusive_scan2(tmp, poff, E, tile, warp_tmp, &total);
    if (tid == 0) poff[E] = total;
    __syncthreads();
    const int64_t capacity = (int64_t)max_tiles * tile;
    const int ntiles = total / tile;
    if (blockIdx.x == 0) {
        for (int e = tid; e <= E; e += kLayoutThreads) padded_offsets[e] = poff[e];
        if (tid == 0) {
            *total_padded = total;
            *num_tiles = total > capacity ? -1 : ntiles;
        }
    }
    if (total > capacity) return;  // the same decision in every block

    const int64_t stride = (int64_t)gridDim.x * kLayoutThreads;
    const int64_t g = (int64_t)blockIdx.x * kLayoutThreads + tid;
    for (int64_t t = g; t < max_tiles; t += stride) {
        if (t < ntiles) {
            const int e = owner_of(poff, E, t * tile);
            tile_group[t] = e;
            tile_limit[t] = poff[e] + cnt[e];
        } else {
            tile_group[t] = -1;
            tile_limit[t] = -1;
        }
    }
    const int nvalid = E > 0 ? off[E - 1] + cnt[E - 1] : 0;
    for (int64_t i = g; i < S; i += stride) {
        const int p = __ldg(out_perm + i);
        int pp = -1;
        if (p >= 0 && p < nvalid) {  // the slot's expert owns dispatched row p
            const int e = owner_of_rows(off, E, p);
            pp = poff[e] + (p - off[e]);
            if (pp >= 0 && pp < capacity) perm2exp[pp] = (int)i;
        }
        exp2perm[i] = pp;
    }
    for (int64_t q = g; q < capacity; q += stride) {
        bool padding = q >= total;
        if (!padding) {
            const int e = owner_of(poff, E, q);
            padding = q - poff[e] >= cnt[e];
        }
        if (padding) perm2exp[q] = -1;
    }
}

}  // namespace

cudaError_t run_problem_sizes(const int32_t *counts, int E, int n1, int k1, int n2, int k2,
                              int32_t *ps1, int32_t *ps2, cudaStream_t stream) {
    const int64_t grid = (E + kLayoutThreads - 1) / kLayoutThreads;
    return launch(problem_sizes_kernel, grid, kLayoutThreads, 0, stream, Start::kEarly, counts, E,
                  n1, k1, n2, k2, ps1, ps2);
}

cudaError_t run_tile_layout(int64_t S, int E, int tile, const int32_t *counts,
                            const int32_t *offsets, const int32_t *out_perm, int max_tiles,
                            int32_t *padded_offsets, int32_t *tile_group, int32_t *tile_limit,
                            int32_t *exp2perm, int32_t *perm2exp, int32_t *num_tiles,
                            int32_t *total_padded, cudaStream_t stream) {
    const size_t smem = (size_t)(4 * E + 1) * sizeof(int);
    int64_t work = (int64_t)max_tiles * tile;
    if (S > work) work = S;
    const int64_t grid =
        persistent_grid(tile_layout_kernel, kLayoutThreads, smem, (work + kLayoutThreads - 1) / kLayoutThreads);
    return launch(tile_layout_kernel, grid, kLayoutThreads, smem, stream, Start::kEarly, S, E, tile,
                  counts, offsets, out_perm, max_tiles, padded_offsets, tile_group, tile_limit,
                  exp2perm, perm2exp, num_tiles, total_padded);
}

}  // namespace moe
