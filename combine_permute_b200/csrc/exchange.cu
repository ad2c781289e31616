// The receiving rank's layout of the expert-parallel exchange between GPUs
// (Mooncake PR #4581: dispatch / combine across ranks; TensorRT-LLM PR
// #9592: all-to-all communication, one rank's experts being the window
// local_expert_offset .. + num_local_experts).
//
// R ranks each own El consecutive experts.  A source's dispatched rows are
// sorted by expert, so what it sends to this rank is one block ordered by
// local expert; the received buffer holds the source blocks in source
// order.  The expert stage wants the rows grouped by local expert, then
// source.  With c[s][le] the rows source s sends for local expert le, the
// (s, le) run starts at
//     qbase = row-major exclusive scan of c     (received buffer)
//     gbase = column-major exclusive scan of c  (grouped layout)
// and row m of the run is received row qbase + m = grouped row gbase + m.
// Every block stages c and both scans in shared memory; then one thread per
// received row finds its run by binary search over qbase (skipping empty
// runs) and writes both maps.
#include "kernels.h"
#include "launch.h"
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int kLayoutThreads = 1024;

__global__ void __launch_bounds__(kLayoutThreads)
    ep_recv_layout_kernel(const int32_t *__restrict__ counts, int R, int El, int64_t capacity,
                          int32_t *recv_offsets, int32_t *local_offsets, int32_t *recv_to_local,
                          int32_t *local_to_recv, int32_t *num_recv) {
    extern __shared__ int smem[];
    __shared__ int warp_tmp[66];
    const int n = R * El;
    int *qbase = smem;       // [n] row-major exclusive scan, indexed s * El + le
    int *gcol = qbase + n;   // [n] column-major exclusive scan, indexed le * R + s
    int *pad = gcol + n;     // [n] scan scratch
    pdl_wait();
    pdl_launch_dependents();
    for (int x = threadIdx.x; x < n; x += blockDim.x) {
        const int v = __ldg(counts + x);  // x = s * El + le
        qbase[x] = v;
        gcol[(x % El) * R + x / El] = v;
    }
    __syncthreads();
    int pad_total = 0;
    const int total = block_exclusive_scan2(qbase, pad, n, 1, warp_tmp, &pad_total);
    block_exclusive_scan2(gcol, pad, n, 1, warp_tmp, &pad_total);
    if (blockIdx.x == 0) {
        for (int s = threadIdx.x; s < R; s += blockDim.x) recv_offsets[s] = qbase[s * El];
        for (int le = threadIdx.x; le < El; le += blockDim.x) local_offsets[le] = gcol[le * R];
        if (threadIdx.x == 0) {
            recv_offsets[R] = total;
            local_offsets[El] = total;
            *num_recv = total;
        }
    }
    if ((int64_t)total > capacity) return;  // the caller learns the size from num_recv
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total; q += stride) {
        int lo = 0, hi = n - 1;  // the last run starting at or before q: never an empty one
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (qbase[mid] <= q) lo = mid;
            else hi = mid - 1;
        }
        const int s = lo / El, le = lo - s * El;
        const int64_t g = gcol[le * R + s] + (q - qbase[lo]);
        recv_to_local[q] = (int32_t)g;
        local_to_recv[g] = (int32_t)q;
    }
}

// Destinations of this rank's slots in the other ranks' grouped buffers
// (the fused exchange: every source stores its rows straight into the
// owners' buffers).  all[s * E + e] = rows source s holds for expert e.
// Per expert e of owner d = e / El:
//     colsum[e] = sum over sources of all[s][e]
//     gstart[e] = sum of colsum over the experts of d's window before e
//     base[e]   = gstart[e] + sum over sources s' < rank of all[s'][e]
// and slot i of expert e, dispatched here to row p, lands on row
// base[e] + (p - offsets[e]) of d's buffer.  Every block stages the matrix
// and the scans in shared memory; the grid walks the slots.
__global__ void __launch_bounds__(kLayoutThreads)
    ep_peer_layout_kernel(const int32_t *__restrict__ all, int R, int rank, int E,
                          const int32_t *__restrict__ ids, int64_t S,
                          const int32_t *__restrict__ offsets,
                          const int32_t *__restrict__ out_perm, int32_t *dest_rank,
                          int32_t *dest_row, int32_t *recv_rows, int32_t *local_offsets) {
    extern __shared__ int smem[];
    __shared__ int warp_tmp[66];
    const int El = E / R;
    int *gpre = smem;      // [E] global exclusive scan of the column sums
    int *before = gpre + E;  // [E] rows of sources before this rank
    int *pad = before + E;   // [E] scan scratch
    pdl_wait();
    pdl_launch_dependents();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int col = 0, pre = 0;
        for (int s = 0; s < R; ++s) {
            const int v = __ldg(all + (int64_t)s * E + e);
            col += v;
            pre += s < rank ? v : 0;
        }
        gpre[e] = col;
        before[e] = pre;
    }
    __syncthreads();
    int pad_total = 0;
    const int total = block_exclusive_scan2(gpre, pad, E, 1, warp_tmp, &pad_total);
    if (blockIdx.x == 0) {
        for (int d = threadIdx.x; d < R; d += blockDim.x)
            recv_rows[d] = (d + 1 < R ? gpre[(d + 1) * El] : total) - gpre[d * El];
        for (int le = threadIdx.x; le <= El; le += blockDim.x)
            local_offsets[le] = (rank * El + le < E ? gpre[rank * El + le] : total) -
                                gpre[rank * El];
    }
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < S; i += stride) {
        const int e = __ldg(ids + i);
        const int p = __ldg(out_perm + i);
        int r = -1, row = -1;
        if (e >= 0 && e < E && p >= 0) {
            const int d = e / El;
            r = d;
            row = gpre[e] - gpre[d * El] + before[e] + (p - __ldg(offsets + e));
        }
        dest_rank[i] = r;
        dest_row[i] = row;
    }
}

}  // namespace

cudaError_t run_ep_peer_layout(const int32_t *all_counts, int R, int rank, int E,
                               const int32_t *ids, int64_t S, const int32_t *offsets,
                               const int32_t *out_perm, int32_t *dest_rank, int32_t *dest_row,
                               int32_t *recv_rows, int32_t *local_offsets, cudaStream_t stream) {
    const size_t smem = (size_t)3 * E * sizeof(int);
    int64_t grid = (S + kLayoutThreads - 1) / kLayoutThreads;
    const int64_t cap = (int64_t)sm_count();
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return launch(ep_peer_layout_kernel, grid, kLayoutThreads, smem, stream, Start::kEarly,
                  all_counts, R, rank, E, ids, S, offsets, out_perm, dest_rank, dest_row, recv_rows,
                  local_offsets);
}

cudaError_t run_ep_recv_layout(const int32_t *counts, int R, int El, int64_t capacity,
                               int32_t *recv_offsets, int32_t *local_offsets,
                               int32_t *recv_to_local, int32_t *local_to_recv,
                               int32_t *num_recv, cudaStream_t stream) {
    const size_t smem = (size_t)3 * R * El * sizeof(int);
    // enough blocks for one received row per thread, at most one per SM
    // (each block redoes the scans; the row pass is what spreads)
    int64_t grid = (capacity + kLayoutThreads - 1) / kLayoutThreads;
    const int64_t cap = (int64_t)sm_count();
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return launch(ep_recv_layout_kernel, grid, kLayoutThreads, smem, stream, Start::kEarly, counts,
                  R, El, capacity, recv_offsets, local_offsets, recv_to_local, local_to_recv,
                  num_recv);
}

}  // namespace moe
