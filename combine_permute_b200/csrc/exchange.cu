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

}  // namespace

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
    return launch(ep_recv_layout_kernel, grid, kLayoutThreads, smem, stream, counts, R, El,
                  capacity, recv_offsets, local_offsets, recv_to_local, local_to_recv, num_recv);
}

}  // namespace moe
