// Routing metadata: a deterministic stable counting sort of the T*k slots by
// expert id (sglang PR #19058, "Changes", item 1 prepare_moe_input: tokens
// per expert, prefix-sum expert offsets, optional FP8 block-scale offsets,
// input / output permutations).
//
// Three paths by problem size:
//  * up to kSingleBlockSlots slots: one block (prep_single_kernel);
//  * up to kClusterMaxSlots: one thread-block cluster that exchanges its
//    blocks' histograms through distributed shared memory
//    (prep_cluster_kernel, described where it is defined);
//  * above that, tiles of kPrepTile slots in two kernels:
//   prep_count_kernel    per-tile shared-memory histogram (warp-aggregated
//                        with __match_any_sync), then a decoupled look-back
//                        across tiles, one column per expert (plus one for
//                        invalid ids), giving every tile the number of
//                        earlier slots of each expert.  The last tile holds
//                        the totals and writes counts, expert offsets and
//                        block-scale offsets (block-wide scans).
//   prep_scatter_kernel  re-reads its tile, ranks every slot among the
//                        earlier slots of the same expert (warp match +
//                        popcount within a round, per-warp running counters
//                        in shared memory, exclusive scan over warps), and
//                        writes both permutations.
// Tiles take their index from an atomic ticket, so every tile a block waits
// on has already been scheduled; each wait is bounded and reports through
// diag[1] instead of hanging.  The ticket counter wraps to zero and the
// scatter kernel clears the look-back words, leaving the workspace zeroed.
//
// Only the tiled path uses the workspace.
#include <cooperative_groups.h>

#include "kernels.h"
#include "launch.h"
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr unsigned long long kFlagAgg = 1ull << 32;
constexpr unsigned long long kFlagIncl = 2ull << 32;
constexpr int kMaxSpins = 1 << 20;  // x ~256 ns sleep: the wait gives up after ~0.3-1 s

struct PrepWs {
    unsigned *ticket;
    unsigned *timeout;
    unsigned long long *state;  // [G][E+1] look-back words: flag << 32 | value
    int *prefix;                // [G][E+1] exclusive tile prefix per column
};

__host__ __device__ inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

__host__ __device__ inline PrepWs carve(void *ws, int G, int C) {
    char *b = (char *)ws;
    PrepWs w;
    w.ticket = (unsigned *)b;
    w.timeout = (unsigned *)(b + 4);
    w.state = (unsigned long long *)(b + 256);
    w.prefix = (int *)(b + 256 + align256((size_t)G * C * 8));
    return w;
}

// Ranks the kWarpChunk slots starting at `wbase` that belong to this warp.
// For round r, e_r[r] is the slot's expert (-1 when invalid or past S) and
// rank_r[r] the number of earlier slots of the chunk with the same expert.
// Leaves the chunk's per-expert counts in wcnt_row (zeroed by the caller).
__device__ __forceinline__ void warp_rank_chunk(const int32_t *__restrict__ ids, int64_t S, int E,
                                                int64_t wbase, int *wcnt_row,
                                                int (&e_r)[kPrepRounds],
                                                int (&rank_r)[kPrepRounds]) {
    const int lane = threadIdx.x & 31;
    const unsigned lt = lanemask_lt();
#pragma unroll
    for (int r = 0; r < kPrepRounds; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        int e = -1;
        if (i < S) {
            const int id = __ldg(ids + i);
            e = (id >= 0 && id < E) ? id : -1;
        }
        e_r[r] = e;
    }
#pragma unroll
    for (int r = 0; r < kPrepRounds; ++r) {
        const int e = e_r[r];
        const unsigned grp = __match_any_sync(0xffffffffu, e);
        const int prior = e >= 0 ? wcnt_row[e] : 0;
        rank_r[r] = prior + __popc(grp & lt);
        __syncwarp();
        if (e >= 0 && (grp & lt) == 0) wcnt_row[e] = prior + __popc(grp);
        __syncwarp();
    }
}

// Whole problem in one block: ranks, totals, offsets, permutations.  When
// `pos` is non-null the dispatched row of every slot is also left there
// (shared memory, S entries).  Global outputs are written only when
// `write_global` is set.
__device__ __forceinline__ void single_block_prepare(const int32_t *__restrict__ ids, int64_t S,
                                                     int E, int A, int *smem, int *pos,
                                                     bool write_global, int32_t *counts,
                                                     int32_t *offsets, int32_t *bso,
                                                     int32_t *in_perm, int32_t *out_perm,
                                                     int32_t *diag) {
    __shared__ int warp_tmp[33];
    __shared__ int s_invalid;
    int *wcnt = smem;                   // [kPrepWarps][E]
    int *off = wcnt + kPrepWarps * E;   // [E+1]
    int *pad = off + (E + 1);           // [E+1]
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;

    for (int x = tid; x < kPrepWarps * E; x += nt) wcnt[x] = 0;
    if (tid == 0) s_invalid = 0;
    __syncthreads();

    int e_r[kPrepRounds], rank_r[kPrepRounds];
    const int64_t wbase = (int64_t)warp * kWarpChunk;
    warp_rank_chunk(ids, S, E, wbase, wcnt + warp * E, e_r, rank_r);
    int bad = 0;
#pragma unroll
    for (int r = 0; r < kPrepRounds; ++r) bad += (wbase + r * 32 + lane < S) && e_r[r] < 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
    if (lane == 0 && bad) atomicAdd(&s_invalid, bad);
    __syncthreads();

    // exclusive scan over warps for every expert; the total is the count
    for (int e = tid; e < E; e += nt) {
        int run = 0;
        for (int w = 0; w < kPrepWarps; ++w) {
            const int c = wcnt[w * E + e];
            wcnt[w * E + e] = run;
            run += c;
        }
        off[e] = run;
        pad[e] = (run + A - 1) / A * A;
    }
    __syncthreads();
    const int total = block_exclusive_scan(off, E, warp_tmp);
    int pad_total = 0;
    if (bso) pad_total = block_exclusive_scan(pad, E, warp_tmp);
    if (write_global) {
        for (int e = tid; e < E; e += nt) {
            const int next = e + 1 < E ? off[e + 1] : total;
            counts[e] = next - off[e];
            offsets[e] = off[e];
            if (bso) bso[e] = pad[e];
        }
        if (tid == 0) {
            offsets[E] = total;
            if (bso) bso[E] = pad_total;
            if (diag) {
                diag[0] = s_invalid;
                diag[1] = 0;
            }
        }
    }
    for (int x = tid; x < kPrepWarps * E; x += nt) wcnt[x] += off[x % E];
    __syncthreads();

#pragma unroll
    for (int r = 0; r < kPrepRounds; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        if (i < S) {
            const int e = e_r[r];
            const int p = e >= 0 ? wcnt[warp * E + e] + rank_r[r] : -1;
            if (pos) pos[i] = p;
            if (write_global) {
                out_perm[i] = p;
                if (p >= 0) in_perm[p] = (int)i;
            }
        }
    }
    if (write_global)
        for (int64_t p = total + tid; p < S; p += nt) in_perm[p] = -1;
}

__global__ void __launch_bounds__(kPrepThreads)
    prep_single_kernel(const int32_t *__restrict__ ids, int64_t S, int E, int A, int32_t *counts,
                       int32_t *offsets, int32_t *bso, int32_t *in_perm, int32_t *out_perm,
                       int32_t *diag) {
    extern __shared__ int smem[];
    pdl_wait();
    pdl_launch_dependents();
    single_block_prepare(ids, S, E, A, smem, nullptr, true, counts, offsets, bso, in_perm,
                         out_perm, diag);
}

__global__ void __launch_bounds__(kPrepThreads)
    prep_count_kernel(const int32_t *__restrict__ ids, int64_t S, int E, int A, int G,
                      void *workspace, int32_t *counts, int32_t *offsets, int32_t *bso,
                      int32_t *diag) {
    extern __shared__ int smem[];
    __shared__ int warp_tmp[33];
    __shared__ unsigned s_ticket;
    const int C = E + 1;  // one column per expert plus one for invalid ids
    int *hist = smem;     // [C]
    int *tot = hist + C;  // [C] totals (last tile only)
    int *pad = tot + C;   // [C]
    const int tid = threadIdx.x, nt = blockDim.x;
    PrepWs ws = carve(workspace, G, C);

    pdl_wait();
    pdl_launch_dependents();
    for (int c = tid; c < C; c += nt) hist[c] = 0;
    if (tid == 0) {
        unsigned t = atomicInc(ws.ticket, (unsigned)(G - 1));
        // a counter left non-zero by an aborted call: stay in bounds; the
        // bounded waits below then report the failure through diag[1]
        s_ticket = t < (unsigned)G ? t : t % (unsigned)G;
    }
    __syncthreads();
    const int tile = (int)s_ticket;
    const int64_t base = (int64_t)tile * kPrepTile;

    // 1. histogram of this tile (warp-aggregated shared-memory atomics)
    {
        int e_r[kPrepRounds];
#pragma unroll
        for (int r = 0; r < kPrepRounds; ++r) {
            const int64_t i = base + r * nt + tid;
            int e = -1;
            if (i < S) {
                const int id = __ldg(ids + i);
                e = (id >= 0 && id < E) ? id : E;
            }
            e_r[r] = e;
        }
        const unsigned lt = lanemask_lt();
#pragma unroll
        for (int r = 0; r < kPrepRounds; ++r) {
            const unsigned grp = __match_any_sync(0xffffffffu, e_r[r]);
            if (e_r[r] >= 0 && (grp & lt) == 0) atomicAdd(&hist[e_r[r]], __popc(grp));
        }
    }
    __syncthreads();

    // 2. publish this tile's aggregates
    unsigned long long *row = ws.state + (size_t)tile * C;
    for (int c = tid; c < C; c += nt) st_relaxed_u64(row + c, kFlagAgg | (unsigned)hist[c]);

    // 3. decoupled look-back, one column per thread
    bool gave_up = false;
    for (int c = tid; c < C; c += nt) {
        int excl = 0;
        for (int pred = tile - 1; pred >= 0 && !gave_up; --pred) {
            const unsigned long long *wp = ws.state + (size_t)pred * C + c;
            unsigned long long v = ld_relaxed_u64(wp);
            int spins = 0;
            while ((v >> 32) == 0) {
                if (++spins > kMaxSpins) {
                    gave_up = true;
                    break;
                }
                __nanosleep(256);
                v = ld_relaxed_u64(wp);
            }
            excl += (int)(unsigned)(v & 0xffffffffu);
            if ((v & kFlagIncl) != 0) break;
        }
        // publish even after giving up, so that no later tile waits on us
        st_relaxed_u64(row + c, kFlagIncl | (unsigned)(excl + hist[c]));
        ws.prefix[(size_t)tile * C + c] = excl;
        tot[c] = excl + hist[c];
    }
    if (gave_up) atomicExch(ws.timeout, 1u);

    // 4. the last tile holds the totals: counts, offsets, block-scale offsets
    if (tile != G - 1) return;
    __syncthreads();
    for (int e = tid; e < E; e += nt) pad[e] = (tot[e] + A - 1) / A * A;
    for (int e = tid; e < E; e += nt) counts[e] = tot[e];
    if (tid == 0 && diag) diag[0] = tot[E];
    __syncthreads();
    const int total = block_exclusive_scan(tot, E, warp_tmp);
    for (int e = tid; e < E; e += nt) offsets[e] = tot[e];
    if (tid == 0) offsets[E] = total;
    if (bso) {
        const int pad_total = block_exclusive_scan(pad, E, warp_tmp);
        for (int e = tid; e < E; e += nt) bso[e] = pad[e];
        if (tid == 0) bso[E] = pad_total;
    }
}

__global__ void __launch_bounds__(kPrepThreads)
    prep_scatter_kernel(const int32_t *__restrict__ ids, int64_t S, int E, int G, void *workspace,
                        const int32_t *offsets, int32_t *in_perm, int32_t *out_perm,
                        int32_t *diag) {
    extern __shared__ int smem[];
    const int C = E + 1;
    int *wcnt = smem;  // [kPrepWarps][E]
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int tile = blockIdx.x;
    const int64_t base = (int64_t)tile * kPrepTile;
    PrepWs ws = carve(workspace, G, C);

    pdl_wait();
    pdl_launch_dependents();
    for (int x = tid; x < kPrepWarps * E; x += nt) wcnt[x] = 0;
    __syncthreads();

    int e_r[kPrepRounds], rank_r[kPrepRounds];
    const int64_t wbase = base + (int64_t)warp * kWarpChunk;
    warp_rank_chunk(ids, S, E, wbase, wcnt + warp * E, e_r, rank_r);
    __syncthreads();

    for (int e = tid; e < E; e += nt) {
        int run = __ldg(offsets + e) + ws.prefix[(size_t)tile * C + e];
        ws.prefix[(size_t)tile * C + e] = 0;  // the workspace is all-zero between calls
        for (int w = 0; w < kPrepWarps; ++w) {
            const int c = wcnt[w * E + e];
            wcnt[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();

#pragma unroll
    for (int r = 0; r < kPrepRounds; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        if (i < S) {
            const int e = e_r[r];
            if (e >= 0) {
                const int p = wcnt[warp * E + e] + rank_r[r];
                out_perm[i] = p;
                if (p >= 0 && p < S) in_perm[p] = (int)i;
            } else {
                out_perm[i] = -1;
            }
        }
    }
    // input_permutation entries past the valid rows, within this tile's range
    const int64_t valid = __ldg(offsets + E);
    const int64_t lo = base > valid ? base : valid;
    const int64_t hi = base + kPrepTile < S ? base + kPrepTile : S;
    for (int64_t p = lo + tid; p < hi; p += nt) in_perm[p] = -1;

    // leave the workspace zeroed for the next call (its layout depends on the
    // problem size, so every byte this call used must return to zero)
    for (int c = tid; c < C; c += nt) ws.state[(size_t)tile * C + c] = 0ull;
    if (tid == 0) ws.prefix[(size_t)tile * C + E] = 0;
    if (tile == 0 && tid == 0) {
        if (diag) diag[1] = *ws.timeout ? 1 : 0;
        *ws.timeout = 0u;
    }
}

// ---------------------------------------------------------------------------
// Mid-size batches: the whole sort in ONE thread-block cluster (up to 16
// blocks, one per SM).  Every warp owns a contiguous run of slots.
//   pass 1  each warp counts its run per expert (warp-private shared-memory
//           row, ballot-based match); the block folds its warps into a
//           per-expert histogram.
//   cluster barrier; every block reads all blocks' histograms through
//           distributed shared memory: totals and the prefix of earlier
//           blocks, then a block-wide scan gives the expert offsets.
//   pass 2  each warp re-reads its run (now in L2) and ranks every slot:
//           offset + earlier blocks + earlier warps + earlier lanes.
// One launch, no global workspace, and the only waits are hardware cluster
// barriers.
// ---------------------------------------------------------------------------
constexpr int kClusterThreads = 1024;
constexpr int kClusterWarps = kClusterThreads / 32;
constexpr int kClusterBatch = 8;  // rounds of 32 slots whose loads are in flight together

// Lanes holding the same key (keys < 2^nbits): a match built from nbits
// ballots.
__device__ __forceinline__ unsigned match_by_ballot(unsigned key, int nbits) {
    unsigned m = 0xffffffffu;
    for (int b = 0; b < nbits; ++b) {
        const unsigned bit = (key >> b) & 1u;
        const unsigned vote = __ballot_sync(0xffffffffu, bit);
        m &= bit ? vote : ~vote;
    }
    return m;
}

// Threads per expert when folding the per-warp counts: a power of two that
// divides the warp count and keeps every thread busy for small E.
__device__ __forceinline__ int fold_parts(int E) {
    int parts = 1;
    while (parts < kClusterWarps && parts * 2 * E <= kClusterThreads) parts *= 2;
    return parts;
}

__global__ void __launch_bounds__(kClusterThreads, 1)
    prep_cluster_kernel(const int32_t *__restrict__ ids, int64_t S, int E, int A, int nbits,
                        int64_t wch, int32_t *counts, int32_t *offsets, int32_t *bso,
                        int32_t *in_perm, int32_t *out_perm, int32_t *diag) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int nc = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    extern __shared__ int smem[];
    __shared__ int warp_tmp[33];
    __shared__ int s_invalid;
    int *wcnt = smem;                          // [kClusterWarps][E]
    int *hist = wcnt + kClusterWarps * E;      // [E+1]: per expert, then invalid ids
    int *tot = hist + (E + 1);                 // [E+1]
    int *pre = tot + (E + 1);                  // [E]
    int *pad = pre + E;                        // [E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = lanemask_lt();
    const unsigned key_invalid = (unsigned)E;

    for (int x = tid; x < kClusterWarps * E; x += kClusterThreads) wcnt[x] = 0;
    if (tid == 0) s_invalid = 0;
    pdl_wait();
    pdl_launch_dependents();
    __syncthreads();

    const int64_t beg = ((int64_t)c * kClusterWarps + warp) * wch;
    const int64_t end = min(S, beg + wch);
    int *row = wcnt + warp * E;

    // pass 1: per-warp counts
    int bad = 0;
    for (int64_t r0 = beg; r0 < end; r0 += 32 * kClusterBatch) {
        int key[kClusterBatch];
#pragma unroll
        for (int b = 0; b < kClusterBatch; ++b) {
            const int64_t i = r0 + b * 32 + lane;
            int k2 = -2;  // past the run
            if (i < end) {
                const int id = __ldg(ids + i);
                k2 = (id >= 0 && id < E) ? id : -1;
            }
            key[b] = k2;
        }
#pragma unroll
        for (int b = 0; b < kClusterBatch; ++b) {
            if (r0 + b * 32 >= end) break;  // warp-uniform
            const bool valid = key[b] >= 0;
            bad += key[b] == -1;
            const unsigned grp = match_by_ballot(valid ? (unsigned)key[b] : key_invalid, nbits);
            if (valid && (grp & lt) == 0) row[key[b]] += __popc(grp);
            __syncwarp();
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
    if (lane == 0 && bad) atomicAdd(&s_invalid, bad);
    __syncthreads();

    // block histogram; per-warp counts become exclusive prefixes over warps.
    // `parts` threads share one expert (consecutive lanes), each folding a
    // contiguous group of warps, then combine with shuffles.
    {
        const int parts = fold_parts(E);
        const int per = kClusterWarps / parts;
        const int q = tid % parts;
        const int stride = kClusterThreads / parts;
        const int iters = (E + stride - 1) / stride;  // the same for every thread
        for (int it = 0; it < iters; ++it) {
            const int e = it * stride + tid / parts;
            const bool live = e < E;
            int sum = 0;
            if (live)
                for (int w = q * per; w < q * per + per; ++w) sum += wcnt[w * E + e];
            int incl = sum;  // inclusive scan of the part sums within the expert's lanes
            for (int o = 1; o < parts; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, o, parts);
                if (q >= o) incl += u;
            }
            if (live) {
                int run = incl - sum;
                for (int w = q * per; w < q * per + per; ++w) {
                    const int v = wcnt[w * E + e];
                    wcnt[w * E + e] = run;
                    run += v;
                }
                if (q == parts - 1) hist[e] = run;
            }
        }
    }
    if (tid == 0) hist[E] = s_invalid;
    cluster.sync();

    // totals and the prefix of earlier blocks, read from every block's
    // shared memory (all loads in flight together)
    for (int e = tid; e <= E; e += kClusterThreads) {
        int v[16];
#pragma unroll
        for (int b = 0; b < 16; ++b) v[b] = b < nc ? cluster.map_shared_rank(hist, b)[e] : 0;
        int t = 0, p = 0;
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            t += v[b];
            p += b < c ? v[b] : 0;
        }
        tot[e] = t;
        if (e < E) {
            pre[e] = p;
            pad[e] = (t + A - 1) / A * A;
        }
    }
    __syncthreads();
    const int n_invalid = tot[E];
    const int total = block_exclusive_scan(tot, E, warp_tmp);  // tot[e] = expert offset
    int pad_total = 0;
    if (bso) pad_total = block_exclusive_scan(pad, E, warp_tmp);
    if (c == 0) {
        for (int e = tid; e < E; e += kClusterThreads) {
            counts[e] = (e + 1 < E ? tot[e + 1] : total) - tot[e];
            offsets[e] = tot[e];
            if (bso) bso[e] = pad[e];
        }
        if (tid == 0) {
            offsets[E] = total;
            if (bso) bso[E] = pad_total;
            if (diag) {
                diag[0] = n_invalid;
                diag[1] = 0;
            }
        }
    }
    for (int x = tid; x < kClusterWarps * E; x += kClusterThreads) {
        const int e = x % E;
        wcnt[x] += tot[e] + pre[e];
    }
    __syncthreads();

    // pass 2: ranks and both permutations
    for (int64_t r0 = beg; r0 < end; r0 += 32 * kClusterBatch) {
        int key[kClusterBatch];
#pragma unroll
        for (int b = 0; b < kClusterBatch; ++b) {
            const int64_t i = r0 + b * 32 + lane;
            int k2 = -2;
            if (i < end) {
                const int id = __ldg(ids + i);
                k2 = (id >= 0 && id < E) ? id : -1;
            }
            key[b] = k2;
        }
#pragma unroll
        for (int b = 0; b < kClusterBatch; ++b) {
            if (r0 + b * 32 >= end) break;
            const int64_t i = r0 + b * 32 + lane;
            const bool valid = key[b] >= 0;
            const unsigned grp = match_by_ballot(valid ? (unsigned)key[b] : key_invalid, nbits);
            int p = -1;
            if (valid) {
                const int basev = row[key[b]];
                p = basev + __popc(grp & lt);
                __syncwarp(grp);
                if ((grp & lt) == 0) row[key[b]] = basev + __popc(grp);
            }
            __syncwarp();
            if (i < end) {
                out_perm[i] = p;
                if (p >= 0 && p < S) in_perm[p] = (int)i;
            }
        }
    }
    // input_permutation past the valid rows
    for (int64_t p = total + (int64_t)c * kClusterThreads + tid; p < S;
         p += (int64_t)nc * kClusterThreads)
        in_perm[p] = -1;
    cluster.sync();  // no block leaves while another may still read its histogram
}

// Tiny batches: every block recomputes the metadata in shared memory (the
// batch is at most kFusedMaxSlots slots), block 0 writes it out, and all
// blocks copy their share of the x rows to their k dispatched rows.
__global__ void __launch_bounds__(kPrepThreads)
    prep_dispatch_kernel(const int32_t *__restrict__ ids, int64_t T, int k, int E, int A,
                         int32_t *counts, int32_t *offsets, int32_t *bso, int32_t *in_perm,
                         int32_t *out_perm, int32_t *diag, const uint4 *__restrict__ x,
                         int64_t nvec, uint4 *__restrict__ out) {
    extern __shared__ int smem[];
    const int64_t S = T * k;
    int *pos = smem + kPrepWarps * E + 2 * (E + 1);  // [S]
    pdl_wait();
    pdl_launch_dependents();
    single_block_prepare(ids, S, E, A, smem, pos, blockIdx.x == 0, counts, offsets, bso, in_perm,
                         out_perm, diag);
    __syncthreads();
    const int64_t total = T * nvec;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = v / nvec, c = v - t * nvec;
        const uint4 val = ld_stream_v4(x + v);
        for (int j = 0; j < k; ++j) {
            const int p = pos[t * k + j];
            if (p >= 0) st_v4(out + (int64_t)p * nvec + c, val);
        }
    }
}

size_t single_block_smem(int E) { return (size_t)(kPrepWarps * E + 2 * (E + 1)) * sizeof(int); }

}  // namespace

size_t prepare_workspace_bytes(int64_t S, int E) {
    if (S <= kSingleBlockSlots) return 0;
    const int64_t G = (S + kPrepTile - 1) / kPrepTile;
    const size_t C = (size_t)E + 1;
    return 256 + align256((size_t)G * C * 8) + align256((size_t)G * C * 4);
}

namespace {

// Largest cluster of prep_cluster_kernel blocks this device can co-schedule
// (16 with the non-portable size, else 8), cached per device; 0 if none.
int cluster_blocks(size_t smem) {
    static std::mutex mu;
    static std::map<std::pair<int, size_t>, int> cache;
    const int dev = current_device();
    std::lock_guard<std::mutex> g(mu);
    auto key = std::make_pair(dev, smem);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int best = 0;
    ensure_smem(prep_cluster_kernel, smem);
    cudaFuncSetAttribute(prep_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    for (int nc : {16, 8}) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(nc, 1, 1);
        cfg.blockDim = dim3(kClusterThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = nc;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, prep_cluster_kernel, &cfg) == cudaSuccess && n > 0) {
            best = nc;
            break;
        }
        cudaGetLastError();
    }
    cache[key] = best;
    return best;
}

size_t cluster_smem(int E) {
    return (size_t)(kClusterWarps * E + 2 * (E + 1) + 2 * E) * sizeof(int);
}

}  // namespace

bool prepare_uses_cluster(int64_t S, int E) {
    return S > kSingleBlockSlots && S <= kClusterMaxSlots && cluster_blocks(cluster_smem(E)) > 0;
}

cudaError_t run_prepare(const int32_t *ids, int64_t S, int E, int A, int32_t *counts,
                        int32_t *offsets, int32_t *bso, int32_t *in_perm, int32_t *out_perm,
                        int32_t *diag, void *workspace, cudaStream_t stream) {
    if (S <= kSingleBlockSlots)
        return launch(prep_single_kernel, 1, kPrepThreads, single_block_smem(E), stream, ids, S,
                      E, A, counts, offsets, bso, in_perm, out_perm, diag);
    if (S <= kClusterMaxSlots) {
        const size_t smem = cluster_smem(E);
        const int nc = cluster_blocks(smem);
        if (nc > 0) {
            const int64_t warps = (int64_t)nc * kClusterWarps;
            const int64_t wch = ((S + warps - 1) / warps + 31) / 32 * 32;
            int nbits = 1;
            while ((1 << nbits) <= E) ++nbits;  // keys 0..E (E marks an invalid id)
            cudaError_t se = ensure_smem(prep_cluster_kernel, smem);
            if (se != cudaSuccess) return se;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(nc, 1, 1);
            cfg.blockDim = dim3(kClusterThreads, 1, 1);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = stream;
            cudaLaunchAttribute attr[2];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = nc;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[1].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 2;
            cudaError_t e = cudaLaunchKernelEx(&cfg, prep_cluster_kernel, ids, S, E, A, nbits, wch,
                                               counts, offsets, bso, in_perm, out_perm, diag);
            if (e != cudaSuccess) return e;
            return cudaGetLastError();
        }
    }
    const int G = (int)((S + kPrepTile - 1) / kPrepTile);
    const size_t smem1 = (size_t)3 * (E + 1) * sizeof(int);
    cudaError_t e = launch(prep_count_kernel, G, kPrepThreads, smem1, stream, ids, S, E, A, G,
                           workspace, counts, offsets, bso, diag);
    if (e != cudaSuccess) return e;
    const size_t smem2 = (size_t)kPrepWarps * E * sizeof(int);
    return launch(prep_scatter_kernel, G, kPrepThreads, smem2, stream, ids, S, E, G, workspace,
                  (const int32_t *)offsets, in_perm, out_perm, diag);
}

cudaError_t run_prepare_dispatch(const int32_t *ids, int64_t T, int k, int E, int A,
                                 int32_t *counts, int32_t *offsets, int32_t *bso,
                                 int32_t *in_perm, int32_t *out_perm, int32_t *diag,
                                 const void *x, int64_t row_bytes, void *out,
                                 cudaStream_t stream) {
    const int64_t S = T * k;
    const int64_t nvec = row_bytes / 16;
    const size_t smem = single_block_smem(E) + (size_t)S * sizeof(int);
    const int64_t units = (T * nvec + kPrepThreads - 1) / kPrepThreads;
    const int64_t grid = persistent_grid(prep_dispatch_kernel, kPrepThreads, smem, units);
    return launch(prep_dispatch_kernel, grid, kPrepThreads, smem, stream, ids, T, k, E, A, counts,
                  offsets, bso, in_perm, out_perm, diag, (const uint4 *)x, nvec, (uint4 *)out);
}

}  // namespace moe
