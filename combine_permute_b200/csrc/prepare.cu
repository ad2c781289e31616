// Routing metadata: a deterministic stable counting sort of the T*k slots by
// expert id (sglang PR #19058, "Changes", item 1 prepare_moe_input: tokens
// per expert, prefix-sum expert offsets, optional FP8 block-scale offsets,
// input / output permutations).
//
// The dispatched row of slot i with expert e is
//     offsets[e] + rank(i),  rank(i) = #{slots i' < i with expert e},
// so every path computes rank(i): within a warp by a ballot-built match over
// 32 consecutive slots, across a warp's rounds by a warp-private running
// counter in shared memory, across warps by an exclusive scan of the
// per-warp counts, and across blocks by one of:
//  * up to kSingleBlockSlots slots: nothing, one block does it all
//    (prep_single_kernel);
//  * above that, tiles of kTileSlots slots over the whole GPU:
//    prep_rank_kernel ranks each tile, then runs a decoupled look-back over
//    the tiles' per-expert aggregates (bounded waits, a window of
//    predecessors read together) and stores rank(i) in output_permutation;
//    the last tile holds the totals and writes counts and offsets.
//    prep_finish_kernel, element-wise, adds the expert offset and writes both
//    permutations.  Tiles take their index from an atomic ticket, so a tile
//    only ever waits on tiles that are already running; a wait that gives up
//    reports through diag[1]; the ticket wraps to zero and the finish kernel
//    clears every look-back word, so the workspace is all-zero between calls.
#include "kernels.h"
#include "launch.h"
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr unsigned long long kFlagAgg = 1ull << 32;
constexpr unsigned long long kFlagIncl = 2ull << 32;
constexpr int kMaxSpins = 1 << 20;  // x ~256 ns sleep: a wait gives up after ~0.3-1 s
constexpr int kLookbackWindow = 8;  // predecessor tiles read together

constexpr int kSingleThreads = 1024;
constexpr int kSingleWarps = kSingleThreads / 32;
constexpr int kSingleRounds = kSingleBlockSlots / kSingleThreads;  // rounds of 32 slots per warp

// Bits of a match key: keys run over 0..E, E standing for "no expert".
__host__ __device__ inline int key_bits(int E) {
    int n = 1;
    while ((1 << n) <= E) ++n;
    return n;
}

constexpr int kMaxKeyBits = 11;  // keys up to kMaxExperts

// Lanes of the warp whose key equals this lane's, built from one ballot per
// key bit (the ballots are independent and issue back to back).  All 32
// lanes must call it.
__device__ __forceinline__ unsigned match_key(unsigned key, int nbits) {
    unsigned m = 0xffffffffu;
#pragma unroll
    for (int b = 0; b < kMaxKeyBits; ++b) {
        if (b < nbits) {
            const unsigned bit = (key >> b) & 1u;
            const unsigned vote = __ballot_sync(0xffffffffu, bit);
            m &= bit ? vote : ~vote;
        }
    }
    return m;
}

// One round of stable ranking over 32 consecutive slots (one per lane, in
// lane order).  `e` is the slot's expert or a negative value; `row` is the
// warp's private running count per expert in shared memory.  Returns the
// number of the warp's earlier slots with expert e (-1 when e < 0) and
// advances row[e].  All 32 lanes must call it.
__device__ __forceinline__ int rank_round(int e, int E, int nbits, int *row, unsigned lt) {
    if (!__any_sync(0xffffffffu, e >= 0)) return -1;  // nothing to rank in this round
    const unsigned grp = match_key(e >= 0 ? (unsigned)e : (unsigned)E, nbits);
    const int base = e >= 0 ? row[e] : 0;
    __syncwarp();  // every lane has read its counter before a leader advances it
    if (e >= 0 && (grp & lt) == 0) row[e] = base + __popc(grp);
    __syncwarp();
    return e >= 0 ? base + __popc(grp & lt) : -1;
}

// Expert of slot i, -1 for an id outside [0, E), -2 past `end`.
__device__ __forceinline__ int load_key(const int32_t *__restrict__ ids, int64_t i, int64_t end,
                                        int E) {
    if (i >= end) return -2;
    const int id = __ldg(ids + i);
    return (id >= 0 && id < E) ? id : -1;
}

// Per-warp counts wcnt[w][e] (NW warps, row stride E+1 so that the lanes
// reading one expert's column hit different banks) become exclusive
// prefixes over w; hist[e] receives the sum.  Segments of NW lanes scan one
// expert's column with shuffles; each warp handles 32/NW experts at a time.
// All NT threads must call it.
template <int NT, int NW>
__device__ __forceinline__ void fold_warp_counts(int *wcnt, int E, int *hist) {
    static_assert(NW <= 32 && (NW & (NW - 1)) == 0, "warps per block: a power of two <= 32");
    constexpr int kExpertsPerPass = 32 / NW;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int w = lane % NW;
    for (int e0 = warp * kExpertsPerPass; e0 < E; e0 += (NT / 32) * kExpertsPerPass) {
        const int e = e0 + lane / NW;
        const bool live = e < E;
        const int v = live ? wcnt[w * (E + 1) + e] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < NW; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o, NW);
            if (w >= o) incl += u;
        }
        if (live) {
            wcnt[w * (E + 1) + e] = incl - v;
            if (w == NW - 1) hist[e] = incl;
        }
    }
}

// Counts / offsets / block-scale offsets from per-expert totals tot[0..E):
// tot becomes the expert offsets in place; pad is scratch of E ints.
// Writes the outputs when `write` is set.  Returns the number of valid
// slots.  All threads must call it.
__device__ __forceinline__ int offsets_from_totals(int *tot, int *pad, int E, int A, bool write,
                                                   int32_t *counts, int32_t *offsets,
                                                   int32_t *bso, int *warp_tmp) {
    const int tid = threadIdx.x, nt = blockDim.x;
    int pad_total = 0;
    const int total = block_exclusive_scan2(tot, pad, E, A, warp_tmp, &pad_total);
    if (write) {
        for (int e = tid; e < E; e += nt) {
            counts[e] = (e + 1 < E ? tot[e + 1] : total) - tot[e];
            offsets[e] = tot[e];
            if (bso) bso[e] = pad[e];
        }
        if (tid == 0) {
            offsets[E] = total;
            if (bso) bso[E] = pad_total;
        }
    }
    return total;
}

__host__ __device__ inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

struct PrepWs {
    unsigned *ticket;
    unsigned *timeout;
    unsigned long long *state;  // [G][E+1] look-back words: flag << 32 | value
};

__host__ __device__ inline PrepWs carve(void *ws) {
    char *b = (char *)ws;
    PrepWs w;
    w.ticket = (unsigned *)b;
    w.timeout = (unsigned *)(b + 4);
    w.state = (unsigned long long *)(b + 256);
    return w;
}

// ---------------------------------------------------------------------------
// One block (kSingleThreads threads, up to kSingleBlockSlots slots).  When
// `pos` is non-null the dispatched row of every slot is also left there
// (shared memory, S entries); global outputs are written when `write` is
// set.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void single_block_prepare(const int32_t *__restrict__ ids, int64_t S,
                                                     int E, int A, int *smem, int *pos,
                                                     bool write, int32_t *counts,
                                                     int32_t *offsets, int32_t *bso,
                                                     int32_t *in_perm, int32_t *out_perm,
                                                     int32_t *diag) {
    __shared__ int warp_tmp[66];
    __shared__ int s_invalid;
    int *wcnt = smem;                          // [kSingleWarps][E+1]
    int *tot = wcnt + kSingleWarps * (E + 1);  // [E]
    int *pad = tot + E;                        // [E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = lanemask_lt();
    const int nbits = key_bits(E);

    for (int x = tid; x < kSingleWarps * (E + 1); x += kSingleThreads) wcnt[x] = 0;
    if (tid == 0) s_invalid = 0;
    int key[kSingleRounds];
    const int64_t wbase = (int64_t)warp * 32 * kSingleRounds;
#pragma unroll
    for (int r = 0; r < kSingleRounds; ++r) key[r] = load_key(ids, wbase + r * 32 + lane, S, E);
    __syncthreads();

    int rank[kSingleRounds];
    int *row = wcnt + warp * (E + 1);
    int bad = 0;
#pragma unroll
    for (int r = 0; r < kSingleRounds; ++r) {
        rank[r] = rank_round(key[r], E, nbits, row, lt);
        bad += key[r] == -1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
    if (lane == 0 && bad) atomicAdd(&s_invalid, bad);
    __syncthreads();
    fold_warp_counts<kSingleThreads, kSingleWarps>(wcnt, E, tot);
    __syncthreads();
    const int total = offsets_from_totals(tot, pad, E, A, write, counts, offsets, bso, warp_tmp);
    if (write && tid == 0 && diag) {
        diag[0] = s_invalid;
        diag[1] = 0;
    }
    // a slot's row: expert offset + earlier warps (wcnt now holds the
    // exclusive prefix over warps) + its rank within the warp's run
#pragma unroll
    for (int r = 0; r < kSingleRounds; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        if (i < S) {
            const int e = key[r];
            const int p = e >= 0 ? tot[e] + row[e] + rank[r] : -1;
            if (pos) pos[i] = p;
            if (write) {
                out_perm[i] = p;
                if (p >= 0) in_perm[p] = (int)i;
            }
        }
    }
    if (write)
        for (int64_t p = total + tid; p < S; p += kSingleThreads) in_perm[p] = -1;
}

__global__ void __launch_bounds__(kSingleThreads, 1)
    prep_single_kernel(const int32_t *__restrict__ ids, int64_t S, int E, int A, int32_t *counts,
                       int32_t *offsets, int32_t *bso, int32_t *in_perm, int32_t *out_perm,
                       int32_t *diag) {
    extern __shared__ int smem[];
    pdl_wait();
    pdl_launch_dependents();
    single_block_prepare(ids, S, E, A, smem, nullptr, true, counts, offsets, bso, in_perm,
                         out_perm, diag);
}

size_t single_block_smem(int E) { return (size_t)(kSingleWarps * (E + 1) + 2 * E) * sizeof(int); }

// ---------------------------------------------------------------------------
// Tiled path, kernel A: rank every slot of a tile, look back across tiles,
// store rank(i) in output_permutation (-1 for an invalid id).  The last tile
// writes counts, offsets and block-scale offsets.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kTileThreads, 2)
    prep_rank_kernel(const int32_t *__restrict__ ids, int64_t S, int E, int A, int G,
                     void *workspace, int32_t *counts, int32_t *offsets, int32_t *bso,
                     int32_t *out_perm, int32_t *diag) {
    extern __shared__ int smem[];
    __shared__ int warp_tmp[66];
    __shared__ unsigned s_ticket;
    __shared__ int s_invalid;
    const int C = E + 1;                  // one column per expert plus one for invalid ids
    int *wcnt = smem;                     // [kTileWarps][E+1]
    int *hist = wcnt + kTileWarps * C;    // [C] this tile's counts
    int *excl = hist + C;                 // [C] slots of earlier tiles, then totals
    int *pad = excl + C;                  // [E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = lanemask_lt();
    const int nbits = key_bits(E);
    PrepWs ws = carve(workspace);

    for (int x = tid; x < kTileWarps * C; x += kTileThreads) wcnt[x] = 0;
    if (tid == 0) s_invalid = 0;
    pdl_wait();
    pdl_launch_dependents();
    if (tid == 0) {
        const unsigned t = atomicInc(ws.ticket, (unsigned)(G - 1));
        // a counter left non-zero by an aborted call: stay in bounds; the
        // bounded waits below then report the failure through diag[1]
        s_ticket = t < (unsigned)G ? t : t % (unsigned)G;
    }
    __syncthreads();
    const int tile = (int)s_ticket;
    const int64_t wbase = (int64_t)tile * kTileSlots + (int64_t)warp * 32 * kTileRounds;

    // 1. ranks within each warp's run, per-warp counts
    int key[kTileRounds], rank[kTileRounds];
#pragma unroll
    for (int r = 0; r < kTileRounds; ++r) key[r] = load_key(ids, wbase + r * 32 + lane, S, E);
    int *row = wcnt + warp * C;
    int bad = 0;
#pragma unroll
    for (int r = 0; r < kTileRounds; ++r) {
        rank[r] = rank_round(key[r], E, nbits, row, lt);
        bad += key[r] == -1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
    if (lane == 0 && bad) atomicAdd(&s_invalid, bad);
    __syncthreads();
    fold_warp_counts<kTileThreads, kTileWarps>(wcnt, E, hist);
    if (tid == 0) hist[E] = s_invalid;
    __syncthreads();

    // 2. publish this tile's aggregates
    unsigned long long *mine = ws.state + (size_t)tile * C;
    for (int c = tid; c < C; c += kTileThreads) st_relaxed_u64(mine + c, kFlagAgg | (unsigned)hist[c]);

    // 3. decoupled look-back, one column per thread, kLookbackWindow
    //    predecessors read together
    bool gave_up = false;
    for (int c = tid; c < C; c += kTileThreads) {
        int sum = 0;
        bool done = false;
        for (int pred = tile - 1; pred >= 0 && !done && !gave_up; pred -= kLookbackWindow) {
            unsigned long long v[kLookbackWindow];
#pragma unroll
            for (int q = 0; q < kLookbackWindow; ++q)
                v[q] = pred - q >= 0 ? ld_relaxed_u64(ws.state + (size_t)(pred - q) * C + c)
                                     : kFlagIncl;
#pragma unroll
            for (int q = 0; q < kLookbackWindow; ++q) {
                if (done || gave_up || pred - q < 0) continue;
                const unsigned long long *wp = ws.state + (size_t)(pred - q) * C + c;
                int spins = 0;
                while ((v[q] >> 32) == 0) {  // not published yet
                    if (++spins > kMaxSpins) {
                        gave_up = true;
                        break;
                    }
                    __nanosleep(256);
                    v[q] = ld_relaxed_u64(wp);
                }
                sum += (int)(unsigned)(v[q] & 0xffffffffu);
                if ((v[q] & kFlagIncl) != 0) done = true;
            }
        }
        // publish even after giving up, so that no later tile waits on us
        st_relaxed_u64(mine + c, kFlagIncl | (unsigned)(sum + hist[c]));
        excl[c] = sum;
    }
    if (gave_up) atomicExch(ws.timeout, 1u);
    __syncthreads();

    // 4. rank(i) = earlier tiles + earlier warps + earlier lanes of the run
#pragma unroll
    for (int r = 0; r < kTileRounds; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        if (i < S) {
            const int e = key[r];
            out_perm[i] = e >= 0 ? excl[e] + row[e] + rank[r] : -1;
        }
    }

    // 5. the last tile holds the totals
    if (tile != G - 1) return;
    __syncthreads();  // every rank above has read excl
    for (int c = tid; c < C; c += kTileThreads) excl[c] += hist[c];
    __syncthreads();
    if (tid == 0 && diag) diag[0] = excl[E];
    offsets_from_totals(excl, pad, E, A, true, counts, offsets, bso, warp_tmp);
}

// Tiled path, kernel B (element-wise): row = expert offset + rank; both
// permutations; clear the look-back words.
__global__ void __launch_bounds__(256)
    prep_finish_kernel(const int32_t *__restrict__ ids, int64_t S, int E, int64_t ws_words,
                       void *workspace, const int32_t *__restrict__ offsets, int32_t *in_perm,
                       int32_t *out_perm, int32_t *diag) {
    PrepWs ws = carve(workspace);
    pdl_wait();
    pdl_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t i = g; i < S; i += stride) {
        const int id = __ldg(ids + i);
        if (id >= 0 && id < E) {
            const int p = __ldg(offsets + id) + out_perm[i];
            out_perm[i] = p;
            if (p >= 0 && p < S) in_perm[p] = (int)i;
        }
    }
    for (int64_t p = __ldg(offsets + E) + g; p < S; p += stride) in_perm[p] = -1;
    for (int64_t w = g; w < ws_words; w += stride) ws.state[w] = 0ull;
    if (g == 0) {
        if (diag) diag[1] = *ws.timeout ? 1 : 0;
        *ws.timeout = 0u;
    }
}

// ---------------------------------------------------------------------------
// Tiny batches: every block recomputes the metadata in shared memory (the
// batch is at most kFusedMaxSlots slots), block 0 writes it out, and all
// blocks copy their share of the x rows to their k dispatched rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSingleThreads, 1)
    prep_dispatch_kernel(const int32_t *__restrict__ ids, int64_t T, int k, int E, int A,
                         int32_t *counts, int32_t *offsets, int32_t *bso, int32_t *in_perm,
                         int32_t *out_perm, int32_t *diag, const uint4 *__restrict__ x,
                         int64_t nvec, uint4 *__restrict__ out) {
    extern __shared__ int smem[];
    const int64_t S = T * k;
    int *pos = smem + kSingleWarps * (E + 1) + 2 * E;  // [S]
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

}  // namespace

size_t prepare_workspace_bytes(int64_t S, int E) {
    if (S <= kSingleBlockSlots) return 0;
    const int64_t G = (S + kTileSlots - 1) / kTileSlots;
    return 256 + align256((size_t)G * ((size_t)E + 1) * 8);
}

cudaError_t run_prepare(const int32_t *ids, int64_t S, int E, int A, int32_t *counts,
                        int32_t *offsets, int32_t *bso, int32_t *in_perm, int32_t *out_perm,
                        int32_t *diag, void *workspace, cudaStream_t stream) {
    if (S <= kSingleBlockSlots)
        return launch(prep_single_kernel, 1, kSingleThreads, single_block_smem(E), stream, ids, S,
                      E, A, counts, offsets, bso, in_perm, out_perm, diag);
    const int G = (int)((S + kTileSlots - 1) / kTileSlots);
    const size_t smem = (size_t)(kTileWarps * (E + 1) + 2 * (E + 1) + E) * sizeof(int);
    cudaError_t e = launch(prep_rank_kernel, G, kTileThreads, smem, stream, ids, S, E, A, G,
                           workspace, counts, offsets, bso, out_perm, diag);
    if (e != cudaSuccess) return e;
    const int64_t words = (int64_t)G * (E + 1);
    const int64_t grid = persistent_grid(prep_finish_kernel, 256, 0, (S + 1023) / 1024);
    return launch(prep_finish_kernel, grid, 256, 0, stream, ids, S, E, words, workspace,
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
    const int64_t units = (T * nvec + kSingleThreads - 1) / kSingleThreads;
    const int64_t grid = persistent_grid(prep_dispatch_kernel, kSingleThreads, smem, units);
    return launch(prep_dispatch_kernel, grid, kSingleThreads, smem, stream, ids, T, k, E, A,
                  counts, offsets, bso, in_perm, out_perm, diag, (const uint4 *)x, nvec,
                  (uint4 *)out);
}

}  // namespace moe
