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
//  * up to kSmallSlots slots: one block, one thread per slot, each slot's
//    rank counted directly over the earlier slots (prep_small_kernel);
//  * up to kSingleBlockSlots slots: one block does it all
//    (prep_single_kernel);
//  * above that, when every block fits on the GPU at once: one cooperative
//    launch (prep_sync_kernel, 512-thread blocks of 1 to 64 rounds).  Each
//    block ranks its slots, publishes its per-expert histogram row and meets
//    the others at a grid barrier (bounded wait); every block then stages
//    all rows, scans them into the expert offsets and its own prefix, and
//    writes both permutations for its slots;
//  * otherwise two kernels: prep_rank_kernel takes tiles of kTileSlots slots
//    by an atomic ticket (so a tile only ever waits on tiles already
//    running), publishes each tile's histogram and runs a decoupled
//    look-back over the earlier tiles' (bounded waits, a window of
//    predecessors read together); the last tile holds the totals and writes
//    counts and offsets, and every slot's rank(i) goes to output_permutation.
//    The element-wise prep_finish_kernel then adds the expert offset and
//    writes both permutations.  Look-back words carry the epoch of the call
//    that wrote them, so the workspace needs zeroing once, not per call.
// A wait that gives up reports through diag[1].
#include "kernels.h"
#include "launch.h"
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr unsigned long long kFlagAgg = 1ull << 32;   // word holds this tile's aggregate
constexpr unsigned long long kFlagIncl = 2ull << 32;  // word holds the inclusive prefix
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

// Expert of slot i (its id minus `base`), -1 for an id outside the window
// [base, base + E), -2 past `end`.  Ids are int32 or int64.
template <typename IdT>
__device__ __forceinline__ int load_key(const IdT *__restrict__ ids, int64_t i, int64_t end,
                                        int64_t base, int E) {
    if (i >= end) return -2;
    const int64_t id = (int64_t)__ldg(ids + i) - base;
    return (id >= 0 && id < E) ? (int)id : -1;
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

// Workspace of the tiled paths, in three fixed parts: a 256-byte header
// (counters), the one-launch path's histogram rows (a fixed kSyncHistBytes,
// one row of E+1 16-bit counts per block), then one 64-bit look-back word
// per (tile, expert column) of the two-kernel path.  The parts never move
// with the problem size, so no call reads another path's data as its own.
// A look-back word holds epoch << 34 | flag << 32 | value; it counts as
// published by this call only when its epoch field is this call's epoch, so
// words left by earlier calls need no clearing.  The epoch advances once per
// two-kernel call (by its last block); the ticket, done and barrier-arrival
// counters return to zero at the end of every call (the last block to
// finish clears them, once every block is past its waits).  The histogram rows are
// written before the grid barrier and read after it, so they need no
// clearing either.
struct PrepWs {
    unsigned *ticket;     // tile tickets, wraps at G
    unsigned *done;       // blocks finished, wraps at G
    unsigned *epoch;      // this call's epoch
    unsigned *timeout;    // set when a bounded wait gave up
    unsigned *arrive;           // one-launch path: blocks arrived at the grid barrier
    unsigned short *hist;       // [G][sync_stride(E)] histogram rows, one-launch path
    unsigned long long *state;  // [G][E+1] look-back words of the two-kernel path
};

// Most blocks of one one-launch prepare (one block per SM on B200, with room
// for parts with more SMs) and the fixed size of its histogram rows.  A row
// holds E+1 counts of at most kSyncMaxRounds * kSyncThreads = 32768 slots,
// so 16 bits each, padded to a multiple of 8 (16 bytes) so that rows are
// staged with 16-byte loads; at most kSyncThreads columns.  The region keeps
// room for 32-bit counts (512 KB), so that the workspace layout and size do
// not depend on the width of a count.
constexpr int kMaxSyncTiles = 256;
constexpr size_t kSyncHistBytes = (size_t)kMaxSyncTiles * 512 * sizeof(int);
__host__ __device__ inline int sync_stride(int E) { return (E + 1 + 7) & ~7; }

__host__ __device__ inline int64_t tiles_of(int64_t S) { return (S + kTileSlots - 1) / kTileSlots; }

__host__ __device__ inline PrepWs carve(void *ws) {
    char *b = (char *)ws;
    PrepWs w;
    w.ticket = (unsigned *)b;
    w.done = (unsigned *)(b + 4);
    w.epoch = (unsigned *)(b + 8);
    w.timeout = (unsigned *)(b + 16);
    w.arrive = (unsigned *)(b + 24);
    w.hist = (unsigned short *)(b + 256);
    w.state = (unsigned long long *)(b + 256 + kSyncHistBytes);
    return w;
}

constexpr unsigned kEpochMask = 0x3fffffffu;

__device__ __forceinline__ unsigned long long lb_word(unsigned epoch, unsigned long long flag,
                                                      int value) {
    return ((unsigned long long)(epoch & kEpochMask) << 34) | flag | (unsigned)value;
}

// Flag bits of a look-back word if it was published in `epoch`, else 0.
__device__ __forceinline__ unsigned long long lb_flag(unsigned long long w, unsigned epoch) {
    return (unsigned)(w >> 34) == (epoch & kEpochMask) ? (w & (3ull << 32)) : 0ull;
}

// ---------------------------------------------------------------------------
// Small batches (up to kSmallSlots slots): one thread per slot, in one
// block.  A slot's rank is counted directly: the number of earlier slots
// with the same expert, read from the keys staged in shared memory (a
// broadcast read, four keys at a time).  Counts come from shared-memory
// atomics, offsets from one block scan; three block barriers in all, where
// the counting sort needs its ranking rounds and a fold over warps.  smem:
// S + 4*(E+1) ints (keys, then counts / offsets, scan scratch).  `pos`, when
// non-null, receives every slot's dispatched row (shared memory, S ints);
// global outputs are written when `write` is set.  Every thread of the block
// calls it; blockDim.x >= S.
// ---------------------------------------------------------------------------
constexpr int kSmallSlots = 512;

template <typename IdT>
__device__ __forceinline__ void small_prepare(const IdT *__restrict__ ids, int64_t base, int S,
                                              int E, int A, int *smem, int *pos, bool write,
                                              int32_t *counts, int32_t *offsets, int32_t *bso,
                                              int32_t *in_perm, int32_t *out_perm,
                                              int32_t *diag) {
    __shared__ int warp_tmp[66];
    __shared__ int s_invalid;
    int *keys = smem;                           // [S], padded to a multiple of 4
    int *cnt = keys + ((S + 3) & ~3);           // [E] counts, then expert offsets
    int *pad = cnt + E;                         // [E] scan scratch
    const int tid = threadIdx.x, nt = blockDim.x;
    const int e = tid < S ? load_key(ids, tid, S, base, E) : -2;
    for (int c = tid; c < E; c += nt) cnt[c] = 0;
    if (tid < ((S + 3) & ~3)) keys[tid] = e;  // the padding keys are -2: no expert
    if (tid == 0) s_invalid = 0;
    __syncthreads();
    int rank = 0;
    if (e >= 0) {
        const int4 *k4 = reinterpret_cast<const int4 *>(keys);
        const int n4 = tid >> 2;
        for (int j = 0; j < n4; ++j) {
            const int4 v = k4[j];
            rank += (v.x == e) + (v.y == e) + (v.z == e) + (v.w == e);
        }
        for (int j = n4 << 2; j < tid; ++j) rank += keys[j] == e;
        atomicAdd(&cnt[e], 1);
    }
    const unsigned bad = __ballot_sync(0xffffffffu, e == -1);
    if ((tid & 31) == 0 && bad) atomicAdd(&s_invalid, __popc(bad));
    __syncthreads();
    const int total = offsets_from_totals(cnt, pad, E, A, write, counts, offsets, bso, warp_tmp);
    if (write && tid == 0 && diag) {
        diag[0] = s_invalid;
        diag[1] = 0;
    }
    __syncthreads();
    if (tid < S) {
        const int p = e >= 0 ? cnt[e] + rank : -1;
        if (pos) pos[tid] = p;
        if (write) {
            out_perm[tid] = p;
            if (p >= 0) in_perm[p] = tid;
        }
    }
    if (write)
        for (int p = total + tid; p < S; p += nt) in_perm[p] = -1;
}

template <typename IdT>
__global__ void __launch_bounds__(kSmallSlots, 1)
    prep_small_kernel(const IdT *__restrict__ ids, int64_t base, int S, int E, int A,
                      int32_t *counts, int32_t *offsets, int32_t *bso, int32_t *in_perm,
                      int32_t *out_perm, int32_t *diag) {
    extern __shared__ int smem[];
    pdl_wait();
    pdl_launch_dependents();
    small_prepare(ids, base, S, E, A, smem, nullptr, true, counts, offsets, bso, in_perm, out_perm,
                  diag);
}

__host__ __device__ inline size_t small_smem(int E, int64_t S) {
    return (size_t)(((S + 3) & ~3) + 2 * E) * sizeof(int);
}

// ---------------------------------------------------------------------------
// One block (kSingleThreads threads, up to kSingleBlockSlots slots).  When
// `pos` is non-null the dispatched row of every slot is also left there
// (shared memory, S entries); global outputs are written when `write` is
// set.
// ---------------------------------------------------------------------------
template <typename IdT>
__device__ __forceinline__ void single_block_prepare(const IdT *__restrict__ ids, int64_t base,
                                                     int64_t S, int E, int A, int *smem, int *pos,
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
    for (int r = 0; r < kSingleRounds; ++r)
        key[r] = load_key(ids, wbase + r * 32 + lane, S, base, E);
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

template <typename IdT>
__global__ void __launch_bounds__(kSingleThreads, 1)
    prep_single_kernel(const IdT *__restrict__ ids, int64_t base, int64_t S, int E, int A,
                       int32_t *counts,
                       int32_t *offsets, int32_t *bso, int32_t *in_perm, int32_t *out_perm,
                       int32_t *diag) {
    extern __shared__ int smem[];
    pdl_wait();
    pdl_launch_dependents();
    single_block_prepare(ids, base, S, E, A, smem, nullptr, true, counts, offsets, bso, in_perm,
                         out_perm, diag);
}

size_t single_block_smem(int E) { return (size_t)(kSingleWarps * (E + 1) + 2 * E) * sizeof(int); }

// A slot's expert e (-2..E-1) and its rank within its warp's run
// (-1..2047) in one int.
__device__ __forceinline__ int pack_key_rank(int e, int rank) { return (rank + 1) << 12 | (e + 2); }
__device__ __forceinline__ int packed_key(int v) { return (v & 4095) - 2; }
__device__ __forceinline__ int packed_rank(int v) { return (v >> 12) - 1; }

// ---------------------------------------------------------------------------
// Tiled paths.  A tile is a run of consecutive slots ranked by one block of
// NT threads: warp w takes nr rounds of 32 consecutive slots starting at
// first + w * 32 * nr.  Round r of a lane's slots keeps its expert, then its
// expert and rank packed, at kr[r * 32] in shared memory (this lane's own
// entries), so that the round loops stay rolled.  rank_tile() ranks the
// slots within each warp's run and folds the warps into the tile histogram:
// hist[c] for c < E is the tile's count of expert c, hist[E] its count of
// invalid ids; wcnt holds the per-warp exclusive prefixes.
// ---------------------------------------------------------------------------
template <typename IdT, int NT>
__device__ __forceinline__ void rank_tile(const IdT *__restrict__ ids, int64_t base, int64_t S,
                                          int E, int64_t first, int nr, int *wcnt, int *hist,
                                          int *s_invalid, int *kr) {
    constexpr int NW = NT / 32;
    const int C = E + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned lt = lanemask_lt();
    const int nbits = key_bits(E);
    const int64_t wbase = first + (int64_t)warp * 32 * nr;
#pragma unroll 4
    for (int r = 0; r < nr; ++r) kr[r * 32] = load_key(ids, wbase + r * 32 + lane, S, base, E);
    for (int x = tid; x < NW * C; x += NT) wcnt[x] = 0;
    if (tid == 0) *s_invalid = 0;
    __syncthreads();
    int *row = wcnt + warp * C;
    int bad = 0;
#pragma unroll 1
    for (int r = 0; r < nr; ++r) {
        const int e = kr[r * 32];
        kr[r * 32] = pack_key_rank(e, rank_round(e, E, nbits, row, lt));
        bad += e == -1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
    if (lane == 0 && bad) atomicAdd(s_invalid, bad);
    __syncthreads();
    fold_warp_counts<NT, NW>(wcnt, E, hist);
    if (tid == 0) hist[E] = *s_invalid;
    __syncthreads();
}

// Both permutations of a tile's slots: row = off[e] (expert offset, or 0) +
// excl[e] (earlier tiles) + wcnt (earlier warps) + rank (earlier lanes and
// rounds).  When `in_perm` is null only the rank part goes to out_perm.
__device__ __forceinline__ void write_tile_rows(int64_t S, int E, int64_t first, int nr,
                                                const int *off, const int *excl, const int *wcnt,
                                                const int *kr, int32_t *in_perm,
                                                int32_t *out_perm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t wbase = first + (int64_t)warp * 32 * nr;
    const int *row = wcnt + warp * (E + 1);
#pragma unroll 1
    for (int r = 0; r < nr; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        if (i < S) {
            const int v = kr[r * 32];
            const int e = packed_key(v);
            const int p = e >= 0 ? (off ? off[e] : 0) + excl[e] + row[e] + packed_rank(v) : -1;
            out_perm[i] = p;
            if (in_perm && p >= 0 && p < S) in_perm[p] = (int)i;
        }
    }
}

// Decoupled look-back (two-kernel path): publish this tile's aggregates,
// then per column sum the earlier tiles' values, kLookbackWindow
// predecessors read together, stopping at an inclusive prefix; publish the
// inclusive prefix.  excl[c] receives the slots of column c in earlier tiles.
template <int NT>
__device__ __forceinline__ void tile_lookback(const PrepWs &ws, int tile, unsigned epoch, int E,
                                              const int *hist, int *excl,
                                              unsigned long long wait_ns) {
    const int C = E + 1;
    unsigned long long *mine = ws.state + (size_t)tile * C;
    for (int c = threadIdx.x; c < C; c += NT)
        st_relaxed_u64(mine + c, lb_word(epoch, kFlagAgg, hist[c]));
    bool gave_up = false;
    for (int c = threadIdx.x; c < C; c += NT) {
        int sum = 0;
        bool done = false;
        for (int pred = tile - 1; pred >= 0 && !done && !gave_up; pred -= kLookbackWindow) {
            unsigned long long v[kLookbackWindow];
#pragma unroll
            for (int q = 0; q < kLookbackWindow; ++q)
                v[q] = pred - q >= 0 ? ld_relaxed_u64(ws.state + (size_t)(pred - q) * C + c) : 0ull;
#pragma unroll
            for (int q = 0; q < kLookbackWindow; ++q) {
                if (done || gave_up || pred - q < 0) continue;
                const unsigned long long *wp = ws.state + (size_t)(pred - q) * C + c;
                unsigned long long t0 = 0;
                while (lb_flag(v[q], epoch) == 0) {  // not published by this call yet
                    const unsigned long long now = globaltimer_ns();
                    if (t0 == 0) t0 = now;
                    if (now - t0 >= wait_ns) {
                        gave_up = true;
                        break;
                    }
                    __nanosleep(128);
                    v[q] = ld_relaxed_u64(wp);
                }
                sum += (int)(unsigned)(v[q] & 0xffffffffu);
                if (lb_flag(v[q], epoch) == kFlagIncl) done = true;
            }
        }
        // publish even after giving up, so that no later tile waits on us
        st_relaxed_u64(mine + c, lb_word(epoch, kFlagIncl, sum + hist[c]));
        excl[c] = sum;
    }
    if (gave_up) atomicExch(ws.timeout, 1u);
    __syncthreads();
}

// The block's exit: the last block of the call to finish reports a wait
// that gave up, clears that flag and advances the epoch for the next call.
__device__ __forceinline__ void tile_finish(const PrepWs &ws, int G, unsigned epoch,
                                            int32_t *diag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicInc(ws.done, (unsigned)(G - 1)) == (unsigned)(G - 1)) {
            const unsigned to = atomicExch(ws.timeout, 0u);
            if (diag) diag[1] = to ? 1 : 0;
            *(volatile unsigned *)ws.epoch = epoch + 1;
        }
    }
}

constexpr int kRankThreads = 256;                  // two-kernel tiles: 8 warps
constexpr int kRankRounds = kTileSlots / kRankThreads;  // of 8 rounds
constexpr int kSyncThreads = 512;                  // one-launch tiles: 16 warps
static_assert(kSyncThreads <= 512, "a histogram row of the one-launch path fits kSyncHistBytes");
constexpr int kSyncStagedRounds = 16;              // staged input_permutation: 5 to 16 rounds
constexpr int kSyncUnrolledRounds = 32;            // id loads unrolled: 5 to 32 rounds
constexpr int kSyncMaxRounds = 64;                 // of up to 64 rounds (32768 slots)
constexpr int kSyncMinRounds = 4;
static_assert(kSyncMaxRounds * kSyncThreads <= 65535, "a block's count of one expert fits 16 bits");

// Shared memory of the two-kernel tiles: per-warp rows, then hist, excl,
// off, pad (one column per expert plus one for invalid ids each), then the
// tile's slots (expert and rank packed).
template <int NT> size_t tile_smem(int E) {
    return ((size_t)(NT / 32 + 4) * (E + 1) + (size_t)kTileSlots) * sizeof(int);
}

// One-launch prepare (a cooperative launch: every block resident, so blocks
// may wait on one another; E + 1 <= kSyncThreads).  Block b ranks slots
// [b*nr*NT, (b+1)*nr*NT) within each warp's run, folds the warps into its
// histogram row (16-bit counts), publishes the row and arrives at a grid
// barrier: one release reduction on an arrival counter, then a bounded
// acquire poll until the counter reads G.  Then every block stages all G
// rows in shared memory; thread c sums column c into the total and this
// block's prefix over earlier blocks (eight rows in flight), and three
// exclusive scans over the experts run in registers: the expert offsets, the
// block-scale offsets (block 0 writes both and the counts) and this block's
// own offsets.  Every slot's row goes to output_permutation.  With kStage
// (from 5 to kSyncStagedRounds rounds) the block's slots are also staged in
// shared memory in dispatched order, so that input_permutation is written in
// runs of consecutive rows rather than one scattered word per slot; with
// fewer rounds that measured slower, with more it would not fit beside the
// rows, and input_permutation is written slot by slot.  Blocks count
// themselves out on a second word whose high half counts the waits that gave
// up; the last one clears both counters and reports the waits in diag[1].
template <int NT> size_t sync_smem(int E, int G, int nr, bool stage) {
    return (size_t)(NT / 32 + 4) * (E + 1) * sizeof(int) +
           (size_t)G * sync_stride(E) * sizeof(unsigned short) +
           (stage ? 3 : 1) * (size_t)nr * NT * sizeof(int);
}

template <typename IdT, bool kStage>
__global__ void __launch_bounds__(kSyncThreads, 1)
    prep_sync_kernel(const IdT *__restrict__ ids, int64_t base, int64_t S, int E, int A, int G,
                     int nr, void *workspace, unsigned long long wait_ns, int32_t *counts,
                     int32_t *offsets, int32_t *bso, int32_t *in_perm, int32_t *out_perm,
                     int32_t *diag) {
    constexpr int NT = kSyncThreads, NW = NT / 32;
    extern __shared__ int smem[];
    __shared__ int s_wsum[3][NW];
    __shared__ int s_invalid;
    const int C = E + 1, Cp = sync_stride(E);
    int *wcnt = smem;            // [NW][C] per-warp counts, then exclusive prefixes
    int *base_row = wcnt + NW * C;  // [C] expert offset + earlier blocks' counts
    int *lofs = base_row + C;       // [C] this block's offsets of its own slots
    // [G][Cp] every block's counts (16-byte aligned: (NW + 4) * 4 is a multiple of 16)
    unsigned short *rows = reinterpret_cast<unsigned short *>(wcnt + (NW + 4) * C);
    // kStage: [nr*NT] slots and [nr*NT] their rows, in dispatched order
    int *s_slot = reinterpret_cast<int *>(rows + (size_t)G * Cp);
    int *s_row = s_slot + (kStage ? nr * NT : 0);
    int *s_kr = s_row + (kStage ? nr * NT : 0);  // [nr*NT] each slot's expert and rank
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tile = blockIdx.x;
    const int64_t first = (int64_t)tile * nr * NT;
    const PrepWs ws = carve(workspace);
    for (int x = tid; x < NW * C; x += NT) wcnt[x] = 0;  // shared memory only: before the wait
    if (tid == 0) s_invalid = 0;
    pdl_wait();
    pdl_launch_dependents();

    // rank within each warp's run of nr * 32 consecutive slots
    const unsigned lt = lanemask_lt();
    const int nbits = key_bits(E);
    const int64_t wbase = first + (int64_t)warp * 32 * nr;
    // Round r of this lane is slot wbase + r*32 + lane; its expert, then its
    // rank, live in shared memory at kr[r*32] (read and written by this lane
    // only).  The ranking and row loops stay rolled: fully unrolled over the
    // largest round count, the kernel's code ran slower than its work (each
    // launch fetches it anew).  From 5 to kSyncUnrolledRounds rounds the
    // loads are unrolled, so that every round's id is in flight at once
    // (above that, four at a time): measured at 11 rounds,
    // 13.6 us a call against 14.0 rolled (16.2 against 17.2 after an L2
    // flush); unrolled at 1 to 4 rounds they cost 0.4-0.6 us more.
    int *kr = s_kr + warp * 32 * nr + lane;
    if (nr <= 4 || nr > kSyncUnrolledRounds) {
#pragma unroll 4
        for (int r = 0; r < nr; ++r) kr[r * 32] = load_key(ids, wbase + r * 32 + lane, S, base, E);
    } else {
        constexpr int NRMAX = kStage ? kSyncStagedRounds : kSyncUnrolledRounds;
        int key[NRMAX];  // every round's id in flight at once
#pragma unroll
        for (int r = 0; r < NRMAX; ++r)
            key[r] = r < nr ? load_key(ids, wbase + r * 32 + lane, S, base, E) : -2;
#pragma unroll
        for (int r = 0; r < NRMAX; ++r)
            if (r < nr) kr[r * 32] = key[r];
    }
    __syncthreads();
    int *row = wcnt + warp * C;
    int bad = 0;
#pragma unroll 1
    for (int r = 0; r < nr; ++r) {
        const int e = kr[r * 32];
        kr[r * 32] = pack_key_rank(e, rank_round(e, E, nbits, row, lt));
        bad += e == -1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
    if (lane == 0 && bad) atomicAdd(&s_invalid, bad);
    __syncthreads();

    // fold the warps: column c becomes exclusive over warps; publish the row
    // (a block has at most nr * NT <= 32768 slots, so every count fits 16 bits)
    if (tid < C) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const int v = wcnt[w * C + tid];
            wcnt[w * C + tid] = run;
            run += v;
        }
        ws.hist[(size_t)tile * Cp + tid] = (unsigned short)(tid < E ? run : s_invalid);
    }
    __syncthreads();
    unsigned done_old = 0, gave_up = 0;
    if (tid == 0) {
        // grid barrier: the arrival releases this block's row (published
        // before the block barrier above); reading G acquires every row
        red_add_release_u32(ws.arrive, 1u);
        const unsigned long long t0 = globaltimer_ns();
        while (ld_acquire_u32(ws.arrive) != (unsigned)G) {
            if (globaltimer_ns() - t0 >= wait_ns) {
                gave_up = 1;
                break;
            }
            __nanosleep(32);
        }
        // count this block out (ordered after its arrival); the result is
        // needed only at the end
        done_old = atom_add_acq_rel_u32(ws.done, 1u + (gave_up << 16));
    }
    __syncthreads();

    // stage the G rows (L2 only: other SMs wrote them; a row is a multiple
    // of 16 bytes), then per column the total, the prefix over earlier
    // blocks and this block's own count
    {
        const int4 *s4 = reinterpret_cast<const int4 *>(ws.hist);
        int4 *d4 = reinterpret_cast<int4 *>(rows);
        const int n4 = G * Cp / 8;
        for (int x = tid; x < n4; x += NT) d4[x] = __ldcg(s4 + x);
    }
    __syncthreads();
    int before = 0, all = 0, mine = 0;
    if (tid < C) {
        const unsigned short *col = rows + tid;
        int t = 0;
        for (; t + 8 <= G; t += 8) {
            int v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = col[(t + q) * Cp];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                all += v[q];
                before += t + q < tile ? v[q] : 0;
            }
        }
        for (; t < G; ++t) {
            const int v = col[t * Cp];
            all += v;
            before += t < tile ? v : 0;
        }
        mine = col[tile * Cp];
    }
    // three exclusive scans over the experts: counts, counts rounded up to
    // A, this block's counts (warp shuffles, then the warp sums)
    const int cnt = tid < E ? all : 0;
    const int padded = (cnt + A - 1) / A * A;
    const int own = tid < E ? mine : 0;
    int ia = cnt, ip = padded, io = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ua = __shfl_up_sync(0xffffffffu, ia, o);
        const int up = __shfl_up_sync(0xffffffffu, ip, o);
        const int uo = __shfl_up_sync(0xffffffffu, io, o);
        if (lane >= o) {
            ia += ua;
            ip += up;
            io += uo;
        }
    }
    if (lane == 31) {
        s_wsum[0][warp] = ia;
        s_wsum[1][warp] = ip;
        s_wsum[2][warp] = io;
    }
    __syncthreads();
    int ba = 0, bp = 0, bo = 0, total = 0, pad_total = 0, own_total = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int xa = s_wsum[0][w], xp = s_wsum[1][w], xo = s_wsum[2][w];
        if (w < warp) {
            ba += xa;
            bp += xp;
            bo += xo;
        }
        total += xa;
        pad_total += xp;
        own_total += xo;
    }
    const int ex_off = ba + ia - cnt;
    if (tid < C) {
        base_row[tid] = ex_off + before;
        lofs[tid] = bo + io - own;
    }
    if (tile == 0) {
        if (tid < E) {
            counts[tid] = cnt;
            offsets[tid] = ex_off;
            if (bso) bso[tid] = bp + ip - padded;
        }
        if (tid == 0) {
            offsets[E] = total;
            if (bso) bso[E] = pad_total;
        }
        if (tid == E && diag) diag[0] = all;  // column E counts the invalid ids
    }
    __syncthreads();

    // rows: slot i of expert e is this block's lr-th slot of e, lr = earlier
    // warps + its rank in the warp's run; output_permutation directly,
    // input_permutation through the staged dispatched order
#pragma unroll 1
    for (int r = 0; r < nr; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        if (i < S) {
            const int v = kr[r * 32];
            const int e = packed_key(v);
            int p = -1;
            if (e >= 0) {
                const int lr = row[e] + packed_rank(v);
                p = base_row[e] + lr;
                if constexpr (kStage) {
                    const int lp = lofs[e] + lr;
                    if (lp >= 0 && lp < nr * NT) {
                        s_slot[lp] = (int)i;
                        s_row[lp] = p;
                    }
                } else if (p < S) {
                    in_perm[p] = (int)i;
                }
            }
            out_perm[i] = p;
        }
    }
    if constexpr (kStage) {
        __syncthreads();
        const int nown = own_total < nr * NT ? own_total : nr * NT;
        for (int lp = tid; lp < nown; lp += NT) {
            const int p = s_row[lp];
            if (p >= 0 && p < S) in_perm[p] = s_slot[lp];
        }
    }
    const int64_t lo = first > total ? first : (int64_t)total;
    const int64_t end = first + (int64_t)nr * NT;
    const int64_t hi = end < S ? end : S;
    for (int64_t p = lo + tid; p < hi; p += NT) in_perm[p] = -1;
    if (tid == 0 && (done_old & 0xffffu) == (unsigned)(G - 1)) {
        // every block is past its wait: the counters can start over
        const unsigned to = (done_old >> 16) + gave_up;
        atomicExch(ws.arrive, 0u);
        atomicExch(ws.done, 0u);
        if (diag) diag[1] = to ? 1 : 0;
    }
}

// Two-kernel variant, kernel 1 (any number of tiles): store rank(i) in
// output_permutation (-1 for an invalid id); the last tile writes counts,
// offsets and block-scale offsets.  Tiles take their index from an atomic
// ticket, so a tile only waits on tiles that are already running.
template <typename IdT>
__global__ void __launch_bounds__(kRankThreads, 2)
    prep_rank_kernel(const IdT *__restrict__ ids, int64_t base, int64_t S, int E, int A, int G,
                     void *workspace, unsigned long long wait_ns, int32_t *counts,
                     int32_t *offsets, int32_t *bso, int32_t *out_perm, int32_t *diag) {
    constexpr int NT = kRankThreads, NR = kRankRounds;
    extern __shared__ int smem[];
    __shared__ int warp_tmp[66];
    __shared__ unsigned s_misc[2];
    __shared__ int s_invalid;
    const int C = E + 1;
    int *wcnt = smem;
    int *hist = wcnt + (NT / 32) * C;
    int *excl = hist + C;
    int *off = excl + C;
    int *pad = off + C;
    int *s_kr = pad + C;  // [NR][NT] each slot's expert and rank, warp by warp
    PrepWs ws = carve(workspace);
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        const unsigned t = atomicInc(ws.ticket, (unsigned)(G - 1));
        // a counter left non-zero by an aborted call: stay in bounds; the
        // bounded waits then report the failure through diag[1]
        s_misc[0] = t < (unsigned)G ? t : t % (unsigned)G;
        s_misc[1] = ld_relaxed_u32(ws.epoch);
    }
    __syncthreads();
    const int tile = (int)s_misc[0];
    const unsigned epoch = s_misc[1];
    const int64_t first = (int64_t)tile * kTileSlots;
    int *kr = s_kr + (threadIdx.x >> 5) * 32 * NR + (threadIdx.x & 31);
    rank_tile<IdT, NT>(ids, base, S, E, first, NR, wcnt, hist, &s_invalid, kr);
    tile_lookback<NT>(ws, tile, epoch, E, hist, excl, wait_ns);
    write_tile_rows(S, E, first, NR, nullptr, excl, wcnt, kr, nullptr, out_perm);
    if (tile == G - 1) {
        for (int c = threadIdx.x; c < C; c += NT) off[c] = excl[c] + hist[c];
        __syncthreads();
        if (threadIdx.x == 0 && diag) diag[0] = off[E];
        offsets_from_totals(off, pad, E, A, true, counts, offsets, bso, warp_tmp);
    }
    tile_finish(ws, G, epoch, diag);
}

// Two-kernel variant, kernel 2 (element-wise): row = expert offset + rank;
// both permutations.
template <typename IdT>
__global__ void __launch_bounds__(256)
    prep_finish_kernel(const IdT *__restrict__ ids, int64_t base, int64_t S, int E,
                       const int32_t *__restrict__ offsets, int32_t *in_perm, int32_t *out_perm) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t i = g; i < S; i += stride) {
        const int e = load_key(ids, i, S, base, E);
        if (e >= 0) {
            const int p = __ldg(offsets + e) + out_perm[i];
            out_perm[i] = p;
            if (p >= 0 && p < S) in_perm[p] = (int)i;
        }
    }
    for (int64_t p = __ldg(offsets + E) + g; p < S; p += stride) in_perm[p] = -1;
}

// ---------------------------------------------------------------------------
// Tiny batches: every block recomputes the metadata in shared memory (the
// batch is at most kFusedMaxSlots slots), block 0 writes it out, and all
// blocks copy their share of the x rows to their k dispatched rows (each
// thread's first x vector is loaded before the metadata is built).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSingleThreads, 1)
    prep_dispatch_kernel(const int32_t *__restrict__ ids, int64_t T, int k, int E, int A,
                         int32_t *counts, int32_t *offsets, int32_t *bso, int32_t *in_perm,
                         int32_t *out_perm, int32_t *diag, const uint4 *__restrict__ x,
                         int64_t nvec, uint4 *__restrict__ out) {
    extern __shared__ int smem[];
    const int64_t S = T * k;
    int *pos;  // [S] dispatched row of every slot
    pdl_wait();
    pdl_launch_dependents();
    // this thread's first x vector, in flight while the metadata is built
    const int64_t total = T * nvec;
    const int64_t v0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const uint4 x0 = v0 < total ? ld_stream_v4(x + v0) : make_uint4(0u, 0u, 0u, 0u);
    if (S <= kSmallSlots) {
        pos = smem + small_smem(E, S) / sizeof(int);
        small_prepare(ids, (int64_t)0, (int)S, E, A, smem, pos, blockIdx.x == 0, counts, offsets,
                      bso, in_perm, out_perm, diag);
    } else {
        pos = smem + kSingleWarps * (E + 1) + 2 * E;
        single_block_prepare(ids, (int64_t)0, S, E, A, smem, pos, blockIdx.x == 0, counts,
                             offsets, bso, in_perm, out_perm, diag);
    }
    __syncthreads();
    for (int64_t v = v0; v < total; v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = v / nvec, c = v - t * nvec;
        const uint4 val = v == v0 ? x0 : ld_stream_v4(x + v);
        for (int j = 0; j < k; ++j) {
            const int p = pos[t * k + j];
            if (p >= 0) st_v4(out + (int64_t)p * nvec + c, val);
        }
    }
}

}  // namespace

size_t prepare_workspace_bytes(int64_t S, int E) {
    if (S <= kSingleBlockSlots) return 0;
    return 256 + kSyncHistBytes + align256((size_t)tiles_of(S) * ((size_t)E + 1) * 8);
}

namespace {

// Tile shape of the one-launch path: nr rounds of kSyncThreads slots per
// block, G = ceil(S / (nr * kSyncThreads)) blocks.  nr is the fewest rounds
// from 1 to kSyncMinRounds that keeps the histogram rows every block stages
// (G x (E+1) counts) within kSyncStagedCounts, else kSyncMinRounds; more
// when the blocks would not all be resident.  Fewer rounds shorten the
// ranking, more blocks lengthen the staging: measured per call back to
// back, 32768 slots of 256 experts took 7.3 us at 1 round against 7.4 at 2
// and 8.5 at 4, 73728 slots 8.25 us at 2 rounds against 8.55 at 3 and 8.75
// at 1, 131072 slots of 288 experts 9.4 us at 4 against 9.45 at 2 and 3 and
// 10.7 at 6.  False when the problem needs more than kSyncMaxRounds rounds
// or kMaxSyncTiles blocks, or has more experts than a block has threads.
constexpr int64_t kSyncStagedCounts = 20480;

bool sync_shape(int64_t S, int E, int64_t resident, int *nr_out, int *G_out) {
    if (E + 1 > kSyncThreads) return false;
    const int64_t cap = resident < kMaxSyncTiles ? resident : kMaxSyncTiles;
    if (cap < 1) return false;
    int64_t least = kSyncMinRounds;
    for (int64_t r = 1; r < kSyncMinRounds; ++r) {
        const int64_t G = (S + r * kSyncThreads - 1) / (r * kSyncThreads);
        if (G * (E + 1) <= kSyncStagedCounts) {
            least = r;
            break;
        }
    }
    int64_t nr = (S + cap * kSyncThreads - 1) / (cap * kSyncThreads);
    if (nr < least) nr = least;
    if (nr > kSyncMaxRounds) return false;
    *nr_out = (int)nr;
    *G_out = (int)((S + nr * kSyncThreads - 1) / (nr * kSyncThreads));
    return true;
}

// One cooperative launch of prep_sync_kernel when every block fits on the
// GPU at once; returns cudaErrorCooperativeLaunchTooLarge (nothing launched)
// when they do not or the launch form is refused.
template <typename IdT>
cudaError_t launch_sync(const IdT *ids, int64_t base, int64_t S, int E, int A, void *workspace,
                        int32_t *counts, int32_t *offsets, int32_t *bso, int32_t *in_perm,
                        int32_t *out_perm, int32_t *diag, cudaStream_t stream) {
    int nr = 0, G = 0;
    if (!sync_shape(S, E, (int64_t)sm_count(), &nr, &G)) return cudaErrorCooperativeLaunchTooLarge;
    // staged from 5 to kSyncStagedRounds rounds: measured per call back to
    // back, 13.7 against 16.0 us at 11 rounds, while at 1 to 4 rounds the
    // slot-by-slot form was 0.1-0.2 us faster (7.25 against 7.33 us at 1)
    const bool stage = nr > 4 && nr <= kSyncStagedRounds;
    auto kern = stage ? prep_sync_kernel<IdT, true> : prep_sync_kernel<IdT, false>;
    const size_t smem = sync_smem<kSyncThreads>(E, G, nr, stage);
    if (smem > 200 * 1024) return cudaErrorCooperativeLaunchTooLarge;
    const int64_t resident = (int64_t)sm_count() * blocks_per_sm(kern, kSyncThreads, smem);
    if (G > resident) return cudaErrorCooperativeLaunchTooLarge;
    cudaError_t se = ensure_smem(kern, smem);
    if (se != cudaSuccess) return se;
    const unsigned long long wait_ns = prepare_wait_ns().load();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G, 1, 1);
    cfg.blockDim = dim3(kSyncThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    for (int n : {2, 1}) {  // with programmatic serialization if allowed, else without
        cfg.numAttrs = n;
        cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ids, base, S, E, A, G, nr, workspace,
                                           wait_ns, counts, offsets, bso, in_perm, out_perm, diag);
        if (e == cudaSuccess) return cudaGetLastError();
        cudaGetLastError();
    }
    return cudaErrorCooperativeLaunchTooLarge;
}

template <typename IdT>
cudaError_t run_prepare_t(const IdT *ids, int64_t base, int64_t S, int E, int A, int32_t *counts,
                          int32_t *offsets, int32_t *bso, int32_t *in_perm, int32_t *out_perm,
                          int32_t *diag, void *workspace, cudaStream_t stream) {
    if (S <= kSmallSlots) {
        const int threads = S < 32 ? 32 : (int)((S + 31) / 32 * 32);
        return launch(prep_small_kernel<IdT>, 1, threads, small_smem(E, S), stream, Start::kEarly,
                      ids, base, (int)S, E, A, counts, offsets, bso, in_perm, out_perm, diag);
    }
    if (S <= kSingleBlockSlots)
        return launch(prep_single_kernel<IdT>, 1, kSingleThreads, single_block_smem(E), stream,
                      Start::kEarly, ids, base, S, E, A, counts, offsets, bso, in_perm, out_perm,
                      diag);
    cudaError_t e = launch_sync(ids, base, S, E, A, workspace, counts, offsets, bso, in_perm,
                                out_perm, diag, stream);
    if (e != cudaErrorCooperativeLaunchTooLarge) return e;
    const int G = (int)tiles_of(S);
    e = launch(prep_rank_kernel<IdT>, G, kRankThreads, tile_smem<kRankThreads>(E), stream,
               Start::kEarly, ids, base, S, E, A, G, workspace,
               (unsigned long long)prepare_wait_ns().load(), counts, offsets, bso, out_perm, diag);
    if (e != cudaSuccess) return e;
    const int64_t grid = persistent_grid(prep_finish_kernel<IdT>, 256, 0, (S + 1023) / 1024);
    return launch(prep_finish_kernel<IdT>, grid, 256, 0, stream, Start::kEarly, ids, base, S, E,
                  (const int32_t *)offsets, in_perm, out_perm);
}

}  // namespace

cudaError_t run_prepare(const void *ids, bool ids64, int64_t base, int64_t S, int E, int A,
                        int32_t *counts, int32_t *offsets, int32_t *bso, int32_t *in_perm,
                        int32_t *out_perm, int32_t *diag, void *workspace, cudaStream_t stream) {
    if (ids64)
        return run_prepare_t((const int64_t *)ids, base, S, E, A, counts, offsets, bso, in_perm,
                             out_perm, diag, workspace, stream);
    return run_prepare_t((const int32_t *)ids, base, S, E, A, counts, offsets, bso, in_perm,
                         out_perm, diag, workspace, stream);
}

cudaError_t run_prepare_dispatch(const int32_t *ids, int64_t T, int k, int E, int A,
                                 int32_t *counts, int32_t *offsets, int32_t *bso,
                                 int32_t *in_perm, int32_t *out_perm, int32_t *diag,
                                 const void *x, int64_t row_bytes, void *out,
                                 cudaStream_t stream) {
    const int64_t S = T * k;
    const int64_t nvec = row_bytes / 16;
    const size_t smem = (S <= kSmallSlots ? small_smem(E, S) : single_block_smem(E)) +
                        (size_t)S * sizeof(int);
    // small batches: blocks of 256 threads (at least one thread per slot),
    // so that more SMs share the copy; larger ones: the 1024-thread block
    const int threads = S <= kSmallSlots ? (S <= 256 ? 256 : (int)((S + 31) / 32 * 32))
                                         : kSingleThreads;
    const int64_t units = (T * nvec + threads - 1) / threads;
    const int64_t grid = persistent_grid(prep_dispatch_kernel, threads, smem, units);
    return launch(prep_dispatch_kernel, grid, threads, smem, stream, Start::kEarly, ids, T, k, E, A,
                  counts, offsets, bso, in_perm, out_perm, diag, (const uint4 *)x, nvec,
                  (uint4 *)out);
}

}  // namespace moe
