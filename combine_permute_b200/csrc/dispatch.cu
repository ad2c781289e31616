// Dispatch: lay token rows out grouped by expert (sglang PR #19058,
// "Changes", item 2 shuffle_rows: dtype-agnostic row gather with 128-bit
// vector accesses), and the same with a fused FP8 E4M3 1x128 block-scale or
// NVFP4 quantisation (the FP8 block-scale and NVFP4 MoE paths of
// TensorRT-LLM PR #9592).
//
// dispatch_bulk_kernel is the scatter form on the TMA engine: it walks
// tokens, stages each x row in shared memory once and bulk-stores it to the
// token's k dispatched rows, so x crosses HBM once although it is written k
// times.  dispatch_gather_kernel walks dispatched rows and reads the source
// row through input_permutation (the literal shuffle_rows form, 16-byte
// vectors).  dispatch_quant_kernel quantises each token row once and stores
// the codes to its k rows.  All are persistent kernels sized to fill every
// SM once.
#include "kernels.h"
#include "launch.h"
#include "moe_device.cuh"

namespace moe {

namespace {

constexpr int kCopyThreads = 128;
constexpr int kCopyUnroll = 8;  // 16-byte vectors in flight per thread

// ---------------------------------------------------------------------------
// Scatter-form dispatch on the TMA engine.  One warp per block drives a ring
// of shared-memory stages: lane 0 bulk-loads a chunk of an x row
// (cp.async.bulk global -> shared, completing on an mbarrier), then lane j
// bulk-stores the staged chunk to dispatched row output_permutation[t*k+j]
// (cp.async.bulk shared -> global).  A stage is refilled once the stores of
// its previous chunk have finished reading it (bulk async-group wait).  The
// row is read from HBM once and written k times with one instruction per
// copy, so the load/store unit queues never throttle.  Each lane loads its
// destinations for the next unit while the current one is stored.  The host splits rows
// into `nch` chunks so that the (token, chunk) units spread evenly over the
// persistent grid.
// ---------------------------------------------------------------------------
constexpr int kBulkMaxStages = 16;
constexpr uint32_t kBulkSmem = 64 * 1024;   // stage ring per block
constexpr int kQuantThreads = 256;          // quantised dispatch: target threads per block
constexpr int kQuantMaxThreads = 512;       // and the most

// Set to 1 by a bulk dispatch block whose bounded wait for a staged chunk gave
// up (its rows are then incomplete); read and cleared by dispatch_error_kernel.
__device__ unsigned g_dispatch_error;

// Where the k copies of a token row go.  LocalRows: rows of this GPU's
// dispatched tensor, through output_permutation.  PeerRows: rows of the
// grouped buffers of R ranks (the fused exchange between GPUs), through each
// slot's destination rank and row; a buffer may be another GPU's memory
// (mapped into this process), reached by plain bulk stores.  The dispatch
// reads a slot's destination one unit ahead of its use in two steps: pre()
// loads it, finish() turns that into the row.  LocalRows does all of it in
// pre(); PeerRows leaves the checks and the address, which need the rank's
// row count and buffer, to finish(), so that pre() is loads that depend on
// nothing (measured both ways on B200, each form is the faster for its rows).
struct LocalRows {
    using Ref = int;
    using Pre = int;
    char *out;
    const int32_t *perm;
    int64_t S, row_bytes;
    __device__ Ref ref(int64_t i) const {
        const int p = __ldg(perm + i);
        return p >= 0 && p < S ? p : -1;
    }
    __device__ Pre pre(int64_t i) const { return ref(i); }
    __device__ static Pre no_pre() { return -1; }
    __device__ Ref finish(Pre p) const { return p; }
    __device__ static bool valid(Ref r) { return r >= 0; }
    __device__ char *addr(Ref r, int64_t off) const { return out + (int64_t)r * row_bytes + off; }
};

struct PeerRows {
    using Ref = char *;
    using Pre = int2;        // (rank, row)
    char *const *bufs;       // [R] each rank's grouped buffer
    const int32_t *rank;     // [S] destination rank of every slot (-1: none)
    const int32_t *row;      // [S] and its row there
    const int32_t *nrows;    // [R] rows of each buffer
    int R;
    int64_t row_bytes;
    __device__ Pre pre(int64_t i) const { return make_int2(__ldg(rank + i), __ldg(row + i)); }
    __device__ static Pre no_pre() { return make_int2(-1, -1); }
    __device__ Ref finish(Pre v) const {
        if (v.x < 0 || v.x >= R) return nullptr;
        if (v.y < 0 || v.y >= __ldg(nrows + v.x)) return nullptr;
        return bufs[v.x] + (int64_t)v.y * row_bytes;
    }
    __device__ Ref ref(int64_t i) const { return finish(pre(i)); }
    __device__ static bool valid(Ref r) { return r != nullptr; }
    __device__ char *addr(Ref r, int64_t off) const { return r + off; }
};

template <typename Rows>
__global__ void __launch_bounds__(32)
    dispatch_bulk_kernel(const char *__restrict__ x, int64_t T, int64_t row_bytes, int k,
                         const Rows rows, int64_t nch, uint32_t chunk, int stages,
                         uint32_t max_polls) {
    extern __shared__ __align__(128) unsigned char stage[];  // stages * chunk
    __shared__ __align__(8) uint64_t bar[kBulkMaxStages];
    const int lane = threadIdx.x;
    const int64_t units = T * nch;
    const int64_t mine =
        units > (int64_t)blockIdx.x ? (units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    if (lane == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    pdl_wait();

    auto load = [&](int64_t n) {  // lane 0: this block's unit n into stage n % stages
        const int64_t u = blockIdx.x + n * (int64_t)gridDim.x;
        const int64_t t = u / nch, off = (u - t * nch) * (int64_t)chunk;
        const uint32_t bytes = (uint32_t)min((int64_t)chunk, row_bytes - off);
        const int s = (int)(n % stages);
        mbar_expect_tx(&bar[s], bytes);
        bulk_g2s(stage + (size_t)s * chunk, x + t * row_bytes + off, bytes, &bar[s]);
    };
    int64_t issued = 0;
    if (lane == 0)
        for (; issued < stages && issued < mine; ++issued) load(issued);
    issued = __shfl_sync(0xffffffffu, issued, 0);

    // lane j's destinations of unit m (slots j and j + 32 of its token)
    auto pres = [&](int64_t m, typename Rows::Pre (&v)[2]) {
        const int64_t t = (blockIdx.x + m * (int64_t)gridDim.x) / nch;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = lane + 32 * h;
            v[h] = m < mine && j < k ? rows.pre(t * k + j) : Rows::no_pre();
        }
    };
    typename Rows::Pre vn[2];
    pres(0, vn);
    bool failed = false;
    int64_t n = 0;
    for (; n < mine; ++n) {
        const int64_t u = blockIdx.x + n * (int64_t)gridDim.x;
        const int64_t t = u / nch, off = (u - t * nch) * (int64_t)chunk;
        const uint32_t bytes = (uint32_t)min((int64_t)chunk, row_bytes - off);
        const int s = (int)(n % stages);
        const typename Rows::Ref p[2] = {rows.finish(vn[0]), rows.finish(vn[1])};
        pres(n + 1, vn);  // the next unit's, in flight while this one is stored
        const bool ok = mbar_wait(&bar[s], (uint32_t)((n / stages) & 1), max_polls);
        if (!__all_sync(0xffffffffu, ok)) {
            failed = true;
            break;
        }
        const unsigned char *src = stage + (size_t)s * chunk;
#pragma unroll
        for (int h = 0; h < 2; ++h)
            if (Rows::valid(p[h])) bulk_s2g(rows.addr(p[h], off), src, bytes);
        for (int j = lane + 64; j < k; j += 32) {  // top-k above 64
            const typename Rows::Ref pj = rows.ref(t * k + j);
            if (Rows::valid(pj)) bulk_s2g(rows.addr(pj, off), src, bytes);
        }
        bulk_commit();
        if (n >= 1) {
            bulk_wait_read<1>();  // this lane's stores of unit n-1 have read their stage
            __syncwarp();
            if (lane == 0 && issued < mine) load(issued);
            issued = __shfl_sync(0xffffffffu, issued < mine ? issued + 1 : issued, 0);
        }
    }
    pdl_launch_dependents();  // after the work loop: see pdl_launch_dependents
    if (failed) {
        if (lane == 0) atomicExch(&g_dispatch_error, 1u);
        // let every load still in flight land before the block releases its
        // shared memory (bounded by the default limit, whatever max_polls is)
        for (int64_t m = n; m < issued; ++m)
            mbar_wait(&bar[m % stages], (uint32_t)((m / stages) & 1), kDefaultDispatchPolls);
    }
    bulk_wait_all();
}

// Copies the error word to *out and clears it (one thread).
__global__ void dispatch_error_kernel(int32_t *out) {
    pdl_wait();
    pdl_launch_dependents();
    *out = (int32_t)atomicExch(&g_dispatch_error, 0u);
}

__global__ void __launch_bounds__(kCopyThreads)
    dispatch_gather_kernel(const uint4 *__restrict__ x, int64_t S, int64_t nvec, int k,
                           const int32_t *__restrict__ in_perm, uint4 *__restrict__ out) {
    pdl_wait();
    for (int64_t p = blockIdx.x; p < S; p += gridDim.x) {
        const int i = __ldg(in_perm + p);
        if (i < 0 || i >= S) continue;
        const uint4 *src = x + (int64_t)(i / k) * nvec;
        uint4 *dst = out + p * nvec;
        for (int64_t c0 = threadIdx.x; c0 < nvec; c0 += kCopyThreads * kCopyUnroll) {
            uint4 v[kCopyUnroll];
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) {
                const int64_t c = c0 + u * kCopyThreads;
                if (c < nvec) v[u] = ld_stream_v4(src + c);
            }
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) {
                const int64_t c = c0 + u * kCopyThreads;
                if (c < nvec) st_v4(dst + c, v[u]);
            }
        }
    }
    pdl_launch_dependents();
}

// Output memset (TensorRT-LLM PR #9592, moe_output_memset_inplace): zero the
// row of every token with at least one routed slot (output_permutation >= 0);
// other rows stay as they are.  One block per token at a time.
__global__ void __launch_bounds__(kCopyThreads)
    output_memset_kernel(uint4 *__restrict__ out, int64_t T, int64_t nvec, int k,
                         const int32_t *__restrict__ out_perm) {
    pdl_wait();
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        bool routed = false;
        for (int j = 0; j < k; ++j) routed |= __ldg(out_perm + t * k + j) >= 0;
        if (!routed) continue;
        uint4 *row = out + t * nvec;
        for (int64_t c = threadIdx.x; c < nvec; c += kCopyThreads) st_v4(row + c, make_uint4(0, 0, 0, 0));
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------------------
// FP8 dispatch.  Each thread owns 16 consecutive elements of a token row (two
// 16-byte loads); the 8 threads of one 128-column block reduce amax with
// shuffles, divide by s = amax / 448 in IEEE fp32 and convert pairs with
// cvt.rn.satfinite.e4m3x2.  The quantised row is computed once per token
// and stored to its k dispatched rows; the first thread of each block also
// stores s into the scale segment of the row's expert (found from the expert
// offsets, so the kernel needs no ids).
// ---------------------------------------------------------------------------

template <typename XT>
__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    const XT *h = reinterpret_cast<const XT *>(&v);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = Elem<XT>::to_f32(h[e]);
}

// FP8 E4M3 1x128 block quantisation of one 16-element group f (columns
// 16g .. 16g+15).  The 8 groups of a 128-column block sit in 8 consecutive
// lanes that are active together; `lanes` is the mask of the lanes of this
// warp still in the row loop.  Returns the 16 E4M3 bytes; *scale = amax/448.
__device__ __forceinline__ uint4 quant_fp8_group(const float *f, unsigned lanes, float *scale) {
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
    amax = fmaxf(amax, __shfl_xor_sync(lanes, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(lanes, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(lanes, amax, 4));
    uint4 packed = make_uint4(0u, 0u, 0u, 0u);
    float s = 0.0f;
    if (amax != 0.0f) {
        s = __fdiv_rn(amax, 448.0f);
        uint32_t w[4];
        if (s >= 0x1p-60f && s <= 0x1p60f) {
            // one reciprocal per block, three flops per element;
            // bit-identical to x / s (div_rn_recip)
            const float rs = __frcp_rn(s);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint16_t lo = cvt_e4m3x2(div_rn_recip(f[4 * e], s, rs),
                                               div_rn_recip(f[4 * e + 1], s, rs));
                const uint16_t hi = cvt_e4m3x2(div_rn_recip(f[4 * e + 2], s, rs),
                                               div_rn_recip(f[4 * e + 3], s, rs));
                w[e] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
        } else {  // scales near the ends of the fp32 range
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint16_t lo = cvt_e4m3x2(__fdiv_rn(f[4 * e], s), __fdiv_rn(f[4 * e + 1], s));
                const uint16_t hi =
                    cvt_e4m3x2(__fdiv_rn(f[4 * e + 2], s), __fdiv_rn(f[4 * e + 3], s));
                w[e] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
        }
        packed = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *scale = s;
    return packed;
}

// NVFP4 quantisation of one 16-element group: the E4M3 scale
// sf = e4m3(amax / 6) and the 16 E2M1 codes of x / value(sf), element 2m in
// the low nibble of byte m.  Returns the 8 code bytes; *sf_out = sf.
__device__ __forceinline__ uint2 quant_nvfp4_group(const float *f, uint8_t *sf_out) {
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
    const uint16_t sf = cvt_e4m3x2(__fdiv_rn(amax, 6.0f), 0.0f) & 0xffu;
    const float d = e4m3_to_f32(sf);
    uint2 packed = make_uint2(0u, 0u);
    if (d != 0.0f) {  // d is an E4M3 value: in [2^-9, 448]
        const float rd = __frcp_rn(d);
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 16; e += 2)
            w[e >> 3] |= cvt_e2m1x2(div_rn_recip(f[e], d, rd), div_rn_recip(f[e + 1], d, rd))
                         << (4 * (e & 7));
        packed = make_uint2(w[0], w[1]);
    }
    *sf_out = (uint8_t)sf;
    return packed;
}

// Lanes of this warp still in a loop over groups g = threadIdx.x + i*blockDim.x
// < n (blockDim.x a multiple of 32): all of them, or those below the row end.
__device__ __forceinline__ unsigned lanes_in_row(int64_t g, int64_t n) {
    const int64_t rem = n - (g - (threadIdx.x & 31));
    return rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
}

// Stages the expert offsets and (block-scale row - dispatched row) per
// expert, then for token t resolves its k dispatched rows and their scale
// rows into s_p / s_srow (-1 for slots with no row).  Threads j < k write.
__device__ __forceinline__ void stage_offsets(const int32_t *offsets, const int32_t *bso, int E,
                                              int *s_off, int *s_delta) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
        s_off[e] = __ldg(offsets + e);
        if (e < E) s_delta[e] = __ldg(bso + e) - __ldg(offsets + e);
    }
}

__device__ __forceinline__ void resolve_rows(const int32_t *out_perm, int64_t t, int k, int64_t S,
                                             int E, const int *s_off, const int *s_delta,
                                             int *s_p, int *s_srow) {
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
        int p = __ldg(out_perm + t * k + j);
        int srow = -1;
        if (p >= 0 && p < S && p < s_off[E]) {
            int lo = 0, hi = E;  // the expert whose rows hold p
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (s_off[mid] <= p) lo = mid;
                else hi = mid;
            }
            srow = p + s_delta[lo];
        } else {
            p = -1;
        }
        s_p[j] = p;
        s_srow[j] = srow;
    }
}

// Quantised dispatch.  A block walks tokens; each thread owns one or two
// 16-element groups of the row (longer rows: a loop over groups).  Per
// group: the quantiser, then its code bytes stored to each of the k
// dispatched rows, plus the scale from the lane that leads its scale block.
template <typename XT, bool kFp4>
__device__ __forceinline__ void quant_store_group(const uint4 &raw0, const uint4 &raw1, int64_t g,
                                                  int64_t n16, int64_t qrow, int64_t srow_len,
                                                  int k, const int *s_p, const int *s_srow,
                                                  uint8_t *__restrict__ q, void *__restrict__ scales) {
    float f[16];
    unpack8<XT>(raw0, f);
    unpack8<XT>(raw1, f + 8);
    if constexpr (kFp4) {
        uint8_t sf;
        const uint2 packed = quant_nvfp4_group(f, &sf);
        for (int j = 0; j < k; ++j) {
            const int p = s_p[j];
            if (p < 0) continue;
            *reinterpret_cast<uint2 *>(q + (int64_t)p * qrow + g * 8) = packed;
            static_cast<uint8_t *>(scales)[(int64_t)s_srow[j] * srow_len + g] = sf;
        }
    } else {
        float sc;
        const uint4 packed = quant_fp8_group(f, lanes_in_row(g, n16), &sc);
        const bool block_lead = (g & 7) == 0;
        for (int j = 0; j < k; ++j) {
            const int p = s_p[j];
            if (p < 0) continue;
            st_v4(q + (int64_t)p * qrow + g * 16, packed);
            if (block_lead)
                static_cast<float *>(scales)[(int64_t)s_srow[j] * srow_len + (g >> 3)] = sc;
        }
    }
}

template <typename XT, bool kFp4, int kG>
__global__ void __launch_bounds__(kQuantMaxThreads)
    dispatch_quant_kernel(const XT *__restrict__ x, int64_t T, int64_t H, int k, int E,
                          const int32_t *__restrict__ out_perm, const int32_t *__restrict__ offsets,
                          const int32_t *__restrict__ bso, uint8_t *__restrict__ q,
                          void *__restrict__ scales) {
    extern __shared__ int smem[];
    int *s_off = smem;             // [E+1] expert offsets
    int *s_delta = s_off + E + 1;  // [E] scale row - dispatched row, per expert
    int *s_p = s_delta + E;        // [k] this token's dispatched rows
    int *s_srow = s_p + k;         // [k] and their scale rows
    const int64_t n16 = H / 16;  // 16-element groups per row
    const int64_t S = T * k;
    const int64_t qrow = kFp4 ? H / 2 : H;
    const int64_t srow_len = kFp4 ? n16 : H / 128;  // scale elements per row
    const int64_t nt = blockDim.x;
    // kG > 0: the row has at most kG * blockDim.x groups; thread i owns
    // groups i + r * blockDim.x (r < kG) of every token, and loads the next
    // token's while this one's are quantised and stored.
    uint4 nxt[kG > 0 ? 2 * kG : 1];
    auto prefetch = [&](int64_t t) {
#pragma unroll
        for (int r = 0; r < kG; ++r) {
            const int64_t g = threadIdx.x + r * nt;
            if (g < n16 && t < T) {
                const XT *src = x + t * H + g * 16;
                nxt[2 * r] = ld_stream_v4(src);
                nxt[2 * r + 1] = ld_stream_v4(src + 8);
            }
        }
    };
    pdl_wait();
    if constexpr (kG > 0) prefetch(blockIdx.x);
    stage_offsets(offsets, bso, E, s_off, s_delta);
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        if constexpr (kG > 0) {
            uint4 cur[2 * kG];
#pragma unroll
            for (int r = 0; r < 2 * kG; ++r) cur[r] = nxt[r];
            prefetch(t + gridDim.x);  // in flight while this token is stored
            __syncthreads();  // offsets staged; the previous token's rows consumed
            resolve_rows(out_perm, t, k, S, E, s_off, s_delta, s_p, s_srow);
            __syncthreads();
#pragma unroll
            for (int r = 0; r < kG; ++r) {
                const int64_t g = threadIdx.x + r * nt;
                if (g < n16)
                    quant_store_group<XT, kFp4>(cur[2 * r], cur[2 * r + 1], g, n16, qrow, srow_len,
                                                k, s_p, s_srow, q, scales);
            }
        } else {
            __syncthreads();
            resolve_rows(out_perm, t, k, S, E, s_off, s_delta, s_p, s_srow);
            __syncthreads();
            for (int64_t g = threadIdx.x; g < n16; g += nt) {
                const XT *src = x + t * H + g * 16;
                quant_store_group<XT, kFp4>(ld_stream_v4(src), ld_stream_v4(src + 8), g, n16, qrow,
                                            srow_len, k, s_p, s_srow, q, scales);
            }
        }
    }
    pdl_launch_dependents();
}

}  // namespace

// Row split for the bulk dispatch.  When the batch fills the persistent
// grid, chunks of about kBulkChunkTarget bytes (16 stages in the ring):
// measured on B200, 14336-byte rows ran at 0.757 of 8 TB/s cut in four
// (3584-byte chunks) against 0.694-0.705 whole or cut in two, three or
// seven, and 4096-byte rows were best whole.  Otherwise (few tokens) the
// number of chunks per row that minimises (units per block) x (bytes per
// unit + a per-unit overhead), the makespan of a persistent grid of
// `grid_max` blocks.
constexpr int64_t kBulkChunkTarget = 4096;

static int64_t bulk_split(int64_t T, int64_t row_bytes, int64_t grid_max) {
    int64_t target = (row_bytes + kBulkChunkTarget / 2) / kBulkChunkTarget;
    if (target < 1) target = 1;
    if (target > 16) target = 16;
    if (T * target >= grid_max) return target;
    constexpr int64_t kUnitOverheadBytes = 1024;
    int64_t best_n = 1, best_cost = -1;
    for (int64_t n = 1; n <= 16; ++n) {
        const int64_t chunk = ((row_bytes + n - 1) / n + 15) / 16 * 16;
        if (chunk > kBulkSmem / 2) continue;  // at least two stages
        const int64_t nch = (row_bytes + chunk - 1) / chunk;
        const int64_t units = T * nch;
        const int64_t grid = units < grid_max ? units : grid_max;
        const int64_t per = (units + grid - 1) / grid;
        const int64_t cost = per * (chunk + kUnitOverheadBytes);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best_n = n;
        }
        if (chunk <= 16) break;
    }
    return best_n;
}

template <typename Rows>
static cudaError_t launch_bulk(const void *x, int64_t T, int64_t row_bytes, int k,
                               const Rows &rows, int64_t nsplit, cudaStream_t stream) {
    // chunks of the row, at least two of which fit the stage ring
    auto chunk_of = [&](int64_t ns) {
        return (uint32_t)(((row_bytes + ns - 1) / ns + 15) / 16 * 16);
    };
    constexpr int64_t kMaxChunk = kBulkSmem / 2;
    if (nsplit < (row_bytes + kMaxChunk - 1) / kMaxChunk)
        nsplit = (row_bytes + kMaxChunk - 1) / kMaxChunk;
    uint32_t chunk = chunk_of(nsplit);
    while (chunk > kMaxChunk) chunk = chunk_of(++nsplit);  // rounding up to 16 bytes
    const int64_t nch = (row_bytes + chunk - 1) / chunk;
    int stages = (int)(kBulkSmem / chunk);
    if (stages > kBulkMaxStages) stages = kBulkMaxStages;
    const size_t smem = (size_t)stages * chunk;
    auto kern = dispatch_bulk_kernel<Rows>;
    const int64_t grid = persistent_grid(kern, 32, smem, T * nch);
    return launch(kern, grid, 32, smem, stream, streaming_start(T * k * row_bytes), (const char *)x,
                  T, row_bytes, k, rows, nch, chunk, stages, dispatch_polls().load());
}

cudaError_t run_dispatch_scatter_split(const void *x, int64_t T, int64_t row_bytes, int k,
                                       const int32_t *out_perm, void *out, int64_t nsplit,
                                       cudaStream_t stream) {
    return launch_bulk(x, T, row_bytes, k, LocalRows{(char *)out, out_perm, T * k, row_bytes},
                       nsplit, stream);
}

cudaError_t run_dispatch_error(int32_t *out, cudaStream_t stream) {
    return launch(dispatch_error_kernel, 1, 1, 0, stream, Start::kEarly, out);
}

static int64_t bulk_grid_max() {
    return (int64_t)sm_count() * blocks_per_sm(dispatch_bulk_kernel<LocalRows>, 32, kBulkSmem);
}

cudaError_t run_dispatch_scatter(const void *x, int64_t T, int64_t row_bytes, int k,
                                 const int32_t *out_perm, void *out, cudaStream_t stream) {
    return run_dispatch_scatter_split(x, T, row_bytes, k, out_perm, out,
                                      bulk_split(T, row_bytes, bulk_grid_max()), stream);
}

cudaError_t run_dispatch_peer(const void *x, int64_t T, int64_t row_bytes, int k,
                              const int32_t *dest_rank, const int32_t *dest_row,
                              void *const *bufs, const int32_t *nrows, int R, cudaStream_t stream) {
    const PeerRows rows{(char *const *)bufs, dest_rank, dest_row, nrows, R, row_bytes};
    return launch_bulk(x, T, row_bytes, k, rows, bulk_split(T, row_bytes, bulk_grid_max()),
                       stream);
}

cudaError_t run_dispatch_gather(const void *x, int64_t T, int64_t row_bytes, int k,
                                const int32_t *in_perm, void *out, cudaStream_t stream) {
    const int64_t nvec = row_bytes / 16;
    const int64_t S = T * k;
    const int64_t grid = persistent_grid(dispatch_gather_kernel, kCopyThreads, 0, S);
    return launch(dispatch_gather_kernel, grid, kCopyThreads, 0, stream,
                  streaming_start(S * row_bytes), (const uint4 *)x, S, nvec, k, in_perm,
                  (uint4 *)out);
}

// Quantised dispatch launcher.  Rows of up to 2 * kQuantThreads groups:
// kG = ceil(groups / kQuantThreads) groups per thread (1 or 2) and
// ceil(groups / kG) threads rounded up to a multiple of 32 (so that the 8
// groups of an FP8 128-column block share a warp).  Longer rows: a plain
// loop without the prefetch.
template <typename XT, bool kFp4>
static cudaError_t run_dispatch_quant_t(const XT *x, int64_t T, int64_t H, int k, int E,
                                        const int32_t *out_perm, const int32_t *offsets,
                                        const int32_t *bso, uint8_t *q, void *scales,
                                        cudaStream_t stream) {
    const int64_t n16 = H / 16;
    const size_t smem = (size_t)(2 * E + 1 + 2 * k) * sizeof(int);
    auto go = [&](auto kern, int64_t per_thread) {
        int64_t threads = ((n16 + per_thread - 1) / per_thread + 31) / 32 * 32;
        if (threads > kQuantMaxThreads) threads = kQuantMaxThreads;
        const int64_t grid = persistent_grid(kern, (int)threads, smem, T);
        return launch(kern, grid, (int)threads, smem, stream, streaming_start(T * k * H), x, T, H,
                      k, E, out_perm, offsets, bso, q, scales);
    };
    if (n16 <= kQuantThreads) return go(dispatch_quant_kernel<XT, kFp4, 1>, 1);
    if (n16 <= 2 * kQuantThreads) return go(dispatch_quant_kernel<XT, kFp4, 2>, 2);
    return go(dispatch_quant_kernel<XT, kFp4, 0>, (n16 + kQuantMaxThreads - 1) / kQuantMaxThreads);
}

cudaError_t run_dispatch_fp8(const void *x, DType x_dtype, int64_t T, int64_t H, int k, int E,
                             const int32_t *out_perm, const int32_t *offsets, const int32_t *bso,
                             uint8_t *q, float *scales, cudaStream_t stream) {
    if (x_dtype == DType::BF16)
        return run_dispatch_quant_t<__nv_bfloat16, false>((const __nv_bfloat16 *)x, T, H, k, E,
                                                          out_perm, offsets, bso, q, scales, stream);
    return run_dispatch_quant_t<__half, false>((const __half *)x, T, H, k, E, out_perm, offsets,
                                               bso, q, scales, stream);
}

cudaError_t run_dispatch_nvfp4(const void *x, DType x_dtype, int64_t T, int64_t H, int k, int E,
                               const int32_t *out_perm, const int32_t *offsets, const int32_t *bso,
                               uint8_t *q, uint8_t *scales, cudaStream_t stream) {
    if (x_dtype == DType::BF16)
        return run_dispatch_quant_t<__nv_bfloat16, true>((const __nv_bfloat16 *)x, T, H, k, E,
                                                         out_perm, offsets, bso, q, scales, stream);
    return run_dispatch_quant_t<__half, true>((const __half *)x, T, H, k, E, out_perm, offsets, bso,
                                              q, scales, stream);
}

cudaError_t run_output_memset(void *out, int64_t T, int64_t row_bytes, int k,
                              const int32_t *out_perm, cudaStream_t stream) {
    const int64_t grid = persistent_grid(output_memset_kernel, kCopyThreads, 0, T);
    return launch(output_memset_kernel, grid, kCopyThreads, 0, stream,
                  streaming_start(T * row_bytes), (uint4 *)out, T, row_bytes / 16, k, out_perm);
}

}  // namespace moe
