/*
 * moe.h - C ABI of the single-GPU MoE dispatch / combine library (libmoe.so,
 * CUDA kernels for sm_100a).
 *
 * The path has three steps, named after the kernels of sglang PR #19058
 * "[jit_kernel] Add prepare_moe_input JIT kernels", section "Changes":
 *
 *   1. moe_prepare         routing metadata (prepare_moe_input: tokens per
 *                          expert, prefix-sum expert offsets, optional FP8
 *                          block-scale offsets, input/output permutations);
 *   2. moe_dispatch_rows   the row gather that lays token rows out grouped by
 *                          expert (shuffle_rows), and moe_dispatch_rows_fp8,
 *                          the same with a fused FP8 E4M3 1x128 block-scale
 *                          quantisation (the FP8 block-scale MoE path of
 *                          TensorRT-LLM PR #9592);
 *   3. moe_combine         gather + scale by router weight + reduce over the
 *                          k slots with fp32 accumulation
 *                          (apply_shuffle_mul_sum).
 *
 * Notation: T tokens, H hidden size, E experts, k slots per token (top-k),
 * S = T*k.  The expanded index of slot j of token t is i = t*k + j; the
 * permuted index p is the row of the dispatched (expert-grouped) tensor
 * (TensorRT-LLM PR #9592 names these expanded_idx / permuted_idx).
 *
 * Conventions shared by every entry point:
 *  - All array arguments are caller-owned DEVICE memory, row-major and
 *    densely packed.  The library never allocates device or host memory and
 *    keeps no state between calls apart from a per-device cache of launch
 *    sizes (guarded by a mutex).
 *  - Every call is asynchronous: it validates its arguments on the host,
 *    enqueues its kernels on `stream` (NULL = the legacy default stream) and
 *    returns without synchronising.  Kernels are launched with programmatic
 *    dependent launch, so consecutive calls on one stream overlap their
 *    launch latency while still seeing each other's results.
 *  - Host-side validation failures return MOE_ERR_INVALID_ARG or
 *    MOE_ERR_UNSUPPORTED and launch nothing.  A failed launch returns
 *    MOE_ERR_CUDA (the CUDA error is consumed with cudaGetLastError).
 *  - Outputs must not alias inputs.
 *  - Index tensors are int32; T*k must be < 2^31.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the same pointer type; this header does not need the CUDA
 * headers). */
typedef struct CUstream_st *moe_stream_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad alignment ... */
    MOE_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels support    */
    MOE_ERR_WORKSPACE = 3,   /* workspace missing or too small                */
    MOE_ERR_CUDA = 4         /* a CUDA launch or runtime call failed          */
} moe_status_t;

typedef enum {
    MOE_F32 = 0,
    MOE_F16 = 1,
    MOE_BF16 = 2,
    MOE_FP8_E4M3 = 3 /* OCP E4M3 "FN": no infinities, max finite 448 */
} moe_dtype_t;

typedef enum {
    MOE_I32 = 0, /* int32 expert ids                                   */
    MOE_I64 = 1  /* int64 expert ids (the Mooncake top-k index type)   */
} moe_index_t;

/* Largest expert count the prepare kernels accept. */
#define MOE_MAX_EXPERTS 1024

/* Human-readable name of a status code (static storage, never NULL). */
const char *moe_status_string(moe_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
int32_t moe_version(void);

/* Name and description of the CUDA error behind the calling thread's most
 * recent MOE_ERR_CUDA ("no CUDA error" if there was none).  The string is
 * thread-local and valid until the thread's next failing call. */
const char *moe_last_cuda_error(void);

/*
 * Bytes of scratch workspace moe_prepare needs for this problem size: 0 up
 * to 4096 slots (T*k), which run in one block without one.  The workspace
 * must be all-zero before its first use (e.g. one cudaMemsetAsync); the
 * library maintains it from then on (it holds a call counter and look-back
 * words tagged with it, so it is not all-zero between calls), and one
 * workspace serves any number of consecutive calls of any size on one
 * stream.  Zero it again only as a whole, and after a call that reported a
 * CUDA error.  Calls that may run concurrently need separate workspaces.
 */
size_t moe_prepare_workspace_bytes(int64_t num_tokens, int32_t top_k, int32_t num_experts);

/*
 * Routing metadata (sglang PR #19058, "Changes", item 1 prepare_moe_input:
 * compute_problem_sizes_kernel counts tokens per expert,
 * compute_expert_offsets_kernel prefix-sums them,
 * compute_expert_blockscale_offsets_kernel gives the optional FP8
 * block-scale offsets, compute_arg_sorts_kernel builds the input and output
 * permutations).
 *
 *   topk_ids            [T, k] int32   expert id of every slot.
 *   expert_counts       [E]    int32   out: slots routed to each expert.
 *   expert_offsets      [E+1]  int32   out: exclusive prefix sum of the
 *                                      counts; expert_offsets[E] is the
 *                                      number of valid slots.
 *   blockscale_offsets  [E+1]  int32   out, optional (NULL to skip):
 *                                      exclusive prefix sum of the counts
 *                                      each rounded up to a multiple of
 *                                      blockscale_align (>= 1).
 *   input_permutation   [T*k]  int32   out: input_permutation[p] = i, the
 *                                      expanded index of dispatched row p;
 *                                      -1 for p >= expert_offsets[E].
 *   output_permutation  [T*k]  int32   out: the inverse, output_permutation[i]
 *                                      = p; -1 for slots with an invalid id.
 *   diag                [2]    int32   out, optional: diag[0] = number of ids
 *                                      outside [0, E); diag[1] = 1 if a
 *                                      bounded inter-block wait gave up (the
 *                                      other outputs are then invalid), else
 *                                      0.  A wait gives up after about one
 *                                      second (moe_set_wait_limits); the
 *                                      kernel still ends and the call's
 *                                      stream stays usable.  A workspace
 *                                      whose counters were disturbed (not
 *                                      zeroed before first use, or written
 *                                      by anything but the library) shows
 *                                      up here: zero it and call again.
 *   workspace                          scratch of moe_prepare_workspace_bytes()
 *                                      bytes, 256-byte aligned, zeroed before
 *                                      its first use and then left to the
 *                                      library (see above); may be NULL when
 *                                      that size is 0.
 *
 * Batches of up to 4096 slots run in one block; larger ones as tiles over
 * the whole GPU (the only case that touches the workspace): one cooperative
 * launch with one grid barrier when every tile fits on the GPU at once (up
 * to 64 rounds of 512 slots per SM and the SM's shared memory: about 4.8
 * million slots on B200 with 64 experts, 3.8 million with 256), else two
 * kernels with a decoupled look-back between tiles.
 *
 * Dispatched order: by expert ascending, and within an expert by expanded
 * index ascending (token, then slot): a stable counting sort, so the result
 * is deterministic.  Ids outside [0, E) are not counted and get no row; the
 * call still succeeds (check diag[0]).  T = 0 writes zero counts/offsets;
 * topk_ids and the permutations may then be NULL.
 */
moe_status_t moe_prepare(const int32_t *topk_ids, int64_t num_tokens, int32_t top_k,
                         int32_t num_experts, int32_t *expert_counts, int32_t *expert_offsets,
                         int32_t *blockscale_offsets, int32_t blockscale_align,
                         int32_t *input_permutation, int32_t *output_permutation, int32_t *diag,
                         void *workspace, size_t workspace_bytes, moe_stream_t stream);

/*
 * Dispatch (sglang PR #19058, "Changes", item 2 shuffle_rows: a
 * dtype-agnostic row gather with 128-bit vector accesses):
 *
 *   out[p, :] = x[input_permutation[p] / k, :]   for every p with
 *                                                 input_permutation[p] >= 0.
 *
 *   x       [T, H]   element type `dtype` (F32, F16 or BF16); H * sizeof
 *                    must be a multiple of 16 bytes, x and out 16-byte
 *                    aligned.
 *   out     [T*k, H] same type; rows that no valid slot maps to are not
 *                    written.
 *   input_permutation / output_permutation  [T*k] int32 as produced by
 *                    moe_prepare.  At least one must be non-NULL.  When
 *                    output_permutation is given the kernel walks tokens and
 *                    reads every x row once, writing it to its k rows
 *                    (output_permutation must then be the inverse of the
 *                    permutation that defines the result); otherwise it
 *                    walks the dispatched rows and gathers through
 *                    input_permutation.
 */
moe_status_t moe_dispatch_rows(const void *x, moe_dtype_t dtype, int64_t num_tokens,
                               int64_t hidden, int32_t top_k, const int32_t *input_permutation,
                               const int32_t *output_permutation, void *out, moe_stream_t stream);

/*
 * Failure report of the TMA dispatch (the scatter form of moe_dispatch_rows,
 * taken when output_permutation is given).  Each of its blocks waits,
 * bounded, for every chunk of x it stages in shared memory; a block whose
 * wait gave up stops, lets its copies in flight finish and sets a device
 * error word, so the call's rows are then incomplete although the call
 * returned MOE_OK.  This enqueues on `stream` one tiny kernel that writes
 * that word to *error (device memory, int32: 1 if some wait gave up since
 * the previous query on this device, else 0) and clears it.  Order it after
 * the dispatches it should cover.  No counterpart in the pages (they give
 * no failure reporting); it is this library's bounded-wait contract.
 * Errors: MOE_ERR_INVALID_ARG for a NULL `error`.
 */
moe_status_t moe_dispatch_error(int32_t *error, moe_stream_t stream);

/*
 * Limits of the bounded waits, for tests of the failure reporting:
 *   prepare_wait_us   how long a prepare block waits for other blocks, in
 *                     microseconds of the GPU's global timer (default
 *                     1000000, one second); 0 gives up at the first check
 *                     that finds the awaited value missing.
 *   dispatch_polls    mbarrier polls the TMA dispatch makes for one staged
 *                     chunk (default 2^24); 0 gives up at once.
 * A negative value restores that default.  The limits apply, process-wide,
 * to every launch made after the call (a CUDA graph keeps those it was
 * captured with).  Lower them only to test the failure reporting: a wait
 * that gives up leaves that call's outputs invalid.  Never fails.
 */
moe_status_t moe_set_wait_limits(int64_t prepare_wait_us, int64_t dispatch_polls);

/*
 * Dispatch with FP8 E4M3 1x128 block-scale quantisation (TensorRT-LLM PR
 * #9592, FP8 block-scale MoE path, "run_moe_fp8_block_scales"; the optional
 * FP8 block-scale offsets of sglang PR #19058 place the scales).  For every
 * valid slot i = t*k + j with p = output_permutation[i] >= 0, e the expert
 * whose rows [expert_offsets[e], expert_offsets[e+1]) hold p, and every
 * 128-column block b:
 *
 *   amax = max |x[t, 128b .. 128b+127]|      (in fp32)
 *   s    = amax / 448                         (fp32, round to nearest)
 *   out_q[p, c] = e4m3_rn_satfinite(x[t, c] / s)   (fp32 division)
 *   out_scales[blockscale_offsets[e] + p - expert_offsets[e], b] = s
 *
 * A block with amax = 0 gets s = 0 and zero bytes.  Rows of out_q and
 * scale rows that no valid slot maps to (including the padding rows of each
 * expert's scale segment) are not written.  The expert of a row comes from
 * the offsets, so any id type or expert window of moe_prepare_local works.
 *
 *   x          [T, H] BF16 or F16, H a multiple of 128, 16-byte aligned.
 *   output_permutation [T*k] int32;
 *   expert_offsets / blockscale_offsets [E+1] int32 (from moe_prepare).
 *   out_q      [T*k, H] uint8 (E4M3 bytes); out_scales [rows, H/128] fp32
 *              with rows >= blockscale_offsets[E].
 */
moe_status_t moe_dispatch_rows_fp8(const void *x, moe_dtype_t x_dtype, int64_t num_tokens,
                                   int64_t hidden, int32_t top_k, int32_t num_experts,
                                   const int32_t *output_permutation,
                                   const int32_t *expert_offsets,
                                   const int32_t *blockscale_offsets, uint8_t *out_q,
                                   float *out_scales, moe_stream_t stream);

/*
 * Dispatch with NVFP4 quantisation (TensorRT-LLM PR #9592: the B200/GB200
 * NVFP4 MoE path, "run_moe_nvfp4", with scaling_vector_size = 16).  The
 * pages name the format and the block size only; this library takes the
 * plain reading of it: one E4M3 scale per 16 consecutive elements of a row,
 * FP4 E2M1 elements, no per-tensor global scale.  For every valid slot
 * i = t*k + j with p = output_permutation[i] >= 0, e the expert whose rows
 * hold p, and every 16-column group g:
 *
 *   amax = max |x[t, 16g .. 16g+15]|                 (in fp32)
 *   sf   = e4m3_rn_satfinite(amax / 6)               (fp32 division)
 *   d    = the value of sf
 *   code(c) = e2m1_rn_satfinite(x[t, c] / d)         (fp32 division; 0 if d = 0)
 *   out_q[p, c/2] holds code(c) in bits 0..3 for even c, bits 4..7 for odd c
 *   out_scales[blockscale_offsets[e] + p - expert_offsets[e], g] = sf
 *
 * E2M1 magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6 (sign in bit 3); rounding is
 * to nearest, ties to the even code, and magnitudes above 6 saturate.
 * Rows and scale rows that no valid slot maps to are not written.
 *
 *   x          [T, H] BF16 or F16, H a multiple of 16, 16-byte aligned.
 *   output_permutation [T*k] int32;
 *   expert_offsets / blockscale_offsets [E+1] int32 (from moe_prepare).
 *   out_q      [T*k, H/2] uint8, 8-byte aligned;
 *   out_scales [rows, H/16] uint8 (E4M3 bytes), rows >= blockscale_offsets[E].
 * Errors: MOE_ERR_UNSUPPORTED for an x type other than BF16/F16;
 * MOE_ERR_INVALID_ARG for H not a multiple of 16, NULL or misaligned buffers.
 */
moe_status_t moe_dispatch_rows_nvfp4(const void *x, moe_dtype_t x_dtype, int64_t num_tokens,
                                     int64_t hidden, int32_t top_k, int32_t num_experts,
                                     const int32_t *output_permutation,
                                     const int32_t *expert_offsets,
                                     const int32_t *blockscale_offsets, uint8_t *out_q,
                                     uint8_t *out_scales, moe_stream_t stream);

/*
 * Combine (sglang PR #19058, "Changes", item 3 apply_shuffle_mul_sum:
 * gather + scale + reduce, fp32 accumulation, fp16 / bf16 / fp32):
 *
 *   out[t, h] = round_out( sum_{j=0}^{k-1} weights[t, j] *
 *                          y[output_permutation[t*k + j], h] )
 *
 * The sum runs over j in ascending order in fp32, each product and each sum
 * rounded separately (no fused multiply-add); the result is rounded once to
 * `out_dtype` (round to nearest even).  Slots with output_permutation = -1
 * contribute nothing.
 *
 *   y        [T*k, H] F32, F16 or BF16 (expert outputs in dispatched order).
 *   weights  [T, k]   fp32 router weights.
 *   out      [T, H]   F32, F16 or BF16.
 *   H * sizeof(y element) and H * sizeof(out element) must be multiples of
 *   16 bytes; y and out 16-byte aligned.
 */
moe_status_t moe_combine(const void *y, moe_dtype_t y_dtype, int64_t num_tokens, int64_t hidden,
                         int32_t top_k, const int32_t *output_permutation, const float *weights,
                         void *out, moe_dtype_t out_dtype, moe_stream_t stream);

/*
 * Problem sizes of the two grouped GEMMs that follow dispatch (sglang PR
 * #19058, "Changes", item 1: compute_problem_sizes_kernel fills
 * problem_sizes1 / problem_sizes2): for every expert e,
 *
 *   problem_sizes1[e] = {expert_counts[e], n1, k1}
 *   problem_sizes2[e] = {expert_counts[e], n2, k2}      (M, N, K)
 *
 * e.g. n1 = 2 * intermediate, k1 = hidden for the gate/up projection and
 * n2 = hidden, k2 = intermediate for the down projection.
 *
 *   expert_counts    [E]    int32 (from moe_prepare)
 *   problem_sizes1   [E, 3] int32 out; problem_sizes2 [E, 3] int32 out or NULL
 */
moe_status_t moe_problem_sizes(const int32_t *expert_counts, int32_t num_experts, int32_t n1,
                               int32_t k1, int32_t n2, int32_t k2, int32_t *problem_sizes1,
                               int32_t *problem_sizes2, moe_stream_t stream);

/*
 * Tile-padded layout for a tiled grouped GEMM (TensorRT-LLM PR #9592, the
 * moe_sort outputs tile_idx_to_group_idx, tile_idx_to_mn_limit,
 * expanded_idx_to_permuted_idx, permuted_idx_to_expanded_idx,
 * total_num_padded_tokens, num_non_exiting_tiles).  Every expert's rows are
 * padded up to a multiple of tile_size:
 *
 *   padded_offsets[e]  = sum over e' < e of roundup(expert_counts[e'], tile)
 *   tile t < num_non_exiting_tiles belongs to the expert e whose padded
 *     range holds row t*tile_size: tile_idx_to_group_idx[t] = e and
 *     tile_idx_to_mn_limit[t] = padded_offsets[e] + expert_counts[e] (the
 *     end of that expert's real rows); later tiles up to max_tiles get -1
 *     in both;
 *   a slot i with dispatched row p = output_permutation[i] >= 0 of expert e
 *     is on padded row expanded_idx_to_permuted_idx[i] =
 *     padded_offsets[e] + p - expert_offsets[e] (-1 for unrouted slots);
 *   permuted_idx_to_expanded_idx is its inverse over all max_tiles *
 *     tile_size rows, -1 on padding rows and past the padded total.
 *
 *   expert_counts [E], expert_offsets [E+1], output_permutation [T*k]
 *                                      int32, from moe_prepare / _local
 *   padded_offsets [E+1], tile_idx_to_group_idx [max_tiles],
 *   tile_idx_to_mn_limit [max_tiles], expanded_idx_to_permuted_idx [T*k],
 *   permuted_idx_to_expanded_idx [max_tiles * tile_size],
 *   num_non_exiting_tiles [1], total_num_padded_tokens [1]   int32 out
 *
 * max_tiles = ceil(T*k / tile_size) + min(E, T*k) always suffices.  When
 * max_tiles * tile_size is smaller than the padded total (known only on the
 * device), num_non_exiting_tiles is set to -1, total_num_padded_tokens and
 * padded_offsets hold the needed sizes and nothing else is written.
 */
moe_status_t moe_tile_layout(int64_t num_tokens, int32_t top_k, int32_t num_experts,
                             int32_t tile_size, const int32_t *expert_counts,
                             const int32_t *expert_offsets, const int32_t *output_permutation,
                             int32_t max_tiles, int32_t *padded_offsets,
                             int32_t *tile_idx_to_group_idx, int32_t *tile_idx_to_mn_limit,
                             int32_t *expanded_idx_to_permuted_idx,
                             int32_t *permuted_idx_to_expanded_idx,
                             int32_t *num_non_exiting_tiles, int32_t *total_num_padded_tokens,
                             moe_stream_t stream);

/*
 * moe_prepare for one rank's window of experts and for int64 ids (the
 * local-expert slice local_expert_offset / num_local_experts of TensorRT-LLM
 * PR #9592's grouped GEMM, and Mooncake PR #4581's int64 top-k index type).
 * Slot i belongs to local expert topk_ids[i] - local_expert_offset when that
 * lies in [0, num_local_experts); every other slot is excluded exactly as an
 * invalid id is in moe_prepare (not counted, output_permutation -1, counted
 * in diag[0]).  All outputs are sized by num_local_experts (E below); the
 * workspace is moe_prepare_workspace_bytes(T, k, num_local_experts).
 *
 *   topk_ids  [T, k] int32 (id_type MOE_I32) or int64 (MOE_I64).
 *   The other arguments are those of moe_prepare.
 */
moe_status_t moe_prepare_local(const void *topk_ids, moe_index_t id_type, int64_t num_tokens,
                               int32_t top_k, int64_t local_expert_offset,
                               int32_t num_local_experts, int32_t *expert_counts,
                               int32_t *expert_offsets, int32_t *blockscale_offsets,
                               int32_t blockscale_align, int32_t *input_permutation,
                               int32_t *output_permutation, int32_t *diag, void *workspace,
                               size_t workspace_bytes, moe_stream_t stream);

/*
 * Output memset (TensorRT-LLM PR #9592, moe_output_memset_inplace): zero
 * out[t, :] for every token t with at least one routed slot
 * (output_permutation[t*k + j] >= 0 for some j); every other row keeps its
 * contents.  Used before an expert stage that accumulates into the output
 * for this rank's experts only.
 *
 *   out [T, H] F32, F16 or BF16, H * sizeof a multiple of 16 bytes,
 *   16-byte aligned; output_permutation [T*k] int32.
 */
moe_status_t moe_output_memset(void *out, moe_dtype_t dtype, int64_t num_tokens, int64_t hidden,
                               int32_t top_k, const int32_t *output_permutation,
                               moe_stream_t stream);

/* Size of the device array that moe_prepare_no_alloc uses as scratch. */
#define MOE_PREPARE_NO_ALLOC_SCRATCH_BYTES ((size_t)4 << 20)

/*
 * moe_prepare without a workspace argument, for callers that cannot
 * allocate device memory: work being recorded into a CUDA graph (cudaMalloc
 * may not run while a stream is captured), serving loops in which a
 * cudaMalloc would synchronise the device and stall every other stream, and
 * processes whose GPU memory is handed to a pool allocator up front.  This
 * call has no counterpart in the paper.
 *
 * Arguments, results and errors are those of moe_prepare.  In place of a
 * workspace the call uses one fixed device array of
 * MOE_PREPARE_NO_ALLOC_SCRATCH_BYTES (4 MiB), which every GPU that loads the
 * library holds until the process exits.  A problem that needs more scratch
 * than that (moe_prepare_workspace_bytes() above 4 MiB: T*k beyond about 3.6
 * million slots with 256 experts, about 0.9 million with 1024) is rejected
 * with MOE_ERR_UNSUPPORTED before anything is launched.  The call allocates
 * nothing: it clears the part of the array it needs with cudaMemsetAsync on
 * `stream`, then launches the same kernels as moe_prepare.
 *
 * All calls on one device share the array and it keeps the last call's
 * contents, so two calls whose work overlaps on the GPU (different streams
 * with no ordering between them) race and produce wrong results: order them
 * on one stream, or use moe_prepare with separate workspaces.  A call that
 * needs the scratch (T*k above 4096) looks up the array's device address on
 * its device whenever its stream is not being captured; a call made during
 * stream capture uses the address found by an earlier call, so make one
 * such call on the device before any stream capture begins.
 */
moe_status_t moe_prepare_no_alloc(const int32_t *topk_ids, int64_t num_tokens, int32_t top_k,
                                  int32_t num_experts, int32_t *expert_counts,
                                  int32_t *expert_offsets, int32_t *blockscale_offsets,
                                  int32_t blockscale_align, int32_t *input_permutation,
                                  int32_t *output_permutation, int32_t *diag,
                                  moe_stream_t stream);

/* Largest num_ranks * num_local_experts of moe_ep_recv_layout. */
#define MOE_EP_MAX_GROUPS 8192

/*
 * Expert-parallel exchange between GPUs, the receiving rank's layout
 * (Mooncake PR #4581: dispatch / combine across ranks, "dispatch and combine
 * kernel implementations"; TensorRT-LLM PR #9592: "Alltoall comm", and one
 * rank's experts being the window local_expert_offset .. +
 * num_local_experts).
 *
 * R = num_ranks ranks each own El = num_local_experts consecutive experts
 * (rank r: experts [r*El, (r+1)*El)).  A source rank runs moe_prepare over
 * all R*El experts and dispatches; its dispatched rows are sorted by
 * expert, so rows [expert_offsets[r*El], expert_offsets[(r+1)*El]) go to
 * rank r as one block ordered by local expert, and its expert_counts,
 * viewed [R][El], are what it tells each rank.  This rank receives:
 *
 *   recv_expert_counts [R, El] int32  rows source s sends for local expert le
 *   (the received buffer holds the source blocks in source order)
 *
 * and this call writes
 *
 *   recv_offsets   [R+1]  int32  first received row of each source block
 *   local_offsets  [El+1] int32  expert offsets of the grouped layout (by
 *                                local expert, then source, then the
 *                                source's own order): what the expert
 *                                stage's grouped GEMM takes
 *   recv_to_local  [N]    int32  grouped row of every received row
 *   local_to_recv  [N]    int32  its inverse
 *   num_recv       [1]    int32  N, the number of received rows
 *
 * The maps are written only when N <= capacity (their allocated length);
 * otherwise only the offsets and num_recv are, so the caller can size them.
 * Received rows move into the grouped layout with moe_dispatch_rows(recv,
 * top_k = 1, input_permutation = local_to_recv) and expert outputs back to
 * the received order with input_permutation = recv_to_local.  All pointers
 * are device memory; nothing is allocated.  Errors: MOE_ERR_INVALID_ARG for
 * num_ranks or num_local_experts < 1, capacity < 0, a NULL offset / count
 * output or a NULL map with capacity > 0; MOE_ERR_UNSUPPORTED when
 * num_ranks * num_local_experts > MOE_EP_MAX_GROUPS.
 */
moe_status_t moe_ep_recv_layout(const int32_t *recv_expert_counts, int32_t num_ranks,
                                int32_t num_local_experts, int64_t capacity,
                                int32_t *recv_offsets, int32_t *local_offsets,
                                int32_t *recv_to_local, int32_t *local_to_recv,
                                int32_t *num_recv, moe_stream_t stream);

/*
 * The exchange between GPUs as stores into the owners' memory (the same
 * exchange as above without all-to-alls: every source rank writes its rows
 * straight into the owners' grouped buffers and later reads the expert
 * outputs straight back from them; Mooncake PR #4581, dispatch / combine
 * kernels that move rows between ranks; TensorRT-LLM PR #9592, one rank's
 * experts being a window).  R ranks each own El = E / R consecutive experts
 * and each holds a grouped buffer of rows laid out by local expert, then
 * source rank, then the source's order (the layout moe_ep_recv_layout
 * gives).  On several GPUs the buffers are other GPUs' memory mapped into
 * this process (CUDA IPC or symmetric memory; peer-to-peer access enabled),
 * reached with plain loads and bulk stores, never with multicast loads.
 *
 * moe_ep_peer_layout: from every rank's expert counts,
 *   all_expert_counts [R, E] int32   rank s's moe_prepare expert_counts in
 *                                    row s (an all-gather of the counts)
 *   topk_ids, expert_offsets, output_permutation   this rank's ([T, k],
 *                                    [E+1], [T*k]) from moe_prepare over all
 *                                    E experts
 * writes
 *   dest_rank [T*k] int32   the rank owning each slot's expert (-1: none)
 *   dest_row  [T*k] int32   the slot's row in that rank's grouped buffer
 *   recv_rows [R]   int32   rows of each rank's grouped buffer
 *   local_offsets [El+1] int32   this rank's grouped expert offsets
 * Errors: MOE_ERR_INVALID_ARG for NULL pointers, num_ranks < 1, rank outside
 * [0, num_ranks), num_experts not a positive multiple of num_ranks;
 * MOE_ERR_UNSUPPORTED for num_experts > MOE_MAX_EXPERTS.
 */
moe_status_t moe_ep_peer_layout(const int32_t *all_expert_counts, int32_t num_ranks,
                                int32_t rank, int32_t num_experts, const int32_t *topk_ids,
                                int64_t num_tokens, int32_t top_k,
                                const int32_t *expert_offsets,
                                const int32_t *output_permutation, int32_t *dest_rank,
                                int32_t *dest_row, int32_t *recv_rows, int32_t *local_offsets,
                                moe_stream_t stream);

/*
 * moe_ep_dispatch_peer: row t of x [T, H] (dtype F32, F16 or BF16, rows a
 * multiple of 16 bytes, 16-byte aligned) goes to row dest_row[t*k+j] of the
 * grouped buffer of rank dest_rank[t*k+j], for every slot j with a
 * destination.  recv_buffers is a DEVICE array of num_ranks pointers to the
 * ranks' grouped buffers (16-byte aligned, recv_rows[r] rows of H elements);
 * slots whose row falls outside recv_rows are skipped.  Each x row is read
 * once (the TMA dispatch of moe_dispatch_rows; its bounded waits report
 * through moe_dispatch_error).  The caller orders the owners' later reads
 * after every source's dispatch (a barrier across ranks).
 */
moe_status_t moe_ep_dispatch_peer(const void *x, moe_dtype_t dtype, int64_t num_tokens,
                                  int64_t hidden, int32_t top_k, const int32_t *dest_rank,
                                  const int32_t *dest_row, void *const *recv_buffers,
                                  const int32_t *recv_rows, int32_t num_ranks,
                                  moe_stream_t stream);

/*
 * moe_ep_combine_peer: out[t] = sum_j weights[t, j] * (row dest_row[t*k+j]
 * of rank dest_rank[t*k+j]'s buffer of expert outputs), accumulated in fp32
 * in slot order exactly as moe_combine does.  out_buffers is a DEVICE array
 * of num_ranks pointers to the ranks' expert-output buffers (the grouped
 * layout, recv_rows[r] rows of H elements of y_dtype, 16-byte aligned).
 * Slots without a valid row contribute nothing.
 */
moe_status_t moe_ep_combine_peer(const void *const *out_buffers, const int32_t *recv_rows,
                                 int32_t num_ranks, moe_dtype_t y_dtype, int64_t num_tokens,
                                 int64_t hidden, int32_t top_k, const int32_t *dest_rank,
                                 const int32_t *dest_row, const float *weights, void *out,
                                 moe_dtype_t out_dtype, moe_stream_t stream);

/* Largest T*k that moe_prepare_dispatch accepts. */
#define MOE_FUSED_MAX_SLOTS 4096

/*
 * Tiny-batch path: moe_prepare followed by moe_dispatch_rows in ONE kernel
 * launch, for T*k <= MOE_FUSED_MAX_SLOTS, where launch latency dominates.
 * Every block recomputes the routing metadata of the whole (small) batch in
 * shared memory, block 0 writes the metadata outputs, and all blocks copy
 * their share of rows.  Arguments and results are exactly those of the two
 * calls (no workspace is needed); `diag` may be NULL.
 */
moe_status_t moe_prepare_dispatch(const int32_t *topk_ids, int64_t num_tokens, int32_t top_k,
                                  int32_t num_experts, int32_t *expert_counts,
                                  int32_t *expert_offsets, int32_t *blockscale_offsets,
                                  int32_t blockscale_align, int32_t *input_permutation,
                                  int32_t *output_permutation, int32_t *diag, const void *x,
                                  moe_dtype_t dtype, int64_t hidden, void *out,
                                  moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
