/*
 * CPU oracle for the MoE dispatch / combine path.
 *
 * TEST INFRASTRUCTURE.  This file is the plain, slow, obviously correct
 * definition that the CUDA library is checked against.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg load it; the library's
 * product path never does.  It shares no code, header or table with the
 * CUDA sources.
 *
 * Sources (the pages' statement of what each step computes):
 *   - sglang PR #19058 "[jit_kernel] Add prepare_moe_input JIT kernels",
 *     section "Changes", item 1 prepare_moe_input:
 *       compute_problem_sizes_kernel  -> tokens per expert   (oracle_prepare)
 *       compute_expert_offsets_kernel -> prefix sum           (oracle_prepare)
 *       compute_expert_blockscale_offsets_kernel (optional)   (oracle_prepare)
 *       compute_arg_sorts_kernel -> input/output permutation  (oracle_prepare)
 *     item 2 shuffle_rows: dtype-agnostic row gather        (oracle_dispatch)
 *     item 3 apply_shuffle_mul_sum: gather + scale + reduce with FP32
 *       accumulation over fp16 / bf16 / fp32                (oracle_combine)
 *   - TensorRT-LLM PR #9592 "Enable CuteDSL MoE with Large EP" (Walkthrough
 *     and review comments): "expanded idx" = t*k + j and "permuted idx" =
 *     dispatched row, int32 index tensors, and the FP8 block-scale MoE path
 *     (run_moe_fp8_block_scales), which oracle_dispatch_fp8 instantiates
 *     with 1x128 blocks and scale = amax / 448; the NVFP4 path
 *     (run_moe_nvfp4, scaling_vector_size = 16: oracle_dispatch_nvfp4); the
 *     moe_sort outputs of a tiled grouped GEMM (oracle_tile_layout); the
 *     local-expert window and moe_output_memset_inplace
 *     (oracle_prepare_local_i64, oracle_output_memset).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes):
 *   - input_permutation[p] is the flat slot (expanded) index i = t*k + j of
 *     the p-th dispatched row; output_permutation is its inverse.
 *   - Within an expert the order is ascending slot index i, i.e. ascending
 *     token then ascending slot (a stable sort by expert id).
 *   - expert_offsets has E+1 entries, the last one the number of valid
 *     slots.
 *   - Block-scale offsets round each expert's row count up to a multiple of
 *     A (A = 1 gives the expert offsets).
 *   - Ids outside [0, E) are excluded from every output: they are not
 *     counted, their output_permutation entry is -1, the trailing
 *     input_permutation entries (p >= offsets[E]) are -1, dispatch leaves
 *     those rows untouched and combine skips those slots.
 *   - FP8: per dispatched row and per 128-column block, amax = max |x|,
 *     s = amax / 448 (fp32, round to nearest), q = e4m3(x / s) with x / s an
 *     fp32 division, round to nearest even, saturating to +-448; a block
 *     with amax = 0 gets s = 0 and all-zero bytes.  The scale of dispatched
 *     row p of expert e goes to row bso[e] + (p - offsets[e]).
 *   - Combine: acc = 0; for j = 0..k-1: acc = acc + w[t,j] * y[row_j, h],
 *     each product and each sum rounded separately to fp32 (this file must
 *     be compiled with -ffp-contract=off), then acc rounded to the output
 *     dtype (round to nearest even; fp32 output is acc itself).
 */

#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/*
 * Timing build only: the benchmark's CPU baseline also compiles this file
 * with -fopenmp, which shares the independent row loops of the dispatches
 * and of combine among the host cores (ROWS_IN_PARALLEL).  Every iteration
 * of those loops writes its own rows, so the results are the same bits.
 * The build the tests check against has no _OPENMP and stays one thread.
 */
#ifdef _OPENMP
#define ROWS_IN_PARALLEL _Pragma("omp parallel for schedule(static)")
#else
#define ROWS_IN_PARALLEL
#endif

/* Threads the row loops use (1 in the plain build). */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2 };

/* ------------------------------------------------------------------ */
/* Scalar formats, written from their bit-level definitions.           */
/* ------------------------------------------------------------------ */

/* bfloat16 is the upper half of an IEEE binary32. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
float oracle_f16_to_f32(uint16_t h)
{
    int sign = h >> 15;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + frac), expo - 25);  /* (1 + frac/1024) * 2^(expo-15) */
    return (float)(sign ? -v : v);
}

/* Round a non-negative double holding an exact value to the nearest
 * integer, ties to even. */
static double round_half_even(double q)
{
    double fl = floor(q);
    double diff = q - fl;
    if (diff > 0.5 || (diff == 0.5 && fmod(fl, 2.0) != 0.0))
        fl += 1.0;
    return fl;
}

/* binary32 -> bfloat16, round to nearest even on the 16 dropped bits. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u)          /* NaN stays NaN (quiet) */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xffffu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;                               /* a carry may reach inf: correct */
    return (uint16_t)upper;
}

/* binary32 -> binary16, round to nearest even, overflow to infinity. */
uint16_t oracle_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)(sign | 0x7e00u);
    double a = fabs((double)f);                    /* exact */
    if (a >= 65520.0)                              /* halfway above 65504 and beyond */
        return (uint16_t)(sign | 0x7c00u);
    if (a < ldexp(1.0, -14)) {                     /* subnormal range: step 2^-24 */
        double q = round_half_even(a / ldexp(1.0, -24));
        return (uint16_t)(sign | (uint16_t)q);     /* q = 1024 encodes 2^-14 */
    }
    int ex;
    frexp(a, &ex);                                 /* a in [2^(ex-1), 2^ex) */
    int e = ex - 1;
    double q = round_half_even(a / ldexp(1.0, e - 10)); /* in [1024, 2048] */
    return (uint16_t)(sign | (uint16_t)((e + 15) * 1024 + (int)q - 1024));
}

/*
 * binary32 -> OCP FP8 E4M3 (the "FN" variant: no infinities, 0x7f / 0xff
 * are NaN, largest finite 448 = 0x7e).  1 sign bit, 4 exponent bits
 * (bias 7), 3 fraction bits; subnormals are frac * 2^-9.  Round to nearest
 * even; finite magnitudes that round above 448 (and infinities) saturate to
 * 448; NaN maps to NaN.
 */
uint8_t oracle_f32_to_e4m3(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint8_t sign = (uint8_t)((u >> 24) & 0x80u);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint8_t)(sign | 0x7fu);
    double a = fabs((double)f);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7eu);
    if (a < ldexp(1.0, -6)) {                      /* subnormal range: step 2^-9 */
        double q = round_half_even(a / ldexp(1.0, -9));
        return (uint8_t)(sign | (uint8_t)q);       /* q = 8 encodes 2^-6 */
    }
    int ex;
    frexp(a, &ex);
    int e = ex - 1;                                /* a in [2^e, 2^(e+1)), e in [-6, 8] */
    double q = round_half_even(a / ldexp(1.0, e - 3)); /* in [8, 16] */
    int code = (e + 7) * 8 + (int)q - 8;
    if (code > 0x7e)
        code = 0x7e;
    return (uint8_t)(sign | (uint8_t)code);
}

float oracle_e4m3_to_f32(uint8_t b)
{
    int sign = b >> 7;
    int expo = (b >> 3) & 0xf;
    int frac = b & 7;
    double v;
    if (expo == 0xf && frac == 7)
        v = NAN;
    else if (expo == 0)
        v = ldexp((double)frac, -9);
    else
        v = ldexp((double)(8 + frac), expo - 10);  /* (1 + frac/8) * 2^(expo-7) */
    return (float)(sign ? -v : v);
}

static float load_as_f32(const void *base, int dtype, int64_t idx)
{
    if (dtype == ORACLE_F32)
        return ((const float *)base)[idx];
    if (dtype == ORACLE_F16)
        return oracle_f16_to_f32(((const uint16_t *)base)[idx]);
    return oracle_bf16_to_f32(((const uint16_t *)base)[idx]);
}

static void store_from_f32(void *base, int dtype, int64_t idx, float v)
{
    if (dtype == ORACLE_F32)
        ((float *)base)[idx] = v;
    else if (dtype == ORACLE_F16)
        ((uint16_t *)base)[idx] = oracle_f32_to_f16(v);
    else
        ((uint16_t *)base)[idx] = oracle_f32_to_bf16(v);
}

/* ------------------------------------------------------------------ */
/* Step A: routing metadata (prepare_moe_input).                       */
/* ------------------------------------------------------------------ */

/*
 * ids [T*k] (row-major [T,k]) -> counts [E], offsets [E+1],
 * bso [E+1] (may be NULL), input_perm [T*k], output_perm [T*k].
 * Returns the number of slots whose id lies outside [0, E).
 *
 * The permutation is built by scanning the slots once per expert, in
 * ascending expert order and ascending slot order: the p-th slot found is
 * dispatched row p.  This is O(E * T * k) on purpose: it is the stable
 * order written out, with nothing shared with a counting sort.
 */
int64_t oracle_prepare(const int32_t *ids, int64_t T, int32_t k, int32_t E, int32_t A,
                       int32_t *counts, int32_t *offsets, int32_t *bso,
                       int32_t *input_perm, int32_t *output_perm)
{
    int64_t S = T * (int64_t)k;
    for (int64_t i = 0; i < S; ++i) {
        output_perm[i] = -1;
        input_perm[i] = -1;
    }
    int64_t p = 0;
    for (int32_t e = 0; e < E; ++e) {
        int32_t c = 0;
        for (int64_t i = 0; i < S; ++i) {
            if (ids[i] == e) {
                input_perm[p] = (int32_t)i;
                output_perm[i] = (int32_t)p;
                ++p;
                ++c;
            }
        }
        counts[e] = c;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    if (bso) {
        bso[0] = 0;
        for (int32_t e = 0; e < E; ++e) {
            int32_t padded = (counts[e] + A - 1) / A * A;
            bso[e + 1] = bso[e] + padded;
        }
    }
    return S - p;
}

/* ------------------------------------------------------------------ */
/* Step B1: dispatch, same dtype (shuffle_rows).                       */
/* ------------------------------------------------------------------ */

/* out[p, :] = x[input_perm[p] / k, :] for every p with input_perm[p] >= 0. */
void oracle_dispatch(const void *x, int64_t row_bytes, int32_t k,
                     const int32_t *input_perm, int64_t S, void *out)
{
    const unsigned char *src = (const unsigned char *)x;
    unsigned char *dst = (unsigned char *)out;
    ROWS_IN_PARALLEL
    for (int64_t p = 0; p < S; ++p) {
        int32_t i = input_perm[p];
        if (i < 0)
            continue;
        int64_t t = i / k;
        memcpy(dst + p * row_bytes, src + t * row_bytes, (size_t)row_bytes);
    }
}

/* ------------------------------------------------------------------ */
/* Step B2: dispatch with FP8 E4M3 1x128 block-scale quantisation.     */
/* ------------------------------------------------------------------ */

/*
 * x [T,H] bf16 or f16; for each dispatched row p (token t = input_perm[p]/k,
 * expert e = ids[input_perm[p]]) and each 128-column block b:
 *   amax = max |x[t, b*128 .. b*128+127]|
 *   s    = amax / 448            (s = 0 and zero bytes when amax = 0)
 *   q[p, c] = e4m3(x[t, c] / s)
 *   scales[(bso[e] + p - offsets[e]) * (H/128) + b] = s
 * Rows and scale rows that no valid slot maps to are left untouched.
 */
void oracle_dispatch_fp8(const uint16_t *x, int x_dtype, int64_t T, int64_t H, int32_t k,
                         const int32_t *ids, const int32_t *input_perm,
                         const int32_t *offsets, const int32_t *bso, int64_t S,
                         uint8_t *q, float *scales)
{
    (void)T;
    int64_t nb = H / 128;
    ROWS_IN_PARALLEL
    for (int64_t p = 0; p < S; ++p) {
        int32_t i = input_perm[p];
        if (i < 0)
            continue;
        int64_t t = i / k;
        int32_t e = ids[i];
        int64_t srow = (int64_t)bso[e] + (p - offsets[e]);
        for (int64_t b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int64_t c = b * 128; c < b * 128 + 128; ++c) {
                float a = fabsf(load_as_f32(x, x_dtype, t * H + c));
                if (a > amax)
                    amax = a;
            }
            float s = 0.0f;
            if (amax == 0.0f) {
                for (int64_t c = b * 128; c < b * 128 + 128; ++c)
                    q[p * H + c] = 0;
            } else {
                s = amax / 448.0f;
                for (int64_t c = b * 128; c < b * 128 + 128; ++c) {
                    float v = load_as_f32(x, x_dtype, t * H + c) / s;
                    q[p * H + c] = oracle_f32_to_e4m3(v);
                }
            }
            scales[srow * nb + b] = s;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Step C1: combine (apply_shuffle_mul_sum).                           */
/* ------------------------------------------------------------------ */

/*
 * out[t, h] = round_out( sum_{j=0..k-1} w[t,j] * y[output_perm[t*k+j], h] ),
 * summed in fp32 in ascending j with every operation rounded separately;
 * slots with output_perm = -1 contribute nothing.
 */
void oracle_combine(const void *y, int y_dtype, int64_t T, int64_t H, int32_t k,
                    const int32_t *output_perm, const float *w, void *out, int out_dtype)
{
    ROWS_IN_PARALLEL
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < k; ++j) {
                int32_t p = output_perm[t * k + j];
                if (p < 0)
                    continue;
                float prod = w[t * k + j] * load_as_f32(y, y_dtype, (int64_t)p * H + h);
                acc = acc + prod;
            }
            store_from_f32(out, out_dtype, t * H + h, acc);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Array forms of the scalar conversions (for exhaustive sweeps).      */
/* ------------------------------------------------------------------ */

void oracle_f32_to_e4m3_n(const float *in, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_e4m3(in[i]);
}

void oracle_f32_to_bf16_n(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_bf16(in[i]);
}

void oracle_f32_to_f16_n(const float *in, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_f16(in[i]);
}

void oracle_f16_to_f32_n(const uint16_t *in, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f16_to_f32(in[i]);
}

void oracle_bf16_to_f32_n(const uint16_t *in, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_bf16_to_f32(in[i]);
}

void oracle_e4m3_to_f32_n(const uint8_t *in, int64_t n, float *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_to_f32(in[i]);
}

/* ------------------------------------------------------------------ */
/* Grouped-GEMM metadata (the step after prepare).                     */
/* ------------------------------------------------------------------ */

/*
 * Problem sizes of the two grouped GEMMs that follow dispatch (sglang PR
 * #19058, item 1: compute_problem_sizes_kernel fills problem_sizes1 /
 * problem_sizes2): for every expert e, ps1[e] = {counts[e], n1, k1} and
 * ps2[e] = {counts[e], n2, k2} as (M, N, K).
 */
void oracle_problem_sizes(const int32_t *counts, int32_t E, int32_t n1, int32_t k1, int32_t n2,
                          int32_t k2, int32_t *ps1, int32_t *ps2)
{
    for (int32_t e = 0; e < E; ++e) {
        ps1[3 * e + 0] = counts[e];
        ps1[3 * e + 1] = n1;
        ps1[3 * e + 2] = k1;
        ps2[3 * e + 0] = counts[e];
        ps2[3 * e + 1] = n2;
        ps2[3 * e + 2] = k2;
    }
}

/*
 * Tile-padded layout for a tiled grouped GEMM (the moe_sort outputs of
 * TensorRT-LLM PR #9592: tile_idx_to_group_idx, tile_idx_to_mn_limit,
 * expanded_idx_to_permuted_idx, permuted_idx_to_expanded_idx,
 * total_num_padded_tokens, num_non_exiting_tiles).  Every expert's rows are
 * padded up to a multiple of the tile size:
 *   padded_offsets[e]  = sum over e' < e of roundup(counts[e'], tile)
 *   tile t (of the first padded_offsets[E] / tile) belongs to the expert e
 *     whose padded range holds row t*tile; its row limit is
 *     padded_offsets[e] + counts[e]; tiles past the last are -1 / -1;
 *   a valid slot i of expert e with dispatched row p lands on padded row
 *     padded_offsets[e] + (p - offsets[e]);
 *   permuted_idx_to_expanded_idx is the inverse, -1 on padding rows and on
 *     every row past the padded total (up to max_tiles * tile).
 * Returns 0, or -1 when max_tiles * tile is too small for the padded total
 * (then nothing is written).
 */
int oracle_tile_layout(const int32_t *ids, int64_t T, int32_t k, int32_t E, int32_t tile,
                       const int32_t *counts, const int32_t *offsets, const int32_t *output_perm,
                       int32_t max_tiles, int32_t *padded_offsets, int32_t *tile_group,
                       int32_t *tile_mn_limit, int32_t *exp2perm, int32_t *perm2exp,
                       int32_t *num_tiles, int32_t *total_padded)
{
    int64_t S = T * (int64_t)k;
    int64_t acc = 0;
    for (int32_t e = 0; e < E; ++e)
        acc += (counts[e] + tile - 1) / tile * (int64_t)tile;
    if (acc > (int64_t)max_tiles * tile)
        return -1;
    padded_offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e)
        padded_offsets[e + 1] = padded_offsets[e] + (counts[e] + tile - 1) / tile * tile;
    *total_padded = padded_offsets[E];
    *num_tiles = padded_offsets[E] / tile;
    for (int32_t t = 0; t < max_tiles; ++t) {
        tile_group[t] = -1;
        tile_mn_limit[t] = -1;
    }
    int32_t t = 0;
    for (int32_t e = 0; e < E; ++e) {
        for (int32_t r = padded_offsets[e]; r < padded_offsets[e + 1]; r += tile) {
            tile_group[t] = e;
            tile_mn_limit[t] = padded_offsets[e] + counts[e];
            ++t;
        }
    }
    for (int64_t q = 0; q < (int64_t)max_tiles * tile; ++q)
        perm2exp[q] = -1;
    for (int64_t i = 0; i < S; ++i) {
        int32_t e = ids[i];
        if (e < 0 || e >= E) {
            exp2perm[i] = -1;
            continue;
        }
        int32_t pp = padded_offsets[e] + (output_perm[i] - offsets[e]);
        exp2perm[i] = pp;
        perm2exp[pp] = (int32_t)i;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* One rank's window of experts, int64 ids, output memset.             */
/* ------------------------------------------------------------------ */

/*
 * Routing metadata for the experts [base, base + E) of one rank, from int64
 * ids (Mooncake's top-k index type): slot i belongs to local expert
 * ids[i] - base when that lies in [0, E); every other slot is excluded
 * exactly as an invalid id is.  Written out directly, without calling
 * oracle_prepare: the same per-expert scan over the slots.
 */
int64_t oracle_prepare_local_i64(const int64_t *ids, int64_t T, int32_t k, int64_t base, int32_t E,
                                 int32_t A, int32_t *counts, int32_t *offsets, int32_t *bso,
                                 int32_t *input_perm, int32_t *output_perm)
{
    int64_t S = T * (int64_t)k;
    for (int64_t i = 0; i < S; ++i) {
        output_perm[i] = -1;
        input_perm[i] = -1;
    }
    int64_t p = 0;
    for (int32_t e = 0; e < E; ++e) {
        int32_t c = 0;
        for (int64_t i = 0; i < S; ++i) {
            if (ids[i] - base == (int64_t)e) {
                input_perm[p] = (int32_t)i;
                output_perm[i] = (int32_t)p;
                ++p;
                ++c;
            }
        }
        counts[e] = c;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    if (bso) {
        bso[0] = 0;
        for (int32_t e = 0; e < E; ++e)
            bso[e + 1] = bso[e] + (counts[e] + A - 1) / A * A;
    }
    return S - p;
}

/*
 * Output memset (TensorRT-LLM PR #9592, moe_output_memset_inplace): zero the
 * output row of every token that has at least one slot with a dispatched
 * row (output_perm >= 0); every other row is left unchanged.
 */
void oracle_output_memset(void *out, int64_t row_bytes, int64_t T, int32_t k,
                          const int32_t *output_perm)
{
    unsigned char *o = (unsigned char *)out;
    for (int64_t t = 0; t < T; ++t) {
        int routed = 0;
        for (int32_t j = 0; j < k; ++j)
            if (output_perm[t * k + j] >= 0)
                routed = 1;
        if (routed)
            memset(o + t * row_bytes, 0, (size_t)row_bytes);
    }
}

/* ------------------------------------------------------------------ */
/* NVFP4 dispatch: E2M1 elements with one E4M3 scale per 16 elements.  */
/* ------------------------------------------------------------------ */

/*
 * binary32 -> FP4 E2M1 (1 sign bit, 2 exponent bits with bias 1, 1 fraction
 * bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinities or NaN), round to
 * nearest even, saturating to +-6.  Returns the 4-bit code (sign in bit 3).
 * NaN maps to +0 (the format has no NaN; inputs here are finite).
 */
uint8_t oracle_f32_to_e2m1(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint8_t sign = (uint8_t)((u >> 28) & 0x8u);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return 0;
    double a = fabs((double)f);
    if (a >= 6.0)
        return (uint8_t)(sign | 0x7u);
    if (a < 1.0) {                                   /* subnormal range: step 0.5 */
        double q = round_half_even(a / 0.5);        /* 0, 1 or 2 (2 encodes 1.0) */
        return (uint8_t)(sign | (uint8_t)q);
    }
    int ex;
    frexp(a, &ex);
    int e = ex - 1;                                  /* a in [2^e, 2^(e+1)), e in 0..2 */
    double q = round_half_even(a / ldexp(1.0, e - 1)); /* in [2, 4] */
    int code = (e + 1) * 2 + (int)q - 2;
    if (code > 7)
        code = 7;
    return (uint8_t)(sign | (uint8_t)code);
}

float oracle_e2m1_to_f32(uint8_t c)
{
    int sign = (c >> 3) & 1;
    int expo = (c >> 1) & 3;
    int frac = c & 1;
    double v = expo == 0 ? 0.5 * frac : ldexp(1.0 + 0.5 * frac, expo - 1);
    return (float)(sign ? -v : v);
}

void oracle_f32_to_e2m1_n(const float *in, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f32_to_e2m1(in[i]);
}

/*
 * NVFP4 dispatch (the B200 NVFP4 MoE path of TensorRT-LLM PR #9592, block
 * size scaling_vector_size = 16).  For each dispatched row p (token t =
 * input_perm[p] / k, expert e = ids[input_perm[p]]) and each 16-column
 * block b:
 *   amax  = max |x[t, 16b .. 16b+15]|
 *   sf    = e4m3(amax / 6)            (fp32 division, then E4M3 RNE, satfinite)
 *   d     = the fp32 value of sf
 *   q[p, c] = e2m1(x[t, c] / d)       (fp32 division, E2M1 RNE, saturating)
 *             or 0 when d = 0
 * Two codes per byte: element 2m in the low nibble, 2m+1 in the high one.
 * The scale byte goes to scales[(bso[e] + p - offsets[e]) * (H/16) + b].
 */
void oracle_dispatch_nvfp4(const uint16_t *x, int x_dtype, int64_t T, int64_t H, int32_t k,
                           const int32_t *ids, const int32_t *input_perm, const int32_t *offsets,
                           const int32_t *bso, int64_t S, uint8_t *q, uint8_t *scales)
{
    (void)T;
    int64_t nb = H / 16;
    for (int64_t p = 0; p < S; ++p) {
        int32_t i = input_perm[p];
        if (i < 0)
            continue;
        int64_t t = i / k;
        int32_t e = ids[i];
        int64_t srow = (int64_t)bso[e] + (p - offsets[e]);
        for (int64_t b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int64_t c = b * 16; c < b * 16 + 16; ++c) {
                float a = fabsf(load_as_f32(x, x_dtype, t * H + c));
                if (a > amax)
                    amax = a;
            }
            uint8_t sf = oracle_f32_to_e4m3(amax / 6.0f);
            float d = oracle_e4m3_to_f32(sf);
            for (int64_t c = b * 16; c < b * 16 + 16; c += 2) {
                uint8_t lo = 0, hi = 0;
                if (d != 0.0f) {
                    lo = oracle_f32_to_e2m1(load_as_f32(x, x_dtype, t * H + c) / d);
                    hi = oracle_f32_to_e2m1(load_as_f32(x, x_dtype, t * H + c + 1) / d);
                }
                q[p * (H / 2) + c / 2] = (uint8_t)(lo | (hi << 4));
            }
            scales[srow * nb + b] = sf;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Expert-parallel exchange: the receiving rank's layout.              */
/* ------------------------------------------------------------------ */

/*
 * Mooncake PR #4581 (expert-parallel dispatch / combine between GPUs) and
 * TensorRT-LLM PR #9592 (all-to-all communication; one rank's experts are
 * the window local_expert_offset .. + num_local_experts).  R ranks each own
 * El consecutive experts.  A source rank's dispatched rows are sorted by
 * expert, so the rows it sends to this rank form one block ordered by local
 * expert.  c[s*El + le] is the number of rows source s sends for local
 * expert le.
 *
 *   received buffer: the source blocks in source order,
 *     recv_offsets[s] = sum over s' < s and all le of c[s'][le]   ([R+1])
 *   grouped layout: by local expert, then source, then the source's order,
 *     local_offsets[le] = sum over le' < le and all s of c[s][le'] ([El+1])
 *   received row q = recv_offsets[s] + sum_{le' < le} c[s][le'] + m
 *     and grouped row g = local_offsets[le] + sum_{s' < s} c[s'][le] + m
 *     are the same row (0 <= m < c[s][le]):
 *     recv_to_local[q] = g, local_to_recv[g] = q.
 * Returns the number of received rows.
 */
int64_t oracle_ep_recv_layout(const int32_t *c, int32_t R, int32_t El, int32_t *recv_offsets,
                              int32_t *local_offsets, int32_t *recv_to_local,
                              int32_t *local_to_recv)
{
    int64_t acc = 0;
    for (int32_t s = 0; s < R; ++s) {
        recv_offsets[s] = (int32_t)acc;
        for (int32_t le = 0; le < El; ++le)
            acc += c[(int64_t)s * El + le];
    }
    recv_offsets[R] = (int32_t)acc;
    int64_t n = acc;
    acc = 0;
    for (int32_t le = 0; le < El; ++le) {
        local_offsets[le] = (int32_t)acc;
        for (int32_t s = 0; s < R; ++s)
            acc += c[(int64_t)s * El + le];
    }
    local_offsets[El] = (int32_t)acc;
    /* walk the grouped layout in its own order and find each row's place in
       the received buffer */
    int64_t g = 0;
    for (int32_t le = 0; le < El; ++le) {
        for (int32_t s = 0; s < R; ++s) {
            int64_t q = recv_offsets[s];
            for (int32_t l2 = 0; l2 < le; ++l2)
                q += c[(int64_t)s * El + l2];
            for (int32_t m = 0; m < c[(int64_t)s * El + le]; ++m) {
                recv_to_local[q + m] = (int32_t)g;
                local_to_recv[g] = (int32_t)(q + m);
                ++g;
            }
        }
    }
    return n;
}
