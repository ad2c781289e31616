/*
 * The C ABI used from plain C: prepare, dispatch and combine through
 * include/moe.h, with device buffers from the CUDA runtime and no Python.
 * Checks what the definitions fix (counts, prefix offsets, inverse and
 * stable permutations, copied rows, one-hot combine) on a batch large
 * enough for the tiled prepare path, and prints "c abi: ok".
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "moe.h"

#define CHECK(cond, ...)                                   \
    do {                                                   \
        if (!(cond)) {                                     \
            fprintf(stderr, "c abi: FAIL " __VA_ARGS__);   \
            fprintf(stderr, "\n");                         \
            return 1;                                      \
        }                                                  \
    } while (0)

#define CUDA(x) CHECK((x) == cudaSuccess, "%s", #x)
#define MOE(x)                                                                       \
    do {                                                                             \
        moe_status_t st_ = (x);                                                      \
        CHECK(st_ == MOE_OK, "%s: %s (%s)", #x, moe_status_string(st_),            \
              moe_last_cuda_error());                                                \
    } while (0)

static uint32_t lcg(uint32_t *s) {
    *s = *s * 1664525u + 1013904223u;
    return *s >> 8;
}

static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

int main(void) {
    const int64_t T = 3000, H = 64;
    const int32_t k = 6, E = 40, A = 16;
    const int64_t S = T * k;
    uint32_t seed = 12345u;

    int32_t *ids = malloc(S * sizeof(int32_t));
    uint16_t *x = malloc(T * H * sizeof(uint16_t));
    float *w = malloc(S * sizeof(float));
    for (int64_t i = 0; i < S; ++i) ids[i] = (int32_t)(lcg(&seed) % (E + 2)) - 1; /* some invalid */
    for (int64_t i = 0; i < T * H; ++i) x[i] = (uint16_t)(0x3c00u + (lcg(&seed) & 0x3ffu)); /* positive normal bf16 */
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) w[t * k + j] = 0.0f;

    int32_t *d_ids, *d_counts, *d_off, *d_bso, *d_in, *d_out, *d_diag;
    float *d_w, *d_comb;
    uint16_t *d_x, *d_disp;
    void *d_ws = NULL;
    CUDA(cudaMalloc((void **)&d_ids, S * sizeof(int32_t)));
    CUDA(cudaMalloc((void **)&d_counts, E * sizeof(int32_t)));
    CUDA(cudaMalloc((void **)&d_off, (E + 1) * sizeof(int32_t)));
    CUDA(cudaMalloc((void **)&d_bso, (E + 1) * sizeof(int32_t)));
    CUDA(cudaMalloc((void **)&d_in, S * sizeof(int32_t)));
    CUDA(cudaMalloc((void **)&d_out, S * sizeof(int32_t)));
    CUDA(cudaMalloc((void **)&d_diag, 2 * sizeof(int32_t)));
    CUDA(cudaMalloc((void **)&d_x, T * H * sizeof(uint16_t)));
    CUDA(cudaMalloc((void **)&d_disp, S * H * sizeof(uint16_t)));
    CUDA(cudaMalloc((void **)&d_w, S * sizeof(float)));
    CUDA(cudaMalloc((void **)&d_comb, T * H * sizeof(float)));
    const size_t ws_bytes = moe_prepare_workspace_bytes(T, k, E);
    CHECK(ws_bytes > 0, "a batch of %lld slots should need the tiled path", (long long)S);
    CUDA(cudaMalloc(&d_ws, ws_bytes));
    CUDA(cudaMemset(d_ws, 0, ws_bytes));
    CUDA(cudaMemcpy(d_ids, ids, S * sizeof(int32_t), cudaMemcpyHostToDevice));
    CUDA(cudaMemcpy(d_x, x, T * H * sizeof(uint16_t), cudaMemcpyHostToDevice));

    MOE(moe_prepare(d_ids, T, k, E, d_counts, d_off, d_bso, A, d_in, d_out, d_diag, d_ws, ws_bytes,
                    NULL));
    MOE(moe_dispatch_rows(d_x, MOE_BF16, T, H, k, d_in, d_out, d_disp, NULL));

    int32_t *counts = malloc(E * sizeof(int32_t)), *off = malloc((E + 1) * sizeof(int32_t));
    int32_t *bso = malloc((E + 1) * sizeof(int32_t)), *in = malloc(S * sizeof(int32_t));
    int32_t *out = malloc(S * sizeof(int32_t)), diag[2];
    uint16_t *disp = malloc(S * H * sizeof(uint16_t));
    CUDA(cudaMemcpy(counts, d_counts, E * sizeof(int32_t), cudaMemcpyDeviceToHost));
    CUDA(cudaMemcpy(off, d_off, (E + 1) * sizeof(int32_t), cudaMemcpyDeviceToHost));
    CUDA(cudaMemcpy(bso, d_bso, (E + 1) * sizeof(int32_t), cudaMemcpyDeviceToHost));
    CUDA(cudaMemcpy(in, d_in, S * sizeof(int32_t), cudaMemcpyDeviceToHost));
    CUDA(cudaMemcpy(out, d_out, S * sizeof(int32_t), cudaMemcpyDeviceToHost));
    CUDA(cudaMemcpy(diag, d_diag, 2 * sizeof(int32_t), cudaMemcpyDeviceToHost));
    CUDA(cudaMemcpy(disp, d_disp, S * H * sizeof(uint16_t), cudaMemcpyDeviceToHost));

    /* counts, offsets and block-scale offsets from their definitions */
    int64_t invalid = 0;
    int32_t *want = calloc(E, sizeof(int32_t));
    for (int64_t i = 0; i < S; ++i) {
        if (ids[i] >= 0 && ids[i] < E) ++want[ids[i]];
        else ++invalid;
    }
    CHECK(diag[0] == invalid && diag[1] == 0, "diag %d %d, invalid %lld", diag[0], diag[1],
          (long long)invalid);
    CHECK(off[0] == 0 && bso[0] == 0, "first offsets");
    for (int32_t e = 0; e < E; ++e) {
        CHECK(counts[e] == want[e], "count of expert %d", e);
        CHECK(off[e + 1] == off[e] + want[e], "offset %d", e + 1);
        CHECK(bso[e + 1] == bso[e] + (want[e] + A - 1) / A * A, "block-scale offset %d", e + 1);
    }
    /* permutations: inverse, grouped by expert, ascending slot inside a group */
    for (int64_t i = 0; i < S; ++i) {
        const int valid = ids[i] >= 0 && ids[i] < E;
        CHECK(valid ? (out[i] >= 0 && in[out[i]] == i) : out[i] == -1, "slot %lld", (long long)i);
    }
    for (int64_t p = 0; p < S; ++p) {
        if (p >= off[E]) {
            CHECK(in[p] == -1, "tail row %lld", (long long)p);
            continue;
        }
        const int32_t e = ids[in[p]];
        CHECK(p >= off[e] && p < off[e + 1], "row %lld outside its expert", (long long)p);
        if (p > off[e]) CHECK(in[p - 1] < in[p], "row %lld not stable", (long long)p);
        CHECK(memcmp(disp + p * H, x + (int64_t)(in[p] / k) * H, H * sizeof(uint16_t)) == 0,
              "dispatched row %lld", (long long)p);
    }

    /* one-hot combine: each token takes its first routed slot with weight 1 */
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j)
            if (out[t * k + j] >= 0) {
                w[t * k + j] = 1.0f;
                break;
            }
    CUDA(cudaMemcpy(d_w, w, S * sizeof(float), cudaMemcpyHostToDevice));
    MOE(moe_combine(d_disp, MOE_BF16, T, H, k, d_out, d_w, d_comb, MOE_F32, NULL));
    float *comb = malloc(T * H * sizeof(float));
    CUDA(cudaMemcpy(comb, d_comb, T * H * sizeof(float), cudaMemcpyDeviceToHost));
    for (int64_t t = 0; t < T; ++t) {
        int routed = 0;
        for (int32_t j = 0; j < k; ++j) routed |= out[t * k + j] >= 0;
        for (int64_t h = 0; h < H; ++h) {
            const float expect = routed ? bf16_to_float(x[t * H + h]) : 0.0f;
            CHECK(comb[t * H + h] == expect, "combine token %lld column %lld", (long long)t,
                  (long long)h);
        }
    }
    /* host-side validation: a NULL output is refused before any launch */
    CHECK(moe_combine(d_disp, MOE_BF16, T, H, k, d_out, d_w, NULL, MOE_F32, NULL) ==
              MOE_ERR_INVALID_ARG,
          "NULL output accepted");
    printf("c abi: ok (%lld slots, %lld invalid, library %d)\n", (long long)S, (long long)invalid,
           moe_version());
    return 0;
}
