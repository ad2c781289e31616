// Test-only kernels: the library's fp32 -> E4M3 conversion helper
// (moe::cvt_e4m3x2, cvt.rn.satfinite.e4m3x2.f32) applied to every fp32 bit
// pattern of a range, for the exhaustive sweep against the oracle's encoder.
// Built by tests/test_gpu_cvt_sweep.py; not part of the library.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_device.cuh"

__global__ void e4m3_of_patterns(uint32_t first, uint32_t n, uint8_t *out) {
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        out[i] = (uint8_t)(moe::cvt_e4m3x2(__uint_as_float(first + i), 0.0f) & 0xffu);
}

// Counts patterns v of [first, first + n) whose code of -v differs from the
// code of v with the sign bit set.
__global__ void e4m3_sign_mismatches(uint32_t first, uint32_t n, unsigned long long *bad) {
    unsigned long long mine = 0;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float v = __uint_as_float(first + i);
        const uint16_t a = moe::cvt_e4m3x2(v, 0.0f) & 0xffu, b = moe::cvt_e4m3x2(-v, 0.0f) & 0xffu;
        mine += b != (a | 0x80u);
    }
    if (mine) atomicAdd(bad, mine);
}

extern "C" int sweep_codes(uint32_t first, uint32_t n, uint8_t *out) {
    e4m3_of_patterns<<<1184, 256>>>(first, n, out);
    return (int)cudaGetLastError();
}

extern "C" int sweep_sign(uint32_t first, uint32_t n, unsigned long long *bad) {
    e4m3_sign_mismatches<<<1184, 256>>>(first, n, bad);
    return (int)cudaGetLastError();
}
