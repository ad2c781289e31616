// Host-side launch helpers: SM count and occupancy caches, and a launcher
// that enables programmatic dependent launch on every kernel.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <map>
#include <mutex>
#include <tuple>

namespace moe {

// Limits of the bounded waits, read at every launch: how long a prepare
// block waits for the other blocks (nanoseconds of the GPU's global timer,
// default one second), and how many mbarrier polls the TMA dispatch makes
// for one staged chunk before it gives up.  Only moe_set_wait_limits
// changes them (tests of the failure reporting).
constexpr uint64_t kDefaultPrepareWaitNs = 1000000000ull;
constexpr uint32_t kDefaultDispatchPolls = 1u << 24;

inline std::atomic<uint64_t> &prepare_wait_ns() {
    static std::atomic<uint64_t> v{kDefaultPrepareWaitNs};
    return v;
}

inline std::atomic<uint32_t> &dispatch_polls() {
    static std::atomic<uint32_t> v{kDefaultDispatchPolls};
    return v;
}

inline int current_device() {
    int d = 0;
    cudaGetDevice(&d);
    return d;
}

inline int sm_count() {
    static std::mutex mu;
    static std::map<int, int> cache;
    const int dev = current_device();
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 1;
    cache[dev] = n;
    return n;
}

// Raises `kernel`'s dynamic shared-memory limit on the current device to at
// least `smem` (needed when dynamic plus static use passes 48 KB).  The limit is per kernel, so
// it is only ever raised: lowering it for a smaller launch would make a later
// larger one invalid.
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, size_t smem) {
    // 48 KB is the default limit for dynamic plus static shared memory; a
    // dynamic request near it needs the attribute once static use is added
    if (smem <= 32 * 1024) return cudaSuccess;
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, size_t> limit;
    const auto key = std::make_pair((const void *)kernel, current_device());
    std::lock_guard<std::mutex> g(mu);
    auto it = limit.find(key);
    if (it != limit.end() && it->second >= smem) return cudaSuccess;
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) limit[key] = smem;
    return e;
}

// Resident blocks per SM of `kernel` at this block size and dynamic shared
// memory, memoised per (kernel, block size, smem, device).
template <typename Kernel>
int blocks_per_sm(Kernel kernel, int threads, size_t smem) {
    static std::mutex mu;
    static std::map<std::tuple<const void *, int, size_t, int>, int> cache;
    const int dev = current_device();
    const auto key = std::make_tuple((const void *)kernel, threads, smem, dev);
    ensure_smem(kernel, smem);
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess ||
        n <= 0) {
        cudaGetLastError();
        n = 1;
    }
    cache[key] = n;
    return n;
}

// Grid for a grid-stride kernel over `units` work items: never more blocks
// than items, never more than fill the GPU once.
template <typename Kernel>
int64_t persistent_grid(Kernel kernel, int threads, size_t smem, int64_t units) {
    const int64_t full = (int64_t)sm_count() * blocks_per_sm(kernel, threads, smem);
    return units < full ? (units > 0 ? units : 1) : full;
}

// How a kernel may start relative to its stream predecessor.  kEarly: with
// programmatic stream serialization (PDL), so that its blocks launch while
// the predecessor finishes and wait for it in griddepcontrol.wait; for the
// short, latency-bound kernels.  kAfter: a plain launch once the predecessor
// has completed; for the streaming kernels (dispatch, combine and the other
// row copies) once they move more than kEarlyStartBytes.  Measured on B200
// over graph-captured steps: with PDL on the streaming kernels the
// 786k-slot workload's step took 1284-1325 us, without it 1245 us, while a
// 32-token step gained 0.5 us from it (7.6 against 8.1 us).
enum class Start { kEarly, kAfter };

constexpr int64_t kEarlyStartBytes = (int64_t)32 << 20;

// The start of a streaming kernel that moves `bytes`.
inline Start streaming_start(int64_t bytes) {
    return bytes < kEarlyStartBytes ? Start::kEarly : Start::kAfter;
}

// Launch with the given start (see Start).
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), int64_t grid, int threads, size_t smem,
                   cudaStream_t stream, Start start, Args &&...args) {
    cudaError_t se = ensure_smem(kernel, smem);
    if (se != cudaSuccess) return se;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3((unsigned)threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = start == Start::kEarly ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace moe
