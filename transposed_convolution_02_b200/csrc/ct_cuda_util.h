// Host-side CUDA helpers shared by the kernel modules: the driver's tensor-map
// encoder (fetched once through the runtime, so libct.so needs no link against
// libcuda) and per-device attribute caches.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

namespace ct {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
        else
            cudaGetLastError();
    });
    return fn;
}

inline int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return dev;
}

inline int sm_count() {
    static std::atomic<int> cache[64];
    const int dev = current_device();
    if (dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = 148;
        }
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Read a module's device error word (set by a bounded wait that ran out) and
// clear it, in order on `st`, then wait for `st`.  Returns the code read (0:
// none), or -1 when a CUDA call failed.
template <typename T>
inline int take_error_word(T &symbol, cudaStream_t st) {
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&v, symbol, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    if (v != 0 && (cudaMemcpyToSymbolAsync(symbol, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess ||
                   cudaStreamSynchronize(st) != cudaSuccess)) {
        cudaGetLastError();
        return -1;
    }
    return v;
}

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename K>
inline bool allow_smem(K kernel, std::atomic<int> *flags, int bytes) {
    const int dev = current_device();
    if (dev < 0 || dev >= 64) return false;
    if (flags[dev].load()) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    flags[dev].store(1);
    return true;
}

}  // namespace ct
