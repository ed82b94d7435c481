// devcache.h -- per-device launch facts cached without locks: the SM count of
// each device and the resident blocks per SM of each kernel (at its fixed
// dynamic shared-memory size).  Two host threads making their first call at
// the same time may both compute a value; both store the same number through
// an atomic, so the caches hold no data race.
#pragma once
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>

namespace lx {

constexpr int MAX_DEVICES = 64;

// The current device and its SM count.
inline cudaError_t current_device_sms(int* dev, int* sms) {
    static std::atomic<int> cache[MAX_DEVICES];  // static storage: starts at 0
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    if (*dev < 0 || *dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
    int v = cache[*dev].load(std::memory_order_relaxed);
    if (v == 0) {
        e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, *dev);
        if (e != cudaSuccess) return e;
        cache[*dev].store(v, std::memory_order_relaxed);
    }
    *sms = v;
    return cudaSuccess;
}

// Resident blocks per SM of KERN on device `dev` with `threads` threads and
// `smem` bytes of dynamic shared memory (the same on every call for one KERN);
// the first call on a device also raises the kernel's dynamic shared-memory
// limit to `smem`.
template <auto KERN>
cudaError_t blocks_per_sm(int dev, int threads, size_t smem, int* per) {
    static std::atomic<int> cache[MAX_DEVICES];
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        cudaError_t e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, KERN, threads, smem);
        if (e != cudaSuccess) return e;
        v = std::max(1, v);
        cache[dev].store(v, std::memory_order_relaxed);
    }
    *per = v;
    return cudaSuccess;
}

}  // namespace lx
