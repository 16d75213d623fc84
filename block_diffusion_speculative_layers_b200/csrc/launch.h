// launch.h -- kernel launch with programmatic dependent launch and optional
// thread-block clusters (cudaLaunchKernelEx).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <utility>

#include "kernels.h"

namespace dfl {

// Set a kernel attribute once per (kernel, device, attribute): function
// attributes are per device, so a process that drives several devices sets them
// on each.  The kernels of a process are few, so a fixed open-addressing table of
// the (kernel, device, attribute) keys already set answers on every launch
// without a lock; the first setting of a key takes the lock.  A key is recorded
// when the setting succeeds, or always when `keep_failed` (a preference whose
// refusal changes nothing).  Thread-safe.
inline cudaError_t func_attr_once(const void *kern, cudaFuncAttribute attr, int value, bool keep_failed) {
    constexpr int N = 1024;
    static std::atomic<uint64_t> table[N];
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // host code addresses fit in 48 bits; device ordinal and attribute in 8 each
    const uint64_t key = ((uint64_t)(uintptr_t)kern << 16) | ((uint64_t)(dev & 0xff) << 8) | ((uint64_t)attr & 0xff);
    const uint32_t h0 = (uint32_t)((key * 0x9E3779B97F4A7C15ull) >> 54);  // 10 bits
    auto find = [&](int &slot) {
        for (int i = 0; i < N; ++i) {
            const int j = (int)((h0 + i) & (N - 1));
            const uint64_t v = table[j].load(std::memory_order_acquire);
            if (v == key) return true;
            if (v == 0) {
                slot = j;
                return false;
            }
        }
        slot = -1;  // full: set the attribute again on every launch (still correct)
        return false;
    };
    int slot = -1;
    if (find(slot)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu);
    if (find(slot)) return cudaSuccess;
    const cudaError_t pending = cudaPeekAtLastError();
    e = cudaFuncSetAttribute(kern, attr, value);
    if (e != cudaSuccess && keep_failed && pending == cudaSuccess) cudaGetLastError();  // drop only our own error
    if ((e == cudaSuccess || keep_failed) && slot >= 0) table[slot].store(key, std::memory_order_release);
    return keep_failed ? cudaSuccess : e;
}

// Raise a kernel's dynamic shared-memory limit to the B200 maximum (227 KB).
inline cudaError_t ensure_smem_attr(const void *kern) {
    return func_attr_once(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024, false);
}

// Process-wide switch for programmatic dependent launch (on by default).
bool &pdl_enabled();

template <typename... Exp, typename... Act>
inline cudaError_t launch_k(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster_z,
                            Act &&...args) {
    note_launch();
    // Every kernel of the library prefers the largest shared-memory carveout.  An
    // SM changes its L1 / shared split only when idle, so a small kernel left to
    // the default (a smaller carveout) between two projections that need the
    // largest one makes SMs drain and reconfigure at both boundaries instead of
    // starting the next kernel's CTAs early (measured on B200: FP8 decode step
    // 3.91 -> 3.88 ms, the MX quantiser being such a kernel; bf16 unchanged).
    func_attr_once((const void *)kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                   (int)cudaSharedmemCarveoutMaxShared, true);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster_z > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = 1;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = cluster_z;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

}  // namespace dfl
