// host_common.h -- host-side argument checks shared by the C-ABI entry points.
// Every check here runs before any CUDA call, so an invalid call launches nothing.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <atomic>
#include <mutex>

#include "../../include/b200attn.h"

namespace b200 {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// a * b without signed overflow; false when the product does not fit in int64.
inline bool mul_ok(int64_t a, int64_t b, int64_t* out)
{
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

// Element count of a product of dims; false on overflow.
inline bool numel(std::initializer_list<int64_t> dims, int64_t* out)
{
    int64_t n = 1;
    for (int64_t d : dims)
        if (!mul_ok(n, d, &n)) return false;
    *out = n;
    return true;
}

// sm_100 check for the current device (cached per device). Returns a status code.
inline int check_arch()
{
    // 0 unknown, 1 ok, 2 wrong arch; atomic, so concurrent first calls do not race
    static std::atomic<int> cached[64] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    if (dev < 64) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c != 0) return c == 1 ? B200ATTN_OK : B200ATTN_ERR_ARCH;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    const bool ok = (major == 10 && minor == 0);
    if (dev < 64) cached[dev].store(ok ? 1 : 2, std::memory_order_relaxed);
    return ok ? B200ATTN_OK : B200ATTN_ERR_ARCH;
}

// Device address of the library's error word on the current device, where kernels whose
// bounded waits give up record B200ATTN_ERR_TIMEOUT (read and cleared by attn_debug_status);
// null if CUDA fails. Defined in attn_api.cu.
int* status_word();

// Stream-ordered pool for the pre-passes' partial results (k_smooth_mean, k_smooth_gate,
// fp8_quantize), one per device. Its release threshold is
// "never", so memory freed at the end of a call stays in the pool for the next call instead of
// being returned to the driver (and mapped again) around every synchronisation.
inline cudaMemPool_t scratch_pool()
{
    static cudaMemPool_t pools[64] = {nullptr};
    static std::mutex mu;  // first calls from several host threads create one pool per device
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (pools[dev] == nullptr) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        uint64_t keep = UINT64_MAX;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        pools[dev] = pool;
    }
    return pools[dev];
}

}  // namespace b200
