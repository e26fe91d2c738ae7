// grid_sync.cuh -- the grid-wide wait of the library's one-launch kernels (the K mean, the
// K-smoothing gate, the FP8 quantiser), launched cooperatively so that every CTA is resident.
//
// Each CTA publishes a per-call tag in its own flag word (st.release after its stores); a call
// never clears flags, since each launch carries a tag no earlier launch of the process used. Every
// wait is bounded: past timeout_ns it sets the error word and returns false, and the caller
// leaves the kernel.
#pragma once

#include <cstdint>

#include "host_common.h"

namespace b200 {

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void publish(unsigned long long* flag, unsigned long long tag)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(flag), "l"(tag) : "memory");
}

// A relaxed (strong, unordered) load of a flag word: polls of several flags issue together.
__device__ __forceinline__ unsigned long long peek(const unsigned long long* flag)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(flag));
    return v;
}

// Phase-1 epilogue of every CTA: all its partial stores, then its flag (release).
__device__ __forceinline__ void publish_cta(unsigned long long* flags, unsigned long long tag)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        publish(flags + blockIdx.x, tag);
    }
}

// Polls until every flag flags[c], c < n (<= 1024), carries `tag`, with the first warp: lane l
// watches flags l, l + 32, ... and loads its unseen ones eight at a time each round (relaxed
// loads, so they do not wait for one another), backing off between rounds. False, with the
// error word set, if that takes longer than timeout_ns (counted from t0). Warp 0 only.
__device__ __forceinline__ bool poll_flags(const unsigned long long* flags, unsigned long long tag,
                                           int n, int* status, uint64_t t0,
                                           unsigned long long timeout_ns)
{
    const int lane = threadIdx.x & 31;
    const int mine = lane < n ? (n - lane + 31) / 32 : 0;  // flags lane, lane + 32, ...
    uint32_t pending = mine >= 32 ? 0xFFFFFFFFu : ((1u << mine) - 1u);
    while (pending) {
        for (int j0 = 0; j0 < mine; j0 += 8) {  // eight loads in flight per lane
            unsigned long long v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if ((pending >> (j0 + j)) & 1u) v[j] = peek(flags + lane + 32 * (j0 + j));
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (((pending >> (j0 + j)) & 1u) && v[j] == tag) pending &= ~(1u << (j0 + j));
        }
        if (!pending) break;
        if (global_ns() - t0 > timeout_ns) {
            atomicCAS(status, 0, (int)B200ATTN_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(32);
    }
    return true;
}

// Waits until each of the first n CTAs of the grid has published `tag` in flags[c]; `waiters` is
// the number of CTAs (the first ones, CTA 0 among them) that call this. A few waiters poll the n
// flags themselves. Many waiters would queue behind each other on the flags' few L2 lines, so
// then only CTA 0 reads the n flags; it publishes `tag` in *go, and every other CTA polls that one
// word (two hops instead of one, but one L2 line polled once per round per CTA).
// A relaxed read followed by a fence is an acquire, and CTA 0's release of *go passes on every
// publisher's writes that it observed (release is cumulative); the CTA barrier then orders the
// waiting thread's view before every thread of its CTA. False, with the error word set, if a wait
// takes longer than timeout_ns.
__device__ __forceinline__ bool wait_all_published(const unsigned long long* flags,
                                                   unsigned long long tag, int n, int waiters,
                                                   unsigned long long* go, int* status,
                                                   unsigned long long timeout_ns)
{
    bool ok = true;
    const uint64_t t0 = global_ns();
    if (waiters <= 16 || blockIdx.x == 0) {
        if (threadIdx.x < 32) {
            ok = __all_sync(0xFFFFFFFFu, poll_flags(flags, tag, n, status, t0, timeout_ns));
            __threadfence();
            __syncwarp();  // every lane's acquire is ordered before lane 0's release
            if (waiters > 16 && threadIdx.x == 0 && ok) publish(go, tag);
        }
    } else if (threadIdx.x == 0) {
        while (peek(go) != tag) {
            if (global_ns() - t0 > timeout_ns) {
                atomicCAS(status, 0, (int)B200ATTN_ERR_TIMEOUT);
                ok = false;
                break;
            }
            __nanosleep(32);
        }
        __threadfence();
    }
    return __syncthreads_and(ok) != 0;
}

}  // namespace b200
