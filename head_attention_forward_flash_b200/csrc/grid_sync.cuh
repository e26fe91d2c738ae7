// grid_sync.cuh -- the grid-wide wait of the library's one-launch kernels (the K mean, the
// K-smoothing gate, the FP8 quantiser), launched cooperatively so that every CTA is resident.
//
// Each CTA publishes a per-call tag in its own flag word (st.release after its stores); a call
// never clears flags, since each launch carries a tag (next_call_tag) that no flag word left in
// memory by an earlier launch, of this or of another loaded copy of the library, holds. Every
// wait is bounded: past timeout_ns it sets the error word and returns false, and the caller
// leaves the kernel.
#pragma once

#include <atomic>
#include <chrono>
#include <cstdint>

#include "host_common.h"

namespace b200 {

// A fresh tag for one launch's flag words: `kind` (the kernel family) in the top 16 bits, a
// 48-bit call counter below. The counter starts at a point drawn once per loaded copy of the
// library (the clock and the counter's own address, mixed by the SplitMix64 finaliser), so flag
// words that recycled memory still holds, from earlier calls or from another copy of the library
// loaded into the same process, never carry a tag that a later call uses. 2^48 calls do not wrap
// in practice.
inline unsigned long long next_call_tag(unsigned kind)
{
    static std::atomic<unsigned long long> counter{[] {
        unsigned long long z =
            (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() ^
            (unsigned long long)(uintptr_t)&counter;
        z += 0x9E3779B97F4A7C15ull;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    }()};
    const unsigned long long c = counter.fetch_add(1, std::memory_order_relaxed) + 1;
    return ((unsigned long long)(kind & 0xFFFFu) << 48) | (c & 0xFFFFFFFFFFFFull);
}

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
