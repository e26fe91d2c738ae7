// kmean.cu -- the K channel-mean pre-pass (k_smooth_mean, k_smooth_mean_noalloc), the K-smoothing
// gate (k_smooth_gate) and the mean subtraction (k_smooth_sub).
//
// K is [b, sk, hk, d] bf16; for a fixed (batch, key position) the hk*d channels of all kv heads
// are one contiguous row, so the mean over the key axis is a column sum of a [sk, hk*d] matrix
// per batch: fully coalesced 16-byte loads, one 8-channel group per thread, no shuffles needed.
//
// The mean and the gate each run as ONE launch of co-resident CTAs (a cooperative launch):
//   phase 1  every CTA sums chunks of key rows into fp32 partials and publishes them with a
//            per-call tag in its own flag word;
//   phase 2  CTAs that own part of the fold wait (with a time limit) until every CTA's flag
//            carries this call's tag, then fold the partials in a fixed order.
// The fold order never depends on timing, so results are bit-identical from run to run: the
// "two deterministic kernels behind one host call" of "[HIP] Mha v4: run the K-smoothing gate as
// one HIP call" (Summary, commit message) become two phases of one kernel.
#include <atomic>
#include <cmath>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "host_common.h"

namespace b200 {
namespace {

constexpr int kThreads = 512;  // one-pass kernels: each thread owns 8 consecutive channels
constexpr int kColsPerCta = kThreads * 8;
constexpr int kFoldWarps = kThreads / 32;
constexpr int kSubThreads = 256;
constexpr int kErrTimeout = 10;                       // B200ATTN_ERR_TIMEOUT
constexpr uint64_t kTagMagic = 0x6B6D65616EULL << 24;  // high bits of every flag tag

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4& x)
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        acc[2 * t] += __uint_as_float(w[t] << 16);
        acc[2 * t + 1] += __uint_as_float(w[t] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void acc_sq_bf16x8(float (&sum)[8], float (&sq)[8], const uint4& x)
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
        sum[2 * q] += lo;
        sum[2 * q + 1] += hi;
        sq[2 * q] = fmaf(lo, lo, sq[2 * q]);  // K^2 of a bf16 value is exact in fp32
        sq[2 * q + 1] = fmaf(hi, hi, sq[2 * q + 1]);
    }
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

__device__ __forceinline__ unsigned long long observe(const unsigned long long* flag)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(flag) : "memory");
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

// Waits until each CTA of the grid has published `tag` (the first warp polls, each lane a share
// of the flags, backing off between polls so that waiting CTAs load L2 as little as possible);
// false, with the error word set, if that takes longer than timeout_ns.
__device__ __forceinline__ bool wait_all_published(const unsigned long long* flags,
                                                   unsigned long long tag, int* status,
                                                   unsigned long long timeout_ns)
{
    bool ok = true;
    if (threadIdx.x < 32) {
        const uint64_t t0 = global_ns();
        for (int c = threadIdx.x; c < (int)gridDim.x && ok; c += 32) {
            while (observe(flags + c) != tag) {
                if (global_ns() - t0 > timeout_ns) {
                    atomicCAS(status, 0, kErrTimeout);
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
    }
    return __syncthreads_and(ok) != 0;
}

// sum over c in [c_lo, c_hi) of src[c * pitch], added in order of c; the loads are issued eight
// at a time (L2 hits, after the flags), so the chain is not one load latency per term.
__device__ __forceinline__ float ordered_sum(const float* src, int64_t pitch, int c_lo, int c_hi)
{
    float sum = 0.f;
    int c = c_lo;
    for (; c + 8 <= c_hi; c += 8) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = __ldcg(src + (int64_t)(c + e) * pitch);
#pragma unroll
        for (int e = 0; e < 8; ++e) sum += v[e];
    }
    for (; c < c_hi; ++c) sum += __ldcg(src + (int64_t)c * pitch);
    return sum;
}

struct OnePass {
    const uint4* k;
    float* partial;             // [b][nchunks][planes][cols]
    unsigned long long* flags;  // [gridDim.x]
    float* mean;                // [b][cols]
    int* gate;                  // gate only: [b][hk]
    float* ratio;               // gate only, may be null
    int64_t b, sk, cols, c8, colgroups;
    int64_t stride;             // rows summed: 0, stride, 2*stride, ... (1: every row)
    int64_t n_rows;             // rows summed per (bi, column): sk, or the sample size
    int64_t rows_per_chunk;
    int nchunks;
    int64_t n_items;            // b * colgroups * nchunks
    int64_t hk, d;              // gate: kv heads and channels per head
    float n_rows_f;             // n_rows as fp32, the divisor
    float threshold;
    unsigned long long tag;
    int* status;
    unsigned long long timeout_ns;
};

// Phase 1 of both kernels: item = (bi, column group, chunk) of rows; each thread sums its 8
// channels over the chunk's rows (sixteen independent 16-byte loads in flight, added in row
// order) into plane 0, and with SQ their squares into plane 1.
template <bool SQ>
__device__ __forceinline__ void sum_chunks(const OnePass& a)
{
    constexpr int PL = SQ ? 2 : 1;
    for (int64_t it = blockIdx.x; it < a.n_items; it += gridDim.x) {
        const int chunk = (int)(it % a.nchunks);
        const int64_t bcg = it / a.nchunks;
        const int64_t cg = bcg % a.colgroups, bi = bcg / a.colgroups;
        const int64_t g8 = cg * kThreads + threadIdx.x;
        if (g8 >= a.c8) continue;
        const int64_t t0 = (int64_t)chunk * a.rows_per_chunk;
        int64_t t1 = t0 + a.rows_per_chunk;
        t1 = t1 < a.n_rows ? t1 : a.n_rows;
        float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float q[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const uint4* src = a.k + (bi * a.sk) * a.c8 + g8;
        const int64_t step = a.stride * a.c8;
        int64_t t = t0;
        for (; t + 16 <= t1; t += 16) {
            uint4 x[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = __ldg(src + (t + e) * step);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                if (SQ) acc_sq_bf16x8(s, q, x[e]);
                else acc_bf16x8(s, x[e]);
            }
        }
        for (; t < t1; ++t) {
            const uint4 x = __ldg(src + t * step);
            if (SQ) acc_sq_bf16x8(s, q, x);
            else acc_bf16x8(s, x);
        }
        float* dst = a.partial + ((bi * a.nchunks + chunk) * PL) * a.cols + g8 * 8;
        reinterpret_cast<float4*>(dst)[0] = make_float4(s[0], s[1], s[2], s[3]);
        reinterpret_cast<float4*>(dst)[1] = make_float4(s[4], s[5], s[6], s[7]);
        if (SQ) {
            reinterpret_cast<float4*>(dst + a.cols)[0] = make_float4(q[0], q[1], q[2], q[3]);
            reinterpret_cast<float4*>(dst + a.cols)[1] = make_float4(q[4], q[5], q[6], q[7]);
        }
    }
}

// mean[bi][col] = (sum of partial[bi][chunk][col] over the chunks) / sk. Fold items are blocks of
// 32 columns of one batch; warp w of the CTA sums the chunks of its fixed contiguous range
// [w*nchunks/16, (w+1)*nchunks/16) in order, then the 16 warp sums are added in warp order.
__global__ void __launch_bounds__(kThreads) k_mean_onepass(const OnePass a)
{
    __shared__ float red[kFoldWarps][32];
    sum_chunks<false>(a);
    publish_cta(a.flags, a.tag);
    const int64_t nblk = (a.cols + 31) / 32;
    const int64_t n_fold = a.b * nblk;
    if ((int64_t)blockIdx.x >= n_fold) return;
    if (!wait_all_published(a.flags, a.tag, a.status, a.timeout_ns)) return;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int c_lo = (int)((int64_t)w * a.nchunks / kFoldWarps);
    const int c_hi = (int)((int64_t)(w + 1) * a.nchunks / kFoldWarps);
    for (int64_t f = blockIdx.x; f < n_fold; f += gridDim.x) {
        const int64_t bi = f / nblk;
        const int64_t col = (f - bi * nblk) * 32 + lane;
        float sum = 0.f;
        if (col < a.cols)
            sum = ordered_sum(a.partial + (bi * a.nchunks) * a.cols + col, a.cols, c_lo, c_hi);
        red[w][lane] = sum;
        __syncthreads();
        if (w == 0 && col < a.cols) {
            float tsum = 0.f;
#pragma unroll
            for (int q = 0; q < kFoldWarps; ++q) tsum += red[q][lane];
            a.mean[bi * a.cols + col] = __fdiv_rn(tsum, a.n_rows_f);
        }
        __syncthreads();
    }
}

// The gate (see k_smooth_gate). Phase 1 sums K and K^2 over the strided sample; phase 2 item =
// (bi, kv head): the 512 threads form 512/d groups of d (one thread per channel); group grp sums
// the chunks of its fixed contiguous range, the group sums are added in group order, giving mu_c
// and e_c; then sum mu_c^2 and sum e_c over the d channels by a fixed tree; ratio = first /
// second (0 for an all-zero K); gate = ratio >= threshold; mean = mu where the gate is on, else 0.
__global__ void __launch_bounds__(kThreads) k_gate_onepass(const OnePass a)
{
    __shared__ float gs[kThreads], gq[kThreads];
    __shared__ float num[256], den[256];
    sum_chunks<true>(a);
    publish_cta(a.flags, a.tag);
    const int64_t n_fold = a.b * a.hk;
    if ((int64_t)blockIdx.x >= n_fold) return;
    if (!wait_all_published(a.flags, a.tag, a.status, a.timeout_ns)) return;
    const int d = (int)a.d;
    const int groups = kThreads / d;
    const int c = threadIdx.x % d, grp = threadIdx.x / d;
    const int c_lo = (int)((int64_t)grp * a.nchunks / groups);
    const int c_hi = (int)((int64_t)(grp + 1) * a.nchunks / groups);
    for (int64_t f = blockIdx.x; f < n_fold; f += gridDim.x) {
        const int64_t bi = f / a.hk, g = f - bi * a.hk;
        const int64_t col = g * d + c;
        const float* src = a.partial + (bi * a.nchunks * 2) * a.cols + col;
        const float sum = ordered_sum(src, 2 * a.cols, c_lo, c_hi);
        const float sq = ordered_sum(src + a.cols, 2 * a.cols, c_lo, c_hi);
        gs[threadIdx.x] = sum;
        gq[threadIdx.x] = sq;
        __syncthreads();
        if (grp == 0) {
            float s = 0.f, e = 0.f;
            for (int q = 0; q < groups; ++q) {
                s += gs[q * d + c];
                e += gq[q * d + c];
            }
            const float mu = __fdiv_rn(s, a.n_rows_f);
            num[c] = mu * mu;
            den[c] = __fdiv_rn(e, a.n_rows_f);
            // only the d threads of group 0 take part: a barrier over exactly those warps (d is
            // a multiple of 32), id 1
            asm volatile("bar.sync 1, %0;" ::"r"(d) : "memory");
            for (int wdt = d / 2; wdt > 0; wdt >>= 1) {
                if (c < wdt) {
                    num[c] += num[c + wdt];
                    den[c] += den[c + wdt];
                }
                asm volatile("bar.sync 1, %0;" ::"r"(d) : "memory");
            }
            const float r = den[0] > 0.f ? __fdiv_rn(num[0], den[0]) : 0.f;
            const bool on = r >= a.threshold;
            a.mean[f * d + c] = on ? mu : 0.f;
            if (c == 0) {
                a.gate[f] = on ? 1 : 0;
                if (a.ratio) a.ratio[f] = r;
            }
        }
        __syncthreads();
    }
}

// k_out = bf16_rne(float(K) - mean[bi, col]), 8 channels (16 bytes) per group; each thread has
// four groups in flight per step.
__device__ __forceinline__ void sub_group(const float* __restrict__ mean, uint4* __restrict__ k_out,
                                          int64_t t, const uint4& x, int64_t c8, int64_t sk,
                                          int64_t cols)
{
    const int64_t r = t / c8;  // bi * sk + s
    const int64_t g8 = t - r * c8;
    const int64_t bi = r / sk;
    const float4* m = reinterpret_cast<const float4*>(mean + bi * cols + g8 * 8);
    const float4 m0 = __ldg(m), m1 = __ldg(m + 1);
    const float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float lo = __fsub_rn(__uint_as_float(w[q] << 16), mv[2 * q]);
        const float hi = __fsub_rn(__uint_as_float(w[q] & 0xFFFF0000u), mv[2 * q + 1]);
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        o[q] = *reinterpret_cast<uint32_t*>(&v);
    }
    k_out[t] = make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void __launch_bounds__(kSubThreads)
    k_sub_kernel(const uint4* __restrict__ k, const float* __restrict__ mean,
                 uint4* __restrict__ k_out, int64_t rows, int64_t sk, int64_t cols)
{
    const int64_t c8 = cols / 8;
    const int64_t n = rows * c8;
    const int64_t stride = (int64_t)gridDim.x * kSubThreads;
    int64_t t = (int64_t)blockIdx.x * kSubThreads + threadIdx.x;
    for (; t + 3 * stride < n; t += 4 * stride) {
        uint4 x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = __ldg(k + t + e * stride);
#pragma unroll
        for (int e = 0; e < 4; ++e) sub_group(mean, k_out, t + e * stride, x[e], c8, sk, cols);
    }
    for (; t < n; t += stride) sub_group(mean, k_out, t, __ldg(k + t), c8, sk, cols);
}

// Fixed scratch for k_smooth_mean_noalloc: file-scope device memory that every GPU loading this
// library holds until the process exits: 2^20 floats of partial sums (4 MiB), then 1024 64-bit
// flag words (8 KiB), one per CTA of the one-pass kernel.
constexpr int64_t kNoAllocScratchFloats = (int64_t)1 << 20;
constexpr int kMaxGrid = 1024;
__device__ __align__(256) float g_kmean_scratch[kNoAllocScratchFloats + 2 * kMaxGrid];

int check_kmean_args(const void* k, const void* mean, int64_t b, int64_t hk, int64_t sk,
                     int64_t d, int64_t* cols_out)
{
    if (b < 0 || hk < 0 || sk <= 0) return B200ATTN_ERR_SHAPE;
    if (!(d == 64 || d == 128 || d == 256)) return B200ATTN_ERR_HEADDIM;
    int64_t cols, n;
    if (!numel({hk, d}, &cols) || !numel({b, sk, cols, 2}, &n) || !numel({b, cols, 4}, &n) ||
        b >= 65536 || sk >= ((int64_t)1 << 40))
        return B200ATTN_ERR_RANGE;
    *cols_out = cols;
    if (b == 0 || hk == 0) return B200ATTN_OK;
    if (!k || !mean) return B200ATTN_ERR_NULL;
    if (!aligned(k, 16) || !aligned(mean, 16)) return B200ATTN_ERR_ALIGN;
    return B200ATTN_OK;
}

// Grid of a one-pass kernel on the current device: its co-resident CTAs (occupancy x SMs),
// at most one per SM and at most kMaxGrid; cached per device (atomics: concurrent first calls
// store the same value).
template <class K>
int onepass_grid(K kernel, std::atomic<int> (&cache)[64])
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 0;
    }
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        n = per_sm >= 1 ? sms : 0;  // one CTA per SM: eight 16-byte loads in flight per thread
        n = n < kMaxGrid ? n : kMaxGrid;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

std::atomic<int> g_mean_grid[64];
std::atomic<int> g_gate_grid[64];
std::atomic<unsigned> g_calls{0};

// A tag no earlier call of this process used, with high bits no partial sum's bits resemble.
unsigned long long next_tag()
{
    const unsigned c = g_calls.fetch_add(1, std::memory_order_relaxed) + 1;
    return kTagMagic | (unsigned long long)c;
}

// Work split of the one-pass kernels: the rows of every (bi, column group of 4096 channels) cut
// into chunks, so that the grid's CTAs get about one item each; at least 16 rows per chunk, at
// most max_chunks chunks (the scratch), at most 1024.
struct Split {
    int64_t colgroups, rows_per_chunk, n_items;
    int nchunks, grid;
};

Split make_split(int64_t b, int64_t cols, int64_t n_rows, int64_t max_chunks, int grid_max)
{
    Split s;
    s.colgroups = (cols + kColsPerCta - 1) / kColsPerCta;
    int64_t nch = (grid_max + b * s.colgroups - 1) / (b * s.colgroups);
    const int64_t by_rows = (n_rows + 15) / 16;
    if (nch > by_rows) nch = by_rows;
    if (nch > max_chunks) nch = max_chunks;
    if (nch > 1024) nch = 1024;
    if (nch < 1) nch = 1;
    s.rows_per_chunk = (n_rows + nch - 1) / nch;
    s.nchunks = (int)((n_rows + s.rows_per_chunk - 1) / s.rows_per_chunk);
    s.n_items = b * s.colgroups * s.nchunks;
    s.grid = (int)(s.n_items < grid_max ? s.n_items : grid_max);
    return s;
}

int launch_onepass(void (*kernel)(const OnePass), OnePass& a, int grid, cudaStream_t st)
{
    void* args[] = {&a};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3((unsigned)grid),
                                    dim3(kThreads), args, 0, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return B200ATTN_OK;
}

// The mean through the one-pass kernel with split sp, partials (room for sp.nchunks chunks) and
// flags (kMaxGrid words) at the given device addresses.
int run_mean(const void* k, float* mean, int64_t b, int64_t sk, int64_t cols, const Split& sp,
             float* partial, unsigned long long* flags, int* status, cudaStream_t st)
{
    OnePass a{};
    a.k = static_cast<const uint4*>(k);
    a.partial = partial;
    a.flags = flags;
    a.mean = mean;
    a.b = b;
    a.sk = sk;
    a.cols = cols;
    a.c8 = cols / 8;
    a.colgroups = sp.colgroups;
    a.stride = 1;
    a.n_rows = sk;
    a.rows_per_chunk = sp.rows_per_chunk;
    a.nchunks = sp.nchunks;
    a.n_items = sp.n_items;
    a.n_rows_f = (float)sk;
    a.tag = next_tag();
    a.status = status;
    a.timeout_ns = 4000000000ull;
    return launch_onepass(k_mean_onepass, a, sp.grid, st);
}

}  // namespace
}  // namespace b200

using namespace b200;

extern "C" int k_smooth_mean(const void* k, float* mean, int64_t b, int64_t hk, int64_t sk,
                             int64_t d, void* stream)
{
    int64_t cols = 0;
    int rc = check_kmean_args(k, mean, b, hk, sk, d, &cols);
    if (rc != B200ATTN_OK || b == 0 || hk == 0) return rc;
    rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    int* status = status_word();
    const int grid_max = onepass_grid(k_mean_onepass, g_mean_grid);
    if (!status || grid_max <= 0) return B200ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // scratch: the partials of the split's chunks, then the grid's flags
    const Split sp = make_split(b, cols, sk, 1024, grid_max);
    const size_t part_bytes = (size_t)(b * sp.nchunks * cols) * sizeof(float);
    const size_t nbytes = part_bytes + kMaxGrid * sizeof(unsigned long long);
    char* scratch = nullptr;
    cudaMemPool_t pool = scratch_pool();
    if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void**>(&scratch), nbytes, pool, st) !=
                     cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    rc = run_mean(k, mean, b, sk, cols, sp, reinterpret_cast<float*>(scratch),
                  reinterpret_cast<unsigned long long*>(scratch + part_bytes), status, st);
    if (cudaFreeAsync(scratch, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return rc;
}

// Device address of g_kmean_scratch on the current device, looked up once per device (the
// host-side name of a __device__ array is not a device address).
static float* noalloc_scratch()
{
    // atomic: concurrent first calls from several host threads store the same address
    static std::atomic<float*> addr[64] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return nullptr;
    }
    float* a = addr[dev].load(std::memory_order_relaxed);
    if (a == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kmean_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        a = static_cast<float*>(p);
        addr[dev].store(a, std::memory_order_relaxed);
    }
    return a;
}

extern "C" int k_smooth_mean_noalloc(const void* k, float* mean, int64_t b, int64_t hk, int64_t sk,
                                     int64_t d, void* stream)
{
    int64_t cols = 0;
    int rc = check_kmean_args(k, mean, b, hk, sk, d, &cols);
    if (rc != B200ATTN_OK || b == 0 || hk == 0) return rc;
    if (b * cols > kNoAllocScratchFloats) return B200ATTN_ERR_SCRATCH;
    rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    float* scratch = noalloc_scratch();
    int* status = status_word();
    const int grid_max = onepass_grid(k_mean_onepass, g_mean_grid);
    if (!scratch || !status || grid_max <= 0) return B200ATTN_ERR_CUDA;
    // The partials of as many chunks as fit in the fixed scratch; the flags after them. Every
    // partial the fold reads is written earlier in the same launch, and a flag counts only when
    // it carries this call's tag, so nothing needs clearing between calls.
    const Split sp = make_split(b, cols, sk, kNoAllocScratchFloats / (b * cols), grid_max);
    return run_mean(k, mean, b, sk, cols, sp, scratch,
                    reinterpret_cast<unsigned long long*>(scratch + kNoAllocScratchFloats),
                    status, static_cast<cudaStream_t>(stream));
}

extern "C" int k_smooth_gate(const void* k, float* mean, int32_t* gate, float* ratio, int64_t b,
                             int64_t hk, int64_t sk, int64_t d, float threshold, void* stream)
{
    int64_t cols = 0;
    int rc = check_kmean_args(k, mean, b, hk, sk, d, &cols);
    if (rc != B200ATTN_OK || b == 0 || hk == 0) return rc;
    if (!gate) return B200ATTN_ERR_NULL;
    if (!aligned(gate, 4) || (ratio && !aligned(ratio, 4))) return B200ATTN_ERR_ALIGN;
    if (!std::isfinite(threshold)) return B200ATTN_ERR_SCALE;
    int64_t n_bg;
    if (!numel({b, hk}, &n_bg) || n_bg >= ((int64_t)1 << 31)) return B200ATTN_ERR_RANGE;
    rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    int* status = status_word();
    const int grid_max = onepass_grid(k_gate_onepass, g_gate_grid);
    if (!status || grid_max <= 0) return B200ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const int64_t stride = (sk + 2047) / 2048;  // every key up to 2048, else a strided sample
    const int64_t n_samp = (sk + stride - 1) / stride;
    const Split sp = make_split(b, cols, n_samp, 1024, grid_max);
    const size_t part_bytes = (size_t)(b * sp.nchunks * 2 * cols) * sizeof(float);
    const size_t nbytes = part_bytes + kMaxGrid * sizeof(unsigned long long);
    char* scratch = nullptr;
    cudaMemPool_t pool = scratch_pool();
    if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void**>(&scratch), nbytes, pool, st) !=
                     cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    OnePass a{};
    a.k = static_cast<const uint4*>(k);
    a.partial = reinterpret_cast<float*>(scratch);
    a.flags = reinterpret_cast<unsigned long long*>(scratch + part_bytes);
    a.mean = mean;
    a.gate = gate;
    a.ratio = ratio;
    a.b = b;
    a.sk = sk;
    a.cols = cols;
    a.c8 = cols / 8;
    a.colgroups = sp.colgroups;
    a.stride = stride;
    a.n_rows = n_samp;
    a.rows_per_chunk = sp.rows_per_chunk;
    a.nchunks = sp.nchunks;
    a.n_items = sp.n_items;
    a.hk = hk;
    a.d = d;
    a.n_rows_f = (float)n_samp;
    a.threshold = threshold;
    a.tag = next_tag();
    a.status = status;
    a.timeout_ns = 4000000000ull;
    rc = launch_onepass(k_gate_onepass, a, sp.grid, st);
    if (cudaFreeAsync(scratch, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return rc;
}

extern "C" int k_smooth_sub(const void* k, const float* mean, void* k_out, int64_t b, int64_t hk,
                            int64_t sk, int64_t d, void* stream)
{
    int64_t cols = 0;
    int rc = check_kmean_args(k, mean, b, hk, sk, d, &cols);
    if (rc != B200ATTN_OK || b == 0 || hk == 0) return rc;
    if (!k_out) return B200ATTN_ERR_NULL;
    if (!aligned(k_out, 16)) return B200ATTN_ERR_ALIGN;
    rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    const int64_t n = b * sk * (cols / 8);
    int64_t blocks = (n + 4 * kSubThreads - 1) / (4 * kSubThreads);
    if (blocks > 148 * 8) blocks = 148 * 8;
    k_sub_kernel<<<(unsigned)blocks, kSubThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k), mean, static_cast<uint4*>(k_out), b * sk, sk, cols);
    return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}
