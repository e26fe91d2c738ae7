// kmean.cu -- the K channel-mean pre-pass: k_smooth_mean and k_smooth_sub.
//
// K is [b, sk, hk, d] bf16; for a fixed (batch, key position) the hk*d channels of all kv heads
// are one contiguous row, so the mean over the key axis is a column sum of a [sk, hk*d] matrix
// per batch: fully coalesced 16-byte loads, one 8-channel group per thread, no shuffles needed.
// Kernel 1 sums a chunk of key rows per CTA into fp32 partials; kernel 2 folds the partials of
// each channel in a fixed order, so the result is bit-identical from run to run (the two
// deterministic kernels behind one host call of "[HIP] Mha v4: run the K-smoothing gate as one
// HIP call", Summary and commit message).
#include <atomic>
#include <cmath>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "host_common.h"

namespace b200 {
namespace {

constexpr int kThreads = 256;      // threads per CTA; each owns 8 consecutive channels
constexpr int kColsPerCta = kThreads * 8;
constexpr int kTargetCtas = 4 * 148;  // about four waves of CTAs on the 148 SMs
constexpr int kMinRowsPerChunk = 16;

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4& x)
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        acc[2 * t] += __uint_as_float(w[t] << 16);
        acc[2 * t + 1] += __uint_as_float(w[t] & 0xFFFF0000u);
    }
}

// partial[bi][chunk][col] = sum over the chunk's key rows of K[bi, s, col]  (col = g*d + c)
__global__ void __launch_bounds__(kThreads)
    k_mean_partial(const uint4* __restrict__ k, float* __restrict__ partial, int64_t sk,
                   int64_t cols, int64_t rows_per_chunk, int nchunks)
{
    const int64_t bi = blockIdx.z;
    const int chunk = blockIdx.y;
    const int64_t g8 = (int64_t)blockIdx.x * kThreads + threadIdx.x;  // 8-channel group
    const int64_t c8 = cols / 8;
    if (g8 >= c8) return;
    const int64_t s0 = (int64_t)chunk * rows_per_chunk;
    int64_t s1 = s0 + rows_per_chunk;
    s1 = s1 < sk ? s1 : sk;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint4* src = k + (bi * sk) * c8 + g8;
    int64_t s = s0;
    for (; s + 4 <= s1; s += 4) {  // four independent 16-byte loads in flight per thread
        const uint4 x0 = __ldg(src + (s + 0) * c8);
        const uint4 x1 = __ldg(src + (s + 1) * c8);
        const uint4 x2 = __ldg(src + (s + 2) * c8);
        const uint4 x3 = __ldg(src + (s + 3) * c8);
        acc_bf16x8(acc, x0);
        acc_bf16x8(acc, x1);
        acc_bf16x8(acc, x2);
        acc_bf16x8(acc, x3);
    }
    for (; s < s1; ++s) acc_bf16x8(acc, __ldg(src + s * c8));
    float4* dst = reinterpret_cast<float4*>(partial + ((bi * nchunks + chunk) * cols) + g8 * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// mean[bi][col] = (sum of partial[bi][chunk][col] over the chunks) / sk, 32 columns per CTA:
// warp w sums chunks w, w+8, w+16, ... in order, then the eight warp sums are added in warp order,
// so the result does not depend on timing.
__global__ void __launch_bounds__(kThreads)
    k_mean_fold(const float* __restrict__ partial, float* __restrict__ mean, int64_t cols,
                int nchunks, float sk_f)
{
    __shared__ float red[kThreads / 32][32];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int64_t col = (int64_t)blockIdx.x * 32 + lane;
    const int64_t bi = blockIdx.y;
    float sum = 0.f;
    if (col < cols) {
        const float* src = partial + bi * nchunks * cols + col;
        for (int c = w; c < nchunks; c += kThreads / 32) sum += src[(int64_t)c * cols];
    }
    red[w][lane] = sum;
    __syncthreads();
    if (w == 0 && col < cols) {
        float t = 0.f;
#pragma unroll
        for (int q = 0; q < kThreads / 32; ++q) t += red[q][lane];
        mean[bi * cols + col] = __fdiv_rn(t, sk_f);
    }
}

// Gate moments over the sampled keys s = t * stride (t < n_samp):
// partial[bi][chunk][0][col] = sum of K, partial[bi][chunk][1][col] = sum of K^2 over the chunk's
// sampled rows (K^2 of a bf16 value is exact in fp32).
__global__ void __launch_bounds__(kThreads)
    k_gate_partial(const uint4* __restrict__ k, float* __restrict__ partial, int64_t sk,
                   int64_t cols, int64_t stride, int64_t n_samp, int64_t per_chunk, int nchunks)
{
    const int64_t bi = blockIdx.z;
    const int chunk = blockIdx.y;
    const int64_t g8 = (int64_t)blockIdx.x * kThreads + threadIdx.x;  // 8-channel group
    const int64_t c8 = cols / 8;
    if (g8 >= c8) return;
    const int64_t t0 = (int64_t)chunk * per_chunk;
    int64_t t1 = t0 + per_chunk;
    t1 = t1 < n_samp ? t1 : n_samp;
    float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float sq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint4* src = k + (bi * sk) * c8 + g8;
    const int64_t step = stride * c8;
    auto add = [&](const uint4& x) {
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
            sum[2 * q] += lo;
            sum[2 * q + 1] += hi;
            sq[2 * q] = fmaf(lo, lo, sq[2 * q]);
            sq[2 * q + 1] = fmaf(hi, hi, sq[2 * q + 1]);
        }
    };
    int64_t t = t0;
    for (; t + 4 <= t1; t += 4) {  // four independent 16-byte loads in flight, added in row order
        const uint4 x0 = __ldg(src + (t + 0) * step);
        const uint4 x1 = __ldg(src + (t + 1) * step);
        const uint4 x2 = __ldg(src + (t + 2) * step);
        const uint4 x3 = __ldg(src + (t + 3) * step);
        add(x0);
        add(x1);
        add(x2);
        add(x3);
    }
    for (; t < t1; ++t) add(__ldg(src + t * step));
    float* dst = partial + ((bi * nchunks + chunk) * 2) * cols + g8 * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        dst[e] = sum[e];
        dst[cols + e] = sq[e];
    }
}

// Per (bi, g), 1024 threads: chunk group grp = threadIdx.x / d of channel c = threadIdx.x % d
// sums the partials of chunks grp, grp + G, grp + 2G, ... (G = 1024 / d groups); the G group
// sums are added in group order, giving mu_c and e_c (mean and mean square over the sample);
// then sum mu_c^2 and sum e_c over the d channels by a fixed tree in shared memory; ratio =
// first / second (0 for an all-zero K); gate = ratio >= threshold; mean = mu where the gate is
// on, else 0. Every order is fixed, so the result does not depend on timing.
constexpr int kFoldThreads = 1024;
__global__ void __launch_bounds__(kFoldThreads)
    k_gate_fold(const float* __restrict__ partial, float* __restrict__ mean,
                int* __restrict__ gate, float* __restrict__ ratio, int64_t hk, int64_t d,
                int nchunks, float n_f, float threshold)
{
    __shared__ float gs[kFoldThreads], gq[kFoldThreads];
    __shared__ float num[256], den[256];
    const int64_t bg = blockIdx.x;  // bi * hk + g
    const int64_t bi = bg / hk, g = bg - bi * hk;
    const int groups = kFoldThreads / (int)d;
    const int c = threadIdx.x % (int)d;
    const int grp = threadIdx.x / (int)d;
    const int64_t cols = hk * d;
    const int64_t col = g * d + c;
    float gsum = 0.f, gsq = 0.f;
#pragma unroll 4
    for (int ch = grp; ch < nchunks; ch += groups) {
        const float* src = partial + ((bi * nchunks + ch) * 2) * cols;
        gsum += src[col];
        gsq += src[cols + col];
    }
    gs[threadIdx.x] = gsum;
    gq[threadIdx.x] = gsq;
    __syncthreads();
    if (grp != 0) return;
    float sum = 0.f, sq = 0.f;
    for (int q = 0; q < groups; ++q) {
        sum += gs[q * (int)d + c];
        sq += gq[q * (int)d + c];
    }
    const float mu = __fdiv_rn(sum, n_f);
    num[c] = mu * mu;
    den[c] = __fdiv_rn(sq, n_f);
    // only the d threads of group 0 remain: a barrier over exactly those warps (d is a multiple
    // of 32), id 1
    asm volatile("bar.sync 1, %0;" ::"r"((int)d) : "memory");
    for (int w = (int)d / 2; w > 0; w >>= 1) {
        if (c < w) {
            num[c] += num[c + w];
            den[c] += den[c + w];
        }
        asm volatile("bar.sync 1, %0;" ::"r"((int)d) : "memory");
    }
    const float r = den[0] > 0.f ? __fdiv_rn(num[0], den[0]) : 0.f;
    const bool on = r >= threshold;
    mean[bg * d + c] = on ? mu : 0.f;
    if (c == 0) {
        gate[bg] = on ? 1 : 0;
        if (ratio) ratio[bg] = r;
    }
}

// k_out = bf16_rne(float(K) - mean[bi, col]), 8 channels (16 bytes) per thread per step.
__global__ void __launch_bounds__(kThreads)
    k_sub_kernel(const uint4* __restrict__ k, const float* __restrict__ mean,
                 uint4* __restrict__ k_out, int64_t rows, int64_t sk, int64_t cols)
{
    const int64_t c8 = cols / 8;
    const int64_t n = rows * c8;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t t = (int64_t)blockIdx.x * kThreads + threadIdx.x; t < n; t += stride) {
        const int64_t r = t / c8;            // (bi * sk + s)
        const int64_t g8 = t - r * c8;
        const int64_t bi = r / sk;
        const float4* m = reinterpret_cast<const float4*>(mean + bi * cols + g8 * 8);
        const float4 m0 = __ldg(m), m1 = __ldg(m + 1);
        const float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
        const uint4 x = __ldg(k + t);
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
}

// Fixed partial-sum scratch for k_smooth_mean_noalloc: file-scope device memory that every GPU
// loading this library holds until the process exits. 1 Mi floats (4 MiB).
constexpr int64_t kNoAllocScratchFloats = (int64_t)1 << 20;
__device__ __align__(256) float g_kmean_scratch[kNoAllocScratchFloats];

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
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const int64_t col_ctas = (cols + kColsPerCta - 1) / kColsPerCta;
    int64_t nchunks = (kTargetCtas + col_ctas * b - 1) / (col_ctas * b);
    const int64_t max_chunks = (sk + kMinRowsPerChunk - 1) / kMinRowsPerChunk;
    if (nchunks > max_chunks) nchunks = max_chunks;
    if (nchunks > 1024) nchunks = 1024;
    if (nchunks < 1) nchunks = 1;
    const int64_t rows_per_chunk = (sk + nchunks - 1) / nchunks;
    nchunks = (sk + rows_per_chunk - 1) / rows_per_chunk;

    float* partial = nullptr;
    cudaMemPool_t pool = scratch_pool();
    if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void**>(&partial),
                                         (size_t)(b * nchunks * cols) * sizeof(float), pool,
                                         st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    dim3 g1((unsigned)col_ctas, (unsigned)nchunks, (unsigned)b);
    k_mean_partial<<<g1, kThreads, 0, st>>>(static_cast<const uint4*>(k), partial, sk, cols,
                                            rows_per_chunk, (int)nchunks);
    k_mean_fold<<<dim3((unsigned)((cols + 31) / 32), (unsigned)b), kThreads, 0, st>>>(
        partial, mean, cols, (int)nchunks, (float)sk);
    const bool launched = cudaGetLastError() == cudaSuccess;
    if (cudaFreeAsync(partial, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return launched ? B200ATTN_OK : B200ATTN_ERR_CUDA;
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
    float* partial = noalloc_scratch();
    if (!partial) return B200ATTN_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // Same split as k_smooth_mean, capped so that the partials fit in the fixed scratch.
    const int64_t col_ctas = (cols + kColsPerCta - 1) / kColsPerCta;
    int64_t nchunks = (kTargetCtas + col_ctas * b - 1) / (col_ctas * b);
    const int64_t max_chunks = (sk + kMinRowsPerChunk - 1) / kMinRowsPerChunk;
    if (nchunks > max_chunks) nchunks = max_chunks;
    if (nchunks > 1024) nchunks = 1024;
    if (nchunks > kNoAllocScratchFloats / (b * cols)) nchunks = kNoAllocScratchFloats / (b * cols);
    if (nchunks < 1) nchunks = 1;
    const int64_t rows_per_chunk = (sk + nchunks - 1) / nchunks;
    nchunks = (sk + rows_per_chunk - 1) / rows_per_chunk;

    // Every partial the fold reads is written by k_mean_partial first, so nothing needs clearing.
    dim3 g1((unsigned)col_ctas, (unsigned)nchunks, (unsigned)b);
    k_mean_partial<<<g1, kThreads, 0, st>>>(static_cast<const uint4*>(k), partial, sk, cols,
                                            rows_per_chunk, (int)nchunks);
    k_mean_fold<<<dim3((unsigned)((cols + 31) / 32), (unsigned)b), kThreads, 0, st>>>(
        partial, mean, cols, (int)nchunks, (float)sk);
    return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
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
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const int64_t stride = (sk + 2047) / 2048;  // every key up to 2048, else a strided sample
    const int64_t n_samp = (sk + stride - 1) / stride;
    const int64_t col_ctas = (cols + kColsPerCta - 1) / kColsPerCta;
    int64_t nchunks = (kTargetCtas + col_ctas * b - 1) / (col_ctas * b);
    // at least 32 sampled rows per chunk: fewer partials for the per-head fold to read
    const int64_t max_chunks = (n_samp + 31) / 32;
    if (nchunks > max_chunks) nchunks = max_chunks;
    if (nchunks > 1024) nchunks = 1024;
    if (nchunks < 1) nchunks = 1;
    const int64_t per_chunk = (n_samp + nchunks - 1) / nchunks;
    nchunks = (n_samp + per_chunk - 1) / per_chunk;

    float* partial = nullptr;
    cudaMemPool_t pool = scratch_pool();
    if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void**>(&partial),
                                         (size_t)(b * nchunks * 2 * cols) * sizeof(float), pool,
                                         st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    dim3 g1((unsigned)col_ctas, (unsigned)nchunks, (unsigned)b);
    k_gate_partial<<<g1, kThreads, 0, st>>>(static_cast<const uint4*>(k), partial, sk, cols,
                                            stride, n_samp, per_chunk, (int)nchunks);
    k_gate_fold<<<(unsigned)n_bg, kFoldThreads, 0, st>>>(partial, mean, gate, ratio, hk, d,
                                                         (int)nchunks, (float)n_samp, threshold);
    const bool launched = cudaGetLastError() == cudaSuccess;
    if (cudaFreeAsync(partial, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return launched ? B200ATTN_OK : B200ATTN_ERR_CUDA;
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
    int64_t blocks = (n + kThreads - 1) / kThreads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    k_sub_kernel<<<(unsigned)blocks, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k), mean, static_cast<uint4*>(k_out), b * sk, sk, cols);
    return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}
