// fp8_quant.cu -- fp8_quantize: E4M3 codes of a bf16 BSHD tensor, one fp32 scale per
// (batch, head), with the K channel mean optionally subtracted first (the quantized recipes of
// "[HIP] Mha v4: run the K-smoothing gate as one HIP call", Summary: smoothing before K is
// quantized).
//
// Two passes over x, both HBM-bound, in ONE cooperative launch (every CTA resident). A head's
// slice x[bi, :, hh, :] is s rows of d contiguous elements, 16-byte loads with one 8-element
// group per thread. Items are (batch, head, chunk of rows).
//   pass 1  each CTA takes its item's amax;
//   pass 2  it derives the factor 448 / amax of the item's head and converts the item's rows
//           (re-read, from L2 where they are still cached), 8 codes per thread; the head's first
//           chunk also writes the descale.
// With several chunks per head (few heads), every CTA holds at most one item; the chunk amaxes go
// to partials, and pass 2 starts once every CTA has published its partial (grid_sync.cuh) and
// folds its head's partials (max is exact, so any order gives the same amax). With one chunk per
// head (many heads), a CTA takes its items one after another and needs no grid-wide wait. Both
// passes compute x' = x - mean with the same fp32 subtraction, so the codes are exactly those of
// the definition in the header.
#include <cfloat>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <atomic>

#include "grid_sync.cuh"
#include "host_common.h"

namespace b200 {
namespace {

constexpr int kQThreads = 512;
constexpr int kQMaxChunks = 64;   // chunks per head slice at most (the fold: one load per thread)
constexpr int kQMaxGrid = 1024;   // CTAs of the launch at most (flag words)
constexpr unsigned kQTagKind = 0x6638u;  // top 16 bits of every flag tag of the quantiser

// The 8 elements of a 16-byte bf16 group (already loaded), minus the mean when given (one fp32
// subtraction).
__device__ __forceinline__ void unpack_group(const uint4& v, const float* m, float (&x)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        x[2 * t] = __uint_as_float(w[t] << 16);
        x[2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
    }
    if (m) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __fsub_rn(x[e], m[e]);
    }
}

// Problem geometry. Item it = (slice bh = bi * h + hh, chunk it % nch). Thread t of a CTA takes
// 16-byte group gi = t % G of a row and rows t / G, t / G + R, ... of its chunk, with G = d / 8
// groups per row and R = 512 / G rows per step.
struct QOnePass {
    const uint4* x;
    const float* mean;  // [b, h, d] or null
    uint2* x8;
    float* descale;
    float* partial;               // [n_items] chunk amaxes (nch > 1)
    unsigned long long* flags;    // [gridDim.x] flag words, then the go word at kQMaxGrid
    int64_t s, h, d8;             // rows, heads, 16-byte groups per row
    int64_t rows_per_chunk;
    int nch;                      // row chunks per head slice
    int64_t n_items;              // b * h * nch
    unsigned long long tag;
    int* status;
    unsigned long long timeout_ns;
};

// The 8 mean values of group gi of head slice bh (mean is [b, h, d] fp32).
__device__ __forceinline__ void head_mean(const float* mean, int64_t bh, int64_t d8, int gi,
                                          float (&mv)[8])
{
    const float4* m4 = reinterpret_cast<const float4*>(mean + (bh * d8 + gi) * 8);
    const float4 a = __ldg(m4), c = __ldg(m4 + 1);
    mv[0] = a.x; mv[1] = a.y; mv[2] = a.z; mv[3] = a.w;
    mv[4] = c.x; mv[5] = c.y; mv[6] = c.z; mv[7] = c.w;
}

// Max over the CTA's threads (non-negative inputs); the result is valid in warp 0.
__device__ __forceinline__ float block_max(float v, float* red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();  // red is free (a previous use has been read)
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kQThreads / 32 ? red[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    }
    return v;  // valid in warp 0
}

// max |x'| over the rows [s0, s1) of slice bh that this thread takes (twelve 16-byte loads in
// flight).
__device__ __forceinline__ float chunk_amax(const QOnePass& a, int64_t bh, int64_t s0, int64_t s1)
{
    const int G = (int)a.d8;
    const int gi = threadIdx.x % G;
    const int R = kQThreads / G;
    const int64_t bi = bh / a.h, hh = bh - bi * a.h;
    float mv[8];
    if (a.mean) head_mean(a.mean, bh, a.d8, gi, mv);
    const int64_t row_stride = a.h * a.d8;  // uint4 per sequence row
    const uint4* base = a.x + (bi * a.s * a.h + hh) * a.d8 + gi;
    float m = 0.f;
    int64_t r = s0 + threadIdx.x / G;
    for (; r + 11 * R < s1; r += 12 * R) {
        uint4 raw[12];
#pragma unroll
        for (int e = 0; e < 12; ++e) raw[e] = __ldg(base + (r + e * R) * row_stride);
#pragma unroll
        for (int e = 0; e < 12; ++e) {
            float v[8];
            unpack_group(raw[e], a.mean ? mv : nullptr, v);
#pragma unroll
            for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v[k]));
        }
    }
    for (; r < s1; r += R) {
        float v[8];
        unpack_group(__ldg(base + r * row_stride), a.mean ? mv : nullptr, v);
#pragma unroll
        for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v[k]));
    }
    return m;
}

// Codes of rows [s0, s1) of slice bh with factor f.
__device__ __forceinline__ void chunk_convert(const QOnePass& a, int64_t bh, int64_t s0,
                                              int64_t s1, float f)
{
    const int G = (int)a.d8;
    const int gi = threadIdx.x % G;
    const int R = kQThreads / G;
    const int64_t bi = bh / a.h, hh = bh - bi * a.h;
    float mv[8];
    if (a.mean) head_mean(a.mean, bh, a.d8, gi, mv);
    const int64_t row_stride = a.h * a.d8;
    const int64_t off = (bi * a.s * a.h + hh) * a.d8 + gi;
    int64_t r = s0 + threadIdx.x / G;
    for (; r < s1; r += 8 * R) {  // eight groups in flight
        uint4 raw[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (r + e * R < s1) raw[e] = __ldg(a.x + off + (r + e * R) * row_stride);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (r + e * R >= s1) break;
            float v[8];
            unpack_group(raw[e], a.mean ? mv : nullptr, v);
            uint32_t w[4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
                w[t] = (uint32_t)__nv_cvt_float2_to_fp8x2(
                    make_float2(__fmul_rn(v[2 * t], f), __fmul_rn(v[2 * t + 1], f)),
                    __NV_SATFINITE, __NV_E4M3);
            a.x8[off + (r + e * R) * row_stride] =
                make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
        }
    }
}

__device__ __forceinline__ float factor_of(float amax)
{
    return amax > 0.f ? fminf(448.f / amax, FLT_MAX) : 1.f;
}

__global__ void __launch_bounds__(kQThreads) fp8_quant_onepass(const QOnePass a)
{
    __shared__ float red[kQThreads / 32];
    __shared__ float amax_s;
    auto rows = [&](int64_t it, int64_t& s0, int64_t& s1) {
        s0 = (it % a.nch) * a.rows_per_chunk;
        s1 = s0 + a.rows_per_chunk < a.s ? s0 + a.rows_per_chunk : a.s;
    };
    if (a.nch == 1) {  // whole head slices, one after another: no grid-wide wait
        for (int64_t bh = blockIdx.x; bh < a.n_items; bh += gridDim.x) {
            float m = block_max(chunk_amax(a, bh, 0, a.s), red);
            if (threadIdx.x == 0) {
                amax_s = m;
                a.descale[bh] = m > 0.f ? m / 448.f : 1.f;
            }
            __syncthreads();
            chunk_convert(a, bh, 0, a.s, factor_of(amax_s));
        }
        return;
    }
    // several chunks per head: at most one item per CTA (the host sizes the split so)
    const int64_t it = blockIdx.x;
    int64_t s0 = 0, s1 = 0;
    if (it < a.n_items) {
        rows(it, s0, s1);
        const float m = block_max(chunk_amax(a, it / a.nch, s0, s1), red);
        if (threadIdx.x == 0) a.partial[it] = m;
    }
    publish_cta(a.flags, a.tag);
    if (!wait_all_published(a.flags, a.tag, (int)gridDim.x, (int)gridDim.x, a.flags + kQMaxGrid,
                            a.status, a.timeout_ns))
        return;
    if (it >= a.n_items) return;
    const int64_t bh = it / a.nch;
    float m = 0.f;
    if ((int)threadIdx.x < a.nch) m = __ldcg(a.partial + bh * a.nch + threadIdx.x);
    m = block_max(m, red);
    if (threadIdx.x == 0) {
        amax_s = m;
        if (it % a.nch == 0) a.descale[bh] = m > 0.f ? m / 448.f : 1.f;
    }
    __syncthreads();
    chunk_convert(a, bh, s0, s1, factor_of(amax_s));
}

std::atomic<int> g_quant_grid[64];

// Grid of the one-pass quantiser on the current device: one CTA per SM when one fits (cached per
// device; atomics: concurrent first calls store the same value), 0 on error.
int quant_grid()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 0;
    }
    int n = g_quant_grid[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        int per_sm = 0, sms = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fp8_quant_onepass, kQThreads,
                                                          0) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        n = per_sm >= 1 ? sms : 0;
        n = n < kQMaxGrid ? n : kQMaxGrid;
        g_quant_grid[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

}  // namespace
}  // namespace b200

using namespace b200;

extern "C" int fp8_quantize(const void* x, const float* mean, void* x8, float* descale, int64_t b,
                            int64_t s, int64_t h, int64_t d, void* stream)
{
    if (b < 0 || s < 0 || h < 0) return B200ATTN_ERR_SHAPE;
    if (!(d == 64 || d == 128 || d == 256)) return B200ATTN_ERR_HEADDIM;
    int64_t n, nbh;
    if (!numel({b, s, h, d, 2}, &n) || !numel({b, h}, &nbh) || !numel({b, h, d, 4}, &n) ||
        nbh >= ((int64_t)1 << 31))
        return B200ATTN_ERR_RANGE;
    if (nbh == 0) return B200ATTN_OK;
    if (!descale || (s > 0 && (!x || !x8))) return B200ATTN_ERR_NULL;
    if (!aligned(descale, 4) || (x && !aligned(x, 16)) || (x8 && !aligned(x8, 16)) ||
        (mean && !aligned(mean, 16)))
        return B200ATTN_ERR_ALIGN;
    int rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const int grid_max = quant_grid();
    int* status = status_word();
    if (grid_max <= 0 || !status) return B200ATTN_ERR_CUDA;

    QOnePass a{};
    a.x = static_cast<const uint4*>(x);
    a.mean = mean;
    a.x8 = static_cast<uint2*>(x8);
    a.descale = descale;
    a.s = s;
    a.h = h;
    a.d8 = d / 8;
    // Chunks per head: as many as keep every CTA at one item at most (few heads), else one (many
    // heads: whole slices, several per CTA); never more chunks than steps of R rows.
    const int64_t R = kQThreads / a.d8;  // rows per step of one CTA
    int64_t nch = nbh < grid_max ? grid_max / nbh : 1;
    const int64_t max_ch = (s + R - 1) / R;
    if (nch > max_ch) nch = max_ch;
    if (nch > kQMaxChunks) nch = kQMaxChunks;
    if (nch < 1) nch = 1;
    const int64_t rpc = s > 0 ? (s + nch - 1) / nch : 0;
    if (s > 0) nch = (s + rpc - 1) / rpc;
    a.rows_per_chunk = rpc;
    a.nch = (int)nch;
    a.n_items = nbh * nch;
    const int grid = (int)(a.n_items < grid_max ? a.n_items : grid_max);
    a.tag = next_call_tag(kQTagKind);
    a.status = status;
    a.timeout_ns = 4000000000ull;

    void* scratch = nullptr;
    const size_t part_bytes = ((size_t)a.n_items * sizeof(float) + 255) / 256 * 256;
    const size_t nbytes = part_bytes + (kQMaxGrid + 32) * sizeof(unsigned long long);
    cudaMemPool_t pool = scratch_pool();
    if (!pool || cudaMallocFromPoolAsync(&scratch, nbytes, pool, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    a.partial = static_cast<float*>(scratch);
    a.flags = reinterpret_cast<unsigned long long*>(static_cast<char*>(scratch) + part_bytes);
    void* args[] = {&a};
    const bool launched =
        cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(fp8_quant_onepass),
                                    dim3((unsigned)grid), dim3(kQThreads), args, 0, st) ==
        cudaSuccess;
    if (!launched) cudaGetLastError();
    if (cudaFreeAsync(scratch, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return launched ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}
