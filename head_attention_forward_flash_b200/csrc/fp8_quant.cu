// fp8_quant.cu -- fp8_quantize: E4M3 codes of a bf16 BSHD tensor, one fp32 scale per
// (batch, head), with the K channel mean optionally subtracted first (the quantized recipes of
// "[HIP] Mha v4: run the K-smoothing gate as one HIP call", Summary: smoothing before K is
// quantized).
//
// Two passes over x, both HBM-bound. A head's slice x[bi, :, hh, :] is s rows of d contiguous
// elements, 16-byte loads with one 8-element group per thread. (1) Every CTA takes one
// (batch, head) and a chunk of its rows and writes the chunk's amax to a partial. (2) Every CTA
// folds its head's partials (max is exact, so any order gives the same amax), derives the
// factor 448 / amax, converts its rows and writes 8 codes per thread; the first chunk's CTA also
// writes the descale. Both passes compute x' = x - mean with the same fp32 subtraction, so the
// codes are exactly those of the definition in the header.
#include <cfloat>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "host_common.h"

namespace b200 {
namespace {

constexpr int kQThreads = 256;
constexpr int kQTargetCtas = 4 * 148;  // about four waves on the 148 SMs

// The 8 elements of a 16-byte bf16 group, minus the mean when given (one fp32 subtraction).
__device__ __forceinline__ void load_group(const uint4* src, const float* m, float (&x)[8])
{
    const uint4 v = __ldg(src);
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

// Problem geometry of both passes. Grid: x = (batch, head) slice bh = bi * h + hh, y = row
// chunk. Thread t of a CTA takes 16-byte group gi = t % G of a row and rows t / G, t / G + R,
// ... of its chunk, with G = d / 8 groups per row and R = 256 / G rows per step.
struct QGeom {
    int64_t s, h, d8;  // rows, heads, 16-byte groups per row
    int64_t rows_per_chunk;
    int nch;           // row chunks per head slice
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

// Max over the CTA's 256 threads (non-negative inputs); the result is valid in warp 0.
__device__ __forceinline__ float block_max(float v, float* red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kQThreads / 32 ? red[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    }
    return v;  // valid in warp 0
}

// Pass 1: partial[bh * nch + chunk] = max |x'| over the chunk's rows of head slice bh.
__global__ void __launch_bounds__(kQThreads)
    fp8_amax_partial(const uint4* __restrict__ x, const float* __restrict__ mean,
                     float* __restrict__ partial, QGeom g)
{
    __shared__ float red[kQThreads / 32];
    const int64_t bh = blockIdx.x;  // bi * h + hh
    const int chunk = blockIdx.y;
    const int G = (int)g.d8;
    const int gi = threadIdx.x % G;
    const int R = kQThreads / G;
    const int64_t bi = bh / g.h, hh = bh - bi * g.h;
    float mv[8];
    if (mean) head_mean(mean, bh, g.d8, gi, mv);
    const int64_t s0 = (int64_t)chunk * g.rows_per_chunk;
    const int64_t s1 = s0 + g.rows_per_chunk < g.s ? s0 + g.rows_per_chunk : g.s;
    const int64_t row_stride = g.h * g.d8;  // uint4 per sequence row
    const uint4* base = x + (bi * g.s * g.h + hh) * g.d8 + gi;
    float m = 0.f;
    int64_t r = s0 + threadIdx.x / G;
    for (; r + 3 * R < s1; r += 4 * R) {  // four 16-byte loads in flight
        float a[8], b[8], c[8], e[8];
        load_group(base + r * row_stride, mean ? mv : nullptr, a);
        load_group(base + (r + R) * row_stride, mean ? mv : nullptr, b);
        load_group(base + (r + 2 * R) * row_stride, mean ? mv : nullptr, c);
        load_group(base + (r + 3 * R) * row_stride, mean ? mv : nullptr, e);
#pragma unroll
        for (int k = 0; k < 8; ++k)
            m = fmaxf(fmaxf(m, fmaxf(fabsf(a[k]), fabsf(b[k]))), fmaxf(fabsf(c[k]), fabsf(e[k])));
    }
    for (; r < s1; r += R) {
        float a[8];
        load_group(base + r * row_stride, mean ? mv : nullptr, a);
#pragma unroll
        for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(a[k]));
    }
    m = block_max(m, red);
    if (threadIdx.x == 0) partial[bh * g.nch + chunk] = m;
}

// Pass 2: fold the head's partials, then write the chunk's codes (and, chunk 0, the descale).
__global__ void __launch_bounds__(kQThreads)
    fp8_convert(const uint4* __restrict__ x, const float* __restrict__ mean,
                const float* __restrict__ partial, uint2* __restrict__ x8,
                float* __restrict__ descale, QGeom g)
{
    __shared__ float red[kQThreads / 32];
    __shared__ float amax_s;
    const int64_t bh = blockIdx.x;
    const int chunk = blockIdx.y;
    float m = 0.f;
    for (int c = threadIdx.x; c < g.nch; c += kQThreads) m = fmaxf(m, partial[bh * g.nch + c]);
    m = block_max(m, red);
    if (threadIdx.x == 0) amax_s = m;
    __syncthreads();
    const float amax = amax_s;
    const float f = amax > 0.f ? fminf(448.f / amax, FLT_MAX) : 1.f;
    if (chunk == 0 && threadIdx.x == 0) descale[bh] = amax > 0.f ? amax / 448.f : 1.f;

    const int G = (int)g.d8;
    const int gi = threadIdx.x % G;
    const int R = kQThreads / G;
    const int64_t bi = bh / g.h, hh = bh - bi * g.h;
    float mv[8];
    if (mean) head_mean(mean, bh, g.d8, gi, mv);
    const int64_t s0 = (int64_t)chunk * g.rows_per_chunk;
    const int64_t s1 = s0 + g.rows_per_chunk < g.s ? s0 + g.rows_per_chunk : g.s;
    const int64_t row_stride = g.h * g.d8;
    const int64_t off = (bi * g.s * g.h + hh) * g.d8 + gi;
    for (int64_t r = s0 + threadIdx.x / G; r < s1; r += R) {
        float a[8];
        load_group(x + off + r * row_stride, mean ? mv : nullptr, a);
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            w[t] = (uint32_t)__nv_cvt_float2_to_fp8x2(
                make_float2(__fmul_rn(a[2 * t], f), __fmul_rn(a[2 * t + 1], f)), __NV_SATFINITE,
                __NV_E4M3);
        x8[off + r * row_stride] = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
    }
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

    QGeom g;
    g.s = s;
    g.h = h;
    g.d8 = d / 8;
    const int64_t R = kQThreads / g.d8;  // rows per step of one CTA
    int64_t nch = (kQTargetCtas + nbh - 1) / nbh;
    const int64_t max_ch = (s + R - 1) / R;
    if (nch > max_ch) nch = max_ch;
    if (nch > 1024) nch = 1024;
    if (nch < 1) nch = 1;
    int64_t rpc = (s + nch - 1) / nch;
    rpc = (rpc + R - 1) / R * R;
    if (rpc < R) rpc = R;
    nch = s > 0 ? (s + rpc - 1) / rpc : 1;
    g.rows_per_chunk = rpc;
    g.nch = (int)nch;

    float* partial = nullptr;
    cudaMemPool_t pool = scratch_pool();
    if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void**>(&partial),
                                         (size_t)(nbh * nch) * sizeof(float), pool,
                                         st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    const dim3 grid((unsigned)nbh, (unsigned)nch);
    fp8_amax_partial<<<grid, kQThreads, 0, st>>>(static_cast<const uint4*>(x), mean, partial, g);
    fp8_convert<<<grid, kQThreads, 0, st>>>(static_cast<const uint4*>(x), mean, partial,
                                            static_cast<uint2*>(x8), descale, g);
    const bool launched = cudaGetLastError() == cudaSuccess;
    if (cudaFreeAsync(partial, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return launched ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}
