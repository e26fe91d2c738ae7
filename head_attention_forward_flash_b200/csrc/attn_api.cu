// attn_api.cu -- C-ABI entry points attn_fwd, attn_fwd_varlen, attn_fwd_window_sink,
// attn_fwd_fp8, attn_status_string, attn_debug_status and attn_debug_starve:
// argument checks, TMA descriptor encoding, head-dim dispatch and the kernel launch.
#include <cmath>
#include <cstring>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <atomic>
#include <mutex>

#include "attn_fwd_kernel.cuh"
#include "host_common.h"

namespace b200 {

// Device error word written by kernels whose bounded waits give up.
__device__ int g_attn_status;

// Failure test armed by attn_debug_starve: the wait limit of the next attention launch, or 0.
std::mutex g_starve_mu;
unsigned long long g_starve_timeout_ns = 0;

// Device address of the error word on the current device (the host-side name of a __device__
// variable is not a device address), cached per device. The per-device caches of this library
// are atomics: concurrent first calls from several host threads store the same value, and no
// thread reads a half-written one.
int* status_word()
{
    static std::atomic<int*> addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int* a = addr[dev].load(std::memory_order_relaxed);
    if (a == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_attn_status) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        a = static_cast<int*>(p);
        addr[dev].store(a, std::memory_order_relaxed);
    }
    return a;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 4-D tensor map over a BSHD tensor [b, s, h, d] (innermost first: d, h, s, b) of bf16
// (eb = 2) or 8-bit codes (eb = 1), box {128 bytes of channels, 1 head, box_rows rows, 1 batch},
// 128-byte swizzle, zero fill out of bounds.
int encode_bshd(CUtensorMap* map, const void* base, int64_t b, int64_t s, int64_t h, int64_t d,
                int box_rows, int eb = 2)
{
    auto fn = encode_fn();
    if (!fn) return B200ATTN_ERR_CUDA;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)h, (cuuint64_t)s, (cuuint64_t)b};
    const cuuint64_t strides[3] = {(cuuint64_t)(d * eb), (cuuint64_t)(h * d * eb),
                                   (cuuint64_t)(s * h * d * eb)};
    const cuuint32_t box[4] = {(cuuint32_t)(128 / eb), 1, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, eb == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    4, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}

// The TMA unit addresses at most 2^32 elements per dimension and byte strides below 2^40.
bool tma_extent_ok(int64_t b, int64_t s, int64_t h, int64_t d)
{
    const int64_t lim_dim = (int64_t)1 << 31;  // coordinates are signed 32-bit
    const int64_t lim_stride = (int64_t)1 << 40;
    if (b >= lim_dim || s >= lim_dim || h >= lim_dim || d >= lim_dim) return false;
    int64_t st;
    if (!numel({s, h, d, 2}, &st)) return false;
    return st < lim_stride;
}

int sm_count()
{
    static std::atomic<int> cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Problem geometry. Dense: b batches of sq queries and sk keys. Packed sequences: b sequences,
// sq = the longest query length, the per-sequence offsets in cu_q / cu_k (device memory), and
// the tensors' total row counts.
struct Shape {
    int64_t b, hq, hk, sq, sk;
    const int* cu_q = nullptr;
    const int* cu_k = nullptr;
    int64_t total_q = 0, total_k = 0;
    int64_t window = -1;          // left window, < 0: none
    const float* sinks = nullptr;  // per query head sink logits, or null
    // E4M3 inputs: per (batch, head) descales of Q [b, hq], K and V [b, hk]
    const float* q_descale = nullptr;
    const float* k_descale = nullptr;
    const float* v_descale = nullptr;
};

template <class T, bool CAUSAL, bool VARLEN, bool EXT>
int launch_attn(const void* q, const void* k, const void* v, void* out, float* lse,
                const Shape& sh, float scale, cudaStream_t stream)
{
    const int64_t b = sh.b, hq = sh.hq, hk = sh.hk, sq = sh.sq, sk = sh.sk;
    static std::atomic<bool> attr_done[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    auto kern = attn_fwd_kernel<T, CAUSAL, VARLEN, EXT>;
    if (!attr_done[dev].load(std::memory_order_relaxed)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)T::SMEM_BYTES) != cudaSuccess) {
            cudaGetLastError();
            return B200ATTN_ERR_CUDA;
        }
        // With two softmax warpgroups the kernel moves registers between warpgroups; the
        // softmax warps' raise is granted only from what the block was launched with, so a
        // build launched with fewer registers per thread would stall for good: refuse it.
        if (T::NSM == 2) {
            cudaFuncAttributes fa;
            if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) {
                cudaGetLastError();
                return B200ATTN_ERR_CUDA;
            }
            if ((int64_t)fa.numRegs * T::NUM_THREADS <
                (int64_t)2 * 128 * T::SOFTMAX_REGS + 128 * T::AUX_REGS)
                return B200ATTN_ERR_CUDA;
        }
        attr_done[dev].store(true, std::memory_order_relaxed);
    }
    // packed sequences: one batch of all rows; each unit adds its sequence's first row
    const int64_t mb = VARLEN ? 1 : b;
    const int64_t mq = VARLEN ? sh.total_q : sq;
    const int64_t mk = VARLEN ? sh.total_k : sk;
    CUtensorMap tq, tk, tv, to;
    int rc = encode_bshd(&tq, q, mb, mq, hq, T::DQK, T::BM, T::EB);
    if (rc == B200ATTN_OK) rc = encode_bshd(&tk, k, mb, mk, hk, T::DQK, T::BN, T::EB);
    if (rc == B200ATTN_OK) rc = encode_bshd(&tv, v, mb, mk, hk, T::DV, T::BN, T::EB);
    // O is stored per warp: boxes of 32 rows (only used when the kernel stages O for TMA)
    if (rc == B200ATTN_OK) rc = encode_bshd(&to, out, mb, mq, hq, T::DV, 32);
    if (rc != B200ATTN_OK) return rc;
    int* status = status_word();
    const int n_sm = sm_count();
    if (!status || n_sm <= 0) return B200ATTN_ERR_CUDA;

    AttnParams p;
    p.o = static_cast<__nv_bfloat16*>(out);
    p.lse = lse;
    p.b = b;
    p.hq = hq;
    p.hk = hk;
    p.sq = sq;
    p.sk = sk;
    p.cu_q = sh.cu_q;
    p.cu_k = sh.cu_k;
    p.total_q = sh.total_q;
    p.total_k = sh.total_k;
    p.window = sh.window;
    p.sinks = sh.sinks;
    p.q_descale = sh.q_descale;
    p.k_descale = sh.k_descale;
    p.v_descale = sh.v_descale;
    p.group = hq / hk;
    p.n_qu = (sq + T::NT * T::BM - 1) / (T::NT * T::BM);
    p.n_units = b * hq * p.n_qu;  // below 2^31 (checked by attn_fwd)
    p.div_nqu = make_fastdiv((uint32_t)p.n_qu);
    p.div_hq = make_fastdiv((uint32_t)hq);
    p.div_group = make_fastdiv((uint32_t)p.group);
    p.div_bh = make_fastdiv((uint32_t)(b * hq > 0 ? b * hq : 1));
    // Unit order (measured on B200 at 8x48:8 2048^2 d64, 128 heads 8192^2 d192/128 and 5 heads
    // 65536^2 d128, all causal). Causal units differ in cost, so CTAs take them in snake order
    // (odd rounds reversed), which evens out the per-CTA totals; where every head's K/V fits in
    // L2 or the kv heads are few, in weight-major order (all heads' heaviest units first), which
    // evens them out best; where many heads' K/V far exceed L2, head-major, so that the CTAs
    // working at the same time share a few heads' K/V. Equal-cost units (no causal mask, or a
    // window band) take plain round robin. Packed sequences rank each sequence's units from its
    // own last query tile (unit_info); with at most kMaxUnitClasses (sequence, rank) classes the
    // kernel sorts the classes by cost and hands them out heaviest first (order 3: interleaved
    // A/B on B200, 8 packed sequences of 1024-2048 keys, hq48:hk8 d64 causal), else weight-major
    // order hands out every sequence's k-th most expensive unit in round k.
    {
        const double kv_bytes =
            (double)(b * sk) * (double)hk * (double)(T::DQK + T::DV) * (double)T::EB;
        if (VARLEN && b * p.n_qu <= kMaxUnitClasses)
            p.order = 3;
        else if (!CAUSAL || (EXT && sh.window >= 0))
            p.order = 0;
        else if (VARLEN)
            p.order = 2;
        else if (b * hk <= 16 || kv_bytes <= 64.0e6)
            p.order = 2;
        else
            p.order = 1;
    }
    // The MMA applies the sign of the scale (negate-A bit of the instruction descriptor), so
    // the softmax only ever sees a non-negative factor. It is kept at 2^-100 or more, so that a
    // masked score of -inf always maps to exp2(-inf) = 0. For |scale| below that (scale 0
    // included) and scores below 2^40 in magnitude, every exp2 argument is then below 2^-60,
    // so each p rounds to exactly 1 in fp32 -- the same weights the unclamped scale gives.
    const double sl2 = std::fabs((double)scale) * 1.4426950408889634;
    p.scale_log2 = (float)(sl2 > 0x1p-100 ? sl2 : 0x1p-100);
    p.idesc_qk = T::IDESC_QK | (scale < 0.f ? (1u << 13) : 0u);
    p.status = status;
    p.timeout_ns = 4000000000ull;  // 4 s: far above any legitimate wait
    p.starve = 0;
    // Two tiles: their softmax take turns (measured on B200: each body then runs alone, at
    // about 1 400 instead of 2 000 cycles per 128 x 128 block while both run together).
    p.alt = T::NT == 2 ? 1 : 0;
    {
        // a pending failure test (attn_debug_starve) applies to this one launch
        std::lock_guard<std::mutex> lk(g_starve_mu);
        if (g_starve_timeout_ns > 0) {
            p.starve = 1;
            p.timeout_ns = g_starve_timeout_ns;
            g_starve_timeout_ns = 0;
        }
    }

    const int64_t grid = p.n_units < n_sm ? p.n_units : n_sm;  // persistent: one CTA per SM
    kern<<<(unsigned)grid, T::NUM_THREADS, T::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
    if (cudaGetLastError() != cudaSuccess) return B200ATTN_ERR_CUDA;
    return B200ATTN_OK;
}

// Head-dim table: (dqk, dv) -> <DQK, DV, keys per block, query tiles per unit, softmax
// warpgroups, Q in TMEM, K slots, V slots, score pairs whose exp2 runs on the FMA pipe, E4M3
// inputs, pipelined two-tile layout>. Shared memory holds the Q staging buffer and the K / V
// rings (and, when it fits, the O staging tile). Measured on B200 (TFLOP/s, causal-halved):
//  - d64: the pipelined layout (two 64-key score buffers per tile, the two tiles' softmax side
//    by side): b8 hq48:hk8 2048^2 causal 501 vs 455 with one 128-key buffer per tile; 8192^2
//    with a 128-key window and sinks 119 vs 80.
//  - d128, d192/128: one 128-key score buffer per tile, the tiles' softmax taking turns (the
//    pipelined layout's 64-key Q K^T from shared memory runs at 2/3 of the tensor rate: 1027 vs
//    1041 at 65536^2 d128, 996 vs 1021 at 8192^2 d192/128).
//  - d256: one tile, two 64-key score buffers.
// The share of score pairs whose exp2 runs on the FMA pipe is the measured best per head dim:
// 3 of 8 at d128 (pairs 0, 2, 5 of every 8: 1141 vs 1060 with 2 of 8 at 65536^2, interleaved
// A/B), 2 of 8 at d192 (3 of 8 is no faster there) and for E4M3 inputs (3 of 8 loses 1-3 %),
// none at d256, bound by the tensor core. At d64, 3 of 8 (pairs 1, 4, 7) measured best (none:
// -7 %, 4 of 8: -3 %).
using T64P = AttnTraits<64, 64, 64, 2, 2, true, 8, 8, 0x92u, false, true>;  // 32 + 64 + 64 (+32) KB
using T128 = AttnTraits<128, 128, 128, 2, 2, false, 3, 2, 0x25u>;         // 64 + 96 + 64 KB
using T192 = AttnTraits<192, 128, 128, 2, 2, false, 2, 1, 0x11u>;         // 96 + 96 + 32 KB
using T256 = AttnTraits<256, 256, 64, 1, 1, true, 2, 2>;                  // 64 + 64 + 64 KB
// E4M3 inputs, (128, 128): the d128 layout with half-size tiles, so eight K and V slots fit next
// to the Q staging buffer and the O staging tile: five K and three V (measured on B200, 5 x
// 65536^2 causal: +0.5-0.7 % against four and four, three and five in between).
using T128F8 = AttnTraits<128, 128, 128, 2, 2, false, 5, 3, 0x11u, true>;  // 32 + 80 + 48 (+64) KB

// Kernel variants: dense, dense with window / sinks (compiled apart so that the plain path
// carries none of the extra bound logic), and packed sequences.
template <class T>
int dispatch_dense(int causal, const void* q, const void* k, const void* v, void* out,
                   float* lse, const Shape& sh, float scale, cudaStream_t st)
{
    if (sh.window >= 0 || sh.sinks)
        return causal ? launch_attn<T, true, false, true>(q, k, v, out, lse, sh, scale, st)
                      : launch_attn<T, false, false, true>(q, k, v, out, lse, sh, scale, st);
    return causal ? launch_attn<T, true, false, false>(q, k, v, out, lse, sh, scale, st)
                  : launch_attn<T, false, false, false>(q, k, v, out, lse, sh, scale, st);
}

template <class T>
int dispatch_varlen(int causal, const void* q, const void* k, const void* v, void* out,
                    float* lse, const Shape& sh, float scale, cudaStream_t st)
{
    return causal ? launch_attn<T, true, true, false>(q, k, v, out, lse, sh, scale, st)
                  : launch_attn<T, false, true, false>(q, k, v, out, lse, sh, scale, st);
}

// Packed sequences take the dense layouts (equal-length packed input is then bitwise the dense
// result).
int dispatch_dims(int64_t dqk, int causal, bool varlen, const void* q, const void* k,
                  const void* v, void* out, float* lse, const Shape& sh, float scale,
                  cudaStream_t st)
{
    if (varlen) {
        switch (dqk) {
        case 64: return dispatch_varlen<T64P>(causal, q, k, v, out, lse, sh, scale, st);
        case 128: return dispatch_varlen<T128>(causal, q, k, v, out, lse, sh, scale, st);
        case 192: return dispatch_varlen<T192>(causal, q, k, v, out, lse, sh, scale, st);
        default: return dispatch_varlen<T256>(causal, q, k, v, out, lse, sh, scale, st);
        }
    }
    switch (dqk) {
    case 64: return dispatch_dense<T64P>(causal, q, k, v, out, lse, sh, scale, st);
    case 128: return dispatch_dense<T128>(causal, q, k, v, out, lse, sh, scale, st);
    case 192: return dispatch_dense<T192>(causal, q, k, v, out, lse, sh, scale, st);
    default: return dispatch_dense<T256>(causal, q, k, v, out, lse, sh, scale, st);
    }
}

// Rows with no key at all (sk == 0): O = 0, LSE = -inf, or the head's sink logit when sinks
// are given (LSE [b, hq, sq]: entry t belongs to head (t / sq) % hq).
__global__ void fill_empty_rows(__nv_bfloat16* out, int64_t n_out, float* lse, int64_t n_lse,
                                const float* sinks = nullptr, int64_t hq = 1, int64_t sq = 1)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_out; t += stride)
        out[t] = __float2bfloat16_rn(0.f);
    if (lse)
        for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_lse; t += stride)
            lse[t] = sinks ? sinks[(t / sq) % hq] : -INFINITY;
}

}  // namespace
}  // namespace b200

using namespace b200;

extern "C" int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                        int64_t b, int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk,
                        int64_t dv, int causal, float scale, void* stream)
{
    if (b < 0 || hq < 0 || sq < 0 || sk < 0 || hk <= 0) return B200ATTN_ERR_SHAPE;
    if (hq % hk != 0) return B200ATTN_ERR_GQA;
    const bool hd_ok = (dqk == 64 && dv == 64) || (dqk == 128 && dv == 128) ||
                       (dqk == 192 && dv == 128) || (dqk == 256 && dv == 256);
    if (!hd_ok) return B200ATTN_ERR_HEADDIM;
    if (!std::isfinite(scale)) return B200ATTN_ERR_SCALE;
    int64_t n_q, n_k, n_v, n_o, n_l;
    if (!numel({b, sq, hq, dqk}, &n_q) || !numel({b, sk, hk, dqk}, &n_k) ||
        !numel({b, sk, hk, dv}, &n_v) || !numel({b, sq, hq, dv}, &n_o) ||
        !numel({b, hq, sq}, &n_l) || !numel({n_q, 2}, &n_q) || !numel({n_k, 2}, &n_k) ||
        !numel({n_v, 2}, &n_v) || !numel({n_o, 2}, &n_o) || !numel({n_l, 4}, &n_l))
        return B200ATTN_ERR_RANGE;
    if (n_o == 0) return B200ATTN_OK;  // b, hq or sq is zero: nothing to compute
    if (!q || !out || (sk > 0 && (!k || !v))) return B200ATTN_ERR_NULL;
    if (!aligned(q, 16) || !aligned(out, 16) || (k && !aligned(k, 16)) ||
        (v && !aligned(v, 16)) || (lse && !aligned(lse, 4)))
        return B200ATTN_ERR_ALIGN;
    if (!tma_extent_ok(b, sq, hq, dqk) ||
        (sk > 0 && (!tma_extent_ok(b, sk, hk, dqk) || !tma_extent_ok(b, sk, hk, dv))))
        return B200ATTN_ERR_RANGE;
    // Work units (b * hq * query tiles) are numbered in 31 bits.
    int64_t n_units;
    if (!numel({b, hq, (sq + 127) / 128}, &n_units) || n_units >= ((int64_t)1 << 31))
        return B200ATTN_ERR_RANGE;
    int rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (sk == 0) {
        fill_empty_rows<<<296, 256, 0, st>>>(static_cast<__nv_bfloat16*>(out), n_o / 2, lse,
                                             n_l / 4);
        return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
    }
    Shape sh;
    sh.b = b;
    sh.hq = hq;
    sh.hk = hk;
    sh.sq = sq;
    sh.sk = sk;
    return dispatch_dims(dqk, causal, false, q, k, v, out, lse, sh, scale, st);
}

extern "C" int attn_fwd_window_sink(const void* q, const void* k, const void* v, void* out,
                                    float* lse, const float* sinks, int64_t b, int64_t hq,
                                    int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
                                    int causal, int64_t window_left, float scale, void* stream)
{
    if (b < 0 || hq < 0 || sq < 0 || sk < 0 || hk <= 0) return B200ATTN_ERR_SHAPE;
    if (hq % hk != 0) return B200ATTN_ERR_GQA;
    const bool hd_ok = (dqk == 64 && dv == 64) || (dqk == 128 && dv == 128) ||
                       (dqk == 192 && dv == 128) || (dqk == 256 && dv == 256);
    if (!hd_ok) return B200ATTN_ERR_HEADDIM;
    if (!std::isfinite(scale)) return B200ATTN_ERR_SCALE;
    int64_t n_q, n_k, n_v, n_o, n_l, n_units;
    if (!numel({b, sq, hq, dqk}, &n_q) || !numel({b, sk, hk, dqk}, &n_k) ||
        !numel({b, sk, hk, dv}, &n_v) || !numel({b, sq, hq, dv}, &n_o) ||
        !numel({b, hq, sq}, &n_l) || !numel({n_q, 2}, &n_q) || !numel({n_k, 2}, &n_k) ||
        !numel({n_v, 2}, &n_v) || !numel({n_o, 2}, &n_o) || !numel({n_l, 4}, &n_l) ||
        !numel({b, hq, (sq + 127) / 128}, &n_units) || n_units >= ((int64_t)1 << 31))
        return B200ATTN_ERR_RANGE;
    if (n_o == 0) return B200ATTN_OK;  // b, hq or sq is zero: nothing to compute
    if (!q || !out || (sk > 0 && (!k || !v))) return B200ATTN_ERR_NULL;
    if (!aligned(q, 16) || !aligned(out, 16) || (k && !aligned(k, 16)) ||
        (v && !aligned(v, 16)) || (lse && !aligned(lse, 4)) || (sinks && !aligned(sinks, 4)))
        return B200ATTN_ERR_ALIGN;
    if (!tma_extent_ok(b, sq, hq, dqk) ||
        (sk > 0 && (!tma_extent_ok(b, sk, hk, dqk) || !tma_extent_ok(b, sk, hk, dv))))
        return B200ATTN_ERR_RANGE;
    int rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (sk == 0) {
        fill_empty_rows<<<296, 256, 0, st>>>(static_cast<__nv_bfloat16*>(out), n_o / 2, lse,
                                             n_l / 4, sinks, hq, sq);
        return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
    }
    Shape sh;
    sh.b = b;
    sh.hq = hq;
    sh.hk = hk;
    sh.sq = sq;
    sh.sk = sk;
    sh.window = window_left < 0 ? -1 : window_left;
    sh.sinks = sinks;
    return dispatch_dims(dqk, causal, false, q, k, v, out, lse, sh, scale, st);
}

extern "C" int attn_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                               const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int64_t b,
                               int64_t hq, int64_t hk, int64_t total_q, int64_t total_k,
                               int64_t max_sq, int64_t dqk, int64_t dv, int causal, float scale,
                               void* stream)
{
    if (b < 0 || hq < 0 || hk <= 0 || total_q < 0 || total_k < 0 || max_sq < 0)
        return B200ATTN_ERR_SHAPE;
    if (hq % hk != 0) return B200ATTN_ERR_GQA;
    const bool hd_ok = (dqk == 64 && dv == 64) || (dqk == 128 && dv == 128) ||
                       (dqk == 192 && dv == 128) || (dqk == 256 && dv == 256);
    if (!hd_ok) return B200ATTN_ERR_HEADDIM;
    if (!std::isfinite(scale)) return B200ATTN_ERR_SCALE;
    int64_t n_q, n_k, n_v, n_o, n_l, n_units;
    if (!numel({total_q, hq, dqk, 2}, &n_q) || !numel({total_k, hk, dqk, 2}, &n_k) ||
        !numel({total_k, hk, dv, 2}, &n_v) || !numel({total_q, hq, dv, 2}, &n_o) ||
        !numel({hq, total_q, 4}, &n_l) || !numel({b, hq, (max_sq + 127) / 128}, &n_units) ||
        n_units >= ((int64_t)1 << 31) || total_q >= ((int64_t)1 << 31) ||
        total_k >= ((int64_t)1 << 31) || b >= ((int64_t)1 << 31))
        return B200ATTN_ERR_RANGE;
    if (n_o == 0 || b == 0 || max_sq == 0) return B200ATTN_OK;  // no query row to compute
    if (!q || !out || !cu_seqlens_q || !cu_seqlens_k || (total_k > 0 && (!k || !v)))
        return B200ATTN_ERR_NULL;
    if (!aligned(q, 16) || !aligned(out, 16) || (k && !aligned(k, 16)) ||
        (v && !aligned(v, 16)) || (lse && !aligned(lse, 4)) || !aligned(cu_seqlens_q, 4) ||
        !aligned(cu_seqlens_k, 4))
        return B200ATTN_ERR_ALIGN;
    if (!tma_extent_ok(1, total_q, hq, dqk) ||
        (total_k > 0 && (!tma_extent_ok(1, total_k, hk, dqk) || !tma_extent_ok(1, total_k, hk, dv))))
        return B200ATTN_ERR_RANGE;
    int rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (total_k == 0) {  // no keys anywhere: every query row gets O = 0, LSE = -inf
        fill_empty_rows<<<296, 256, 0, st>>>(static_cast<__nv_bfloat16*>(out), n_o / 2, lse,
                                             n_l / 4);
        return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
    }
    Shape sh;
    sh.b = b;
    sh.hq = hq;
    sh.hk = hk;
    sh.sq = max_sq;
    sh.sk = 0;
    sh.cu_q = cu_seqlens_q;
    sh.cu_k = cu_seqlens_k;
    sh.total_q = total_q;
    sh.total_k = total_k;
    return dispatch_dims(dqk, causal, true, q, k, v, out, lse, sh, scale, st);
}

extern "C" int attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_descale,
                            const float* k_descale, const float* v_descale, void* out, float* lse,
                            int64_t b, int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk,
                            int64_t dv, int causal, float scale, void* stream)
{
    if (b < 0 || hq < 0 || sq < 0 || sk < 0 || hk <= 0) return B200ATTN_ERR_SHAPE;
    if (hq % hk != 0) return B200ATTN_ERR_GQA;
    if (!(dqk == 128 && dv == 128)) return B200ATTN_ERR_HEADDIM;
    if (!std::isfinite(scale)) return B200ATTN_ERR_SCALE;
    int64_t n_q, n_k, n_v, n_o, n_l, n_units;
    if (!numel({b, sq, hq, dqk}, &n_q) || !numel({b, sk, hk, dqk}, &n_k) ||
        !numel({b, sk, hk, dv}, &n_v) || !numel({b, sq, hq, dv, 2}, &n_o) ||
        !numel({b, hq, sq, 4}, &n_l) || !numel({b, hq, (sq + 127) / 128}, &n_units) ||
        n_units >= ((int64_t)1 << 31))
        return B200ATTN_ERR_RANGE;
    if (n_o == 0) return B200ATTN_OK;  // b, hq or sq is zero: nothing to compute
    if (!q8 || !out || !q_descale || (sk > 0 && (!k8 || !v8 || !k_descale || !v_descale)))
        return B200ATTN_ERR_NULL;
    if (!aligned(q8, 16) || !aligned(out, 16) || (k8 && !aligned(k8, 16)) ||
        (v8 && !aligned(v8, 16)) || (lse && !aligned(lse, 4)) || !aligned(q_descale, 4) ||
        (k_descale && !aligned(k_descale, 4)) || (v_descale && !aligned(v_descale, 4)))
        return B200ATTN_ERR_ALIGN;
    if (!tma_extent_ok(b, sq, hq, dqk) ||
        (sk > 0 && (!tma_extent_ok(b, sk, hk, dqk) || !tma_extent_ok(b, sk, hk, dv))))
        return B200ATTN_ERR_RANGE;
    int rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (sk == 0) {
        fill_empty_rows<<<296, 256, 0, st>>>(static_cast<__nv_bfloat16*>(out), n_o / 2, lse,
                                             n_l / 4);
        return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
    }
    Shape sh;
    sh.b = b;
    sh.hq = hq;
    sh.hk = hk;
    sh.sq = sq;
    sh.sk = sk;
    sh.q_descale = q_descale;
    sh.k_descale = k_descale;
    sh.v_descale = v_descale;
    return causal ? launch_attn<T128F8, true, false, false>(q8, k8, v8, out, lse, sh, scale, st)
                  : launch_attn<T128F8, false, false, false>(q8, k8, v8, out, lse, sh, scale, st);
}

extern "C" const char* attn_status_string(int status)
{
    switch (status) {
    case B200ATTN_OK: return "ok";
    case B200ATTN_ERR_NULL: return "a required pointer is NULL";
    case B200ATTN_ERR_SHAPE: return "invalid shape (negative size, or hk <= 0)";
    case B200ATTN_ERR_GQA: return "hq is not a multiple of hk";
    case B200ATTN_ERR_HEADDIM:
        return "unsupported head dims ((dqk,dv) must be (64,64), (128,128), (192,128) or "
               "(256,256); d for the K mean must be 64, 128 or 256)";
    case B200ATTN_ERR_ALIGN: return "pointer misaligned (bf16 tensors need 16 bytes, fp32 4)";
    case B200ATTN_ERR_RANGE: return "size or byte extent out of range";
    case B200ATTN_ERR_SCALE: return "scale is not finite";
    case B200ATTN_ERR_ARCH: return "device is not compute capability 10.0 (sm_100)";
    case B200ATTN_ERR_CUDA: return "CUDA call or kernel launch failed";
    case B200ATTN_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
    case B200ATTN_ERR_SCRATCH:
        return "b*hk*d exceeds the fixed scratch of k_smooth_mean_noalloc (2^20 floats)";
    default: return "unknown status";
    }
}

extern "C" int attn_debug_starve(int64_t timeout_us)
{
    if (timeout_us < 1 || timeout_us > 1000000) return B200ATTN_ERR_RANGE;
    std::lock_guard<std::mutex> lk(g_starve_mu);
    g_starve_timeout_ns = (unsigned long long)timeout_us * 1000ull;
    return B200ATTN_OK;
}

extern "C" int attn_debug_status(void* stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_attn_status, sizeof v) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_attn_status, &zero, sizeof zero);
    }
    return v;
}
