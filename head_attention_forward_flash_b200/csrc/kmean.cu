// kmean.cu -- the K channel-mean pre-pass (k_smooth_mean, k_smooth_mean_noalloc), the K-smoothing
// gate (k_smooth_gate), the mean subtraction (k_smooth_sub) and both steps in one launch
// (k_smooth_mean_sub).
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
// one HIP call" (Summary, commit message) become two phases of one kernel. The fused mean and
// subtraction adds
//   phase 3  the fold CTAs publish their columns of the mean in a second set of flags; once every
//            one has, all CTAs write K - mean, re-reading K (from L2 when it fits there).
#include <atomic>
#include <cmath>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "grid_sync.cuh"
#include "host_common.h"
#include "sm100_ptx.cuh"

namespace b200 {
namespace {

constexpr int kThreads = 512;  // one-pass kernels: each thread owns 8 consecutive channels
constexpr int kColsPerCta = kThreads * 8;
constexpr int kFoldWarps = kThreads / 32;
constexpr int kSubThreads = 256;
constexpr unsigned kTagKind = 0x6B6Du;  // top 16 bits of every flag tag of these kernels
constexpr int kMaxGrid = 1024;  // CTAs of a one-pass launch at most (flag words per set)
constexpr int kGo1 = kMaxGrid, kGo2 = kMaxGrid + 16;  // go words after the phase-1 flags
constexpr int kFlagWords = kMaxGrid + 32;  // one flag set with its go words (16 words apart)
// The mean's phase 1 when a CTA spans whole rows: a ring of kStages shared-memory buffers of
// kStageBytes each, filled by bulk copies (dynamic shared memory of the one-pass mean kernels).
constexpr int kStages = 4;
constexpr int kStageBytes = 32768;
constexpr int kRingBytes = kStages * kStageBytes;

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

// sum over c in [c_lo, c_hi) of src[c * pitch], added in order of c; the loads are issued eight
// at a time (L2 hits, after the flags), so the chain is not one load latency per term. (Sixteen
// at a time made ptxas give the mean kernel fewer registers than its phase 1 needs.)
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
    unsigned long long* flags;  // [gridDim.x] phase 1 done, then go words at kGo1 and kGo2
    unsigned long long* flags2; // fused mean and subtraction only: [gridDim.x], fold done
    uint4* k_out;               // fused mean and subtraction only: [b, sk, hk, d] bf16
    float* mean;                // [b][cols]
    int* gate;                  // gate only: [b][hk]
    float* ratio;               // gate only, may be null
    int64_t b, sk, cols, c8, colgroups;
    int64_t stride;             // rows summed: 0, stride, 2*stride, ... (1: every row)
    int64_t n_rows;             // rows summed per (bi, column): sk, or the sample size
    int64_t rows_per_chunk;
    int nchunks;
    int lanes;                  // mean, whole rows per CTA: row lanes of the bulk-copy phase 1;
                                // 0: the register path (sum_chunks)
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

// Phase 1 of the mean when one CTA spans whole rows (colgroups = 1): each item's chunk of rows
// is one contiguous range of K, streamed through the shared-memory ring by bulk copies that
// thread 0 issues (kStages in flight, completion on one mbarrier per buffer), so the bytes in
// flight per SM do not depend on registers. Thread t owns group t % c8 at rows t0 + t / c8, + R,
// + 2R, ... of the chunk (R = lanes = kThreads / c8 row lanes; threads past R * c8 idle) and adds
// them in row order; the R lane sums of a group are then added in lane order through shared
// memory, so the split alone fixes the bits. `fills` counts the buffers filled so far (the
// barrier phases), the same in every thread. False, with the status word set, if a copy does not
// land within the time limit; the copies still in flight are then waited for (bounded) first.
__device__ __forceinline__ bool sum_chunks_bulk(const OnePass& a, float4 (&lred)[kThreads * 2],
                                                uint8_t* ring, uint64_t* full,
                                                volatile int* abort_flag)
{
    const int c8 = (int)a.c8, R = a.lanes;
    const int tid = (int)threadIdx.x;
    const int lane = tid / c8, g8 = tid - lane * c8;
    const int64_t row_bytes = a.c8 * 16;
    const int rps = (int)(kStageBytes / row_bytes);  // rows per buffer (row_bytes <= 8 KB)
    const WaitCtx w{abort_flag, a.status, a.timeout_ns};
    uint32_t fills = 0;
    for (int64_t it = blockIdx.x; it < a.n_items; it += gridDim.x) {
        const int chunk = (int)(it % a.nchunks);
        const int64_t bi = it / a.nchunks;
        const int64_t t0 = (int64_t)chunk * a.rows_per_chunk;
        int64_t t1 = t0 + a.rows_per_chunk;
        t1 = t1 < a.n_rows ? t1 : a.n_rows;
        const int nst = (int)((t1 - t0 + rps - 1) / rps);
        const char* src = reinterpret_cast<const char*>(a.k) + (bi * a.sk + t0) * row_bytes;
        auto issue = [&](int st) {  // thread 0: buffer st of this chunk
            const uint32_t slot = (fills + (uint32_t)st) % kStages;
            const int64_t r0 = (int64_t)st * rps;
            const int64_t n = (t1 - t0 - r0) < rps ? (t1 - t0 - r0) : rps;
            const uint32_t bar = smem_addr(full + slot);
            mbar_arrive_expect_tx(bar, (uint32_t)(n * row_bytes));
            bulk_load(smem_addr(ring + (size_t)slot * kStageBytes), src + r0 * row_bytes,
                      (uint32_t)(n * row_bytes), bar);
        };
        if (tid == 0)
            for (int st = 0; st < nst && st < kStages; ++st) issue(st);
        float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int st = 0; st < nst; ++st) {
            const uint32_t f = fills + (uint32_t)st;
            const uint32_t slot = f % kStages;
            const bool ok = mbar_wait(smem_addr(full + slot), (f / kStages) & 1u, w,
                                      B200ATTN_ERR_TIMEOUT);
            if (__syncthreads_or(!ok)) {
                if (tid == 0) {  // let the copies in flight land before leaving (bounded)
                    const int last = (st + kStages < nst ? st + kStages : nst);
                    for (int q = st; q < last; ++q) {
                        const uint32_t fq = fills + (uint32_t)q;
                        const uint64_t tq = global_timer_ns();
                        while (!mbar_try_wait(smem_addr(full + fq % kStages), (fq / kStages) & 1u) &&
                               global_timer_ns() - tq < 1000000000ull) {
                        }
                    }
                }
                __syncthreads();
                return false;
            }
            if (lane < R) {
                const int64_t r0 = (int64_t)st * rps;  // the buffer's first row, from t0
                const int64_t n64 = (t1 - t0 - r0) < rps ? (t1 - t0 - r0) : rps;
                const int n = (int)n64;
                int r = (int)((lane - r0 % R + R) % R);  // first row with (row - t0) % R == lane
                const uint4* rows = reinterpret_cast<const uint4*>(ring + (size_t)slot * kStageBytes);
                for (; r < n; r += R) acc_bf16x8(s, rows[r * c8 + g8]);
            }
            __syncthreads();  // every thread is done with the buffer
            if (tid == 0 && st + kStages < nst) issue(st + kStages);
        }
        fills += (uint32_t)nst;
        lred[2 * tid] = make_float4(s[0], s[1], s[2], s[3]);
        lred[2 * tid + 1] = make_float4(s[4], s[5], s[6], s[7]);
        __syncthreads();
        if (tid < c8) {
            float4 u = lred[2 * tid], v = lred[2 * tid + 1];
            for (int q = 1; q < R; ++q) {
                const float4 u2 = lred[2 * (q * c8 + tid)], v2 = lred[2 * (q * c8 + tid) + 1];
                u.x += u2.x; u.y += u2.y; u.z += u2.z; u.w += u2.w;
                v.x += v2.x; v.y += v2.y; v.z += v2.z; v.w += v2.w;
            }
            float4* dst = reinterpret_cast<float4*>(
                a.partial + (bi * a.nchunks + chunk) * a.cols + tid * 8);
            dst[0] = u;
            dst[1] = v;
        }
        __syncthreads();
    }
    return true;
}

// The mean's phase 1 by either path; false if it gave up (the status word is set).
__device__ __forceinline__ bool mean_phase1(const OnePass& a, float4 (&lred)[kThreads * 2],
                                            uint8_t* ring, uint64_t* full, int* abort_flag)
{
    if (a.lanes == 0) {
        sum_chunks<false>(a);
        return true;
    }
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int q = 0; q < kStages; ++q) mbar_init(smem_addr(full + q), 1);
        fence_barrier_init();
    }
    __syncthreads();
    return sum_chunks_bulk(a, lred, ring, full, abort_flag);
}

// mean[bi][col] = (sum of partial[bi][chunk][col] over the chunks) / sk. Fold items are blocks of
// 32 columns of one batch; warp w of the CTA sums the chunks of its fixed contiguous range
// [w*nchunks/16, (w+1)*nchunks/16) in order, then the 16 warp sums are added in warp order.
// Run by CTAs below n_fold(a), after the wait for every CTA's phase 1.
__device__ __forceinline__ int64_t n_fold(const OnePass& a) { return a.b * ((a.cols + 31) / 32); }

__device__ __forceinline__ void fold_mean(const OnePass& a, float (&red)[kFoldWarps][32])
{
    const int64_t nblk = (a.cols + 31) / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int c_lo = (int)((int64_t)w * a.nchunks / kFoldWarps);
    const int c_hi = (int)((int64_t)(w + 1) * a.nchunks / kFoldWarps);
    for (int64_t f = blockIdx.x; f < n_fold(a); f += gridDim.x) {
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

__global__ void __launch_bounds__(kThreads) k_mean_onepass(const OnePass a)
{
    __shared__ float red[kFoldWarps][32];
    __shared__ float4 lred[kThreads * 2];
    __shared__ uint64_t full[kStages];
    __shared__ int abort_flag;
    extern __shared__ __align__(128) uint8_t ring[];
    if (!mean_phase1(a, lred, ring, full, &abort_flag)) return;
    publish_cta(a.flags, a.tag);
    const int64_t nf = n_fold(a);
    if ((int64_t)blockIdx.x >= nf) return;
    const int waiters = (int)(nf < (int64_t)gridDim.x ? nf : (int64_t)gridDim.x);
    if (!wait_all_published(a.flags, a.tag, (int)gridDim.x, waiters, a.flags + kGo1, a.status,
                            a.timeout_ns))
        return;
    fold_mean(a, red);
}

// The gate (see k_smooth_gate). Phase 1 sums K and K^2 over the strided sample; phase 2 item =
// (bi, kv head). Its 2d partial columns (d channel sums, then d sums of squares) are read as d/2
// float4 columns: thread t takes float4 column t % (d/2) over the chunks of group t / (d/2)
// (1024/d groups, each a fixed contiguous range of chunks, added in chunk order, up to twelve
// 16-byte loads in flight: sixteen made ptxas spill); the group sums are added in group order,
// giving mu_c and e_c; then sum mu_c^2 and sum e_c over the d channels by a fixed tree (a
// butterfly in each warp of 32 channels, then the warp sums in order); ratio = first / second
// (0 for an all-zero K); gate = ratio >= threshold; mean = mu where the gate is on, else 0.
__global__ void __launch_bounds__(kThreads) k_gate_onepass(const OnePass a)
{
    __shared__ float4 gsum[kThreads];  // [group][float4 column]
    __shared__ float num[8], den[8];  // per warp of 32 channels
    sum_chunks<true>(a);
    publish_cta(a.flags, a.tag);
    const int64_t n_fold = a.b * a.hk;
    if ((int64_t)blockIdx.x >= n_fold) return;
    const int waiters = (int)(n_fold < (int64_t)gridDim.x ? n_fold : (int64_t)gridDim.x);
    if (!wait_all_published(a.flags, a.tag, (int)gridDim.x, waiters, a.flags + kGo1, a.status,
                            a.timeout_ns))
        return;
    const int d = (int)a.d;
    const int c4s = d / 2;  // float4 columns: d/4 of sums, then d/4 of squares
    const int groups = kThreads / c4s;
    const int c4 = threadIdx.x % c4s, grp = threadIdx.x / c4s;
    const int plane = c4 < d / 4 ? 0 : 1;
    const int ch = 4 * (c4 - plane * (d / 4));  // first of the column's four channels
    const int c_lo = (int)((int64_t)grp * a.nchunks / groups);
    const int c_hi = (int)((int64_t)(grp + 1) * a.nchunks / groups);
    const int64_t pitch = 2 * a.cols / 4;  // float4s from one chunk's row to the next's
    for (int64_t f = blockIdx.x; f < n_fold; f += gridDim.x) {
        const int64_t bi = f / a.hk, g = f - bi * a.hk;
        const float4* src = reinterpret_cast<const float4*>(
            a.partial + (bi * a.nchunks * 2 + plane) * a.cols + g * d + ch);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        int c = c_lo;
        for (; c < c_hi; c += 12) {
            float4 v[12];
#pragma unroll
            for (int e = 0; e < 12; ++e)
                if (c + e < c_hi) v[e] = __ldcg(src + (int64_t)(c + e) * pitch);
#pragma unroll
            for (int e = 0; e < 12; ++e)
                if (c + e < c_hi) {
                    acc.x += v[e].x;
                    acc.y += v[e].y;
                    acc.z += v[e].z;
                    acc.w += v[e].w;
                }
        }
        gsum[threadIdx.x] = acc;
        __syncthreads();
        if ((int)threadIdx.x < d) {
            const int cc = threadIdx.x;  // channel
            const float* gs = reinterpret_cast<const float*>(gsum);
            float s = 0.f, e = 0.f;  // a group's row: d channel sums, then d sums of squares
            for (int q = 0; q < groups; ++q) {
                s += gs[q * 2 * d + cc];
                e += gs[q * 2 * d + d + cc];
            }
            const float mu = __fdiv_rn(s, a.n_rows_f);
            float nu = mu * mu, de = __fdiv_rn(e, a.n_rows_f);
            // fixed tree: butterfly within each warp of 32 channels, then the d/32 warp sums
            // in warp order (only the first d threads take part: a barrier over exactly those
            // warps, d a multiple of 32, id 1)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                nu += __shfl_xor_sync(0xFFFFFFFFu, nu, o);
                de += __shfl_xor_sync(0xFFFFFFFFu, de, o);
            }
            if ((cc & 31) == 0) {
                num[cc >> 5] = nu;
                den[cc >> 5] = de;
            }
            asm volatile("bar.sync 1, %0;" ::"r"(d) : "memory");
            float tn = 0.f, td = 0.f;
            for (int w = 0; w < d / 32; ++w) {
                tn += num[w];
                td += den[w];
            }
            const float r = td > 0.f ? __fdiv_rn(tn, td) : 0.f;
            const bool on = r >= a.threshold;
            a.mean[f * d + cc] = on ? mu : 0.f;
            if (cc == 0) {
                a.gate[f] = on ? 1 : 0;
                if (a.ratio) a.ratio[f] = r;
            }
        }
        __syncthreads();
    }
}

// 8 channels of K - mean (16 bytes of bf16, each an fp32 subtraction rounded to bf16).
__device__ __forceinline__ uint4 sub8(const uint4& x, const float (&mv)[8])
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float lo = __fsub_rn(__uint_as_float(w[q] << 16), mv[2 * q]);
        const float hi = __fsub_rn(__uint_as_float(w[q] & 0xFFFF0000u), mv[2 * q + 1]);
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        o[q] = *reinterpret_cast<uint32_t*>(&v);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// The mean is read through the read-only path (NC) when no CTA of the launch writes it, else
// through L2; so is K (the fused kernel reads K through L2, where phase 1 left it).
template <bool NC, class T>
__device__ __forceinline__ T load(const T* p) { return NC ? __ldg(p) : __ldcg(p); }

template <bool NC>
__device__ __forceinline__ void load_mean8(float (&mv)[8], const float* m)
{
    const float4 m0 = load<NC>(reinterpret_cast<const float4*>(m));
    const float4 m1 = load<NC>(reinterpret_cast<const float4*>(m) + 1);
    mv[0] = m0.x; mv[1] = m0.y; mv[2] = m0.z; mv[3] = m0.w;
    mv[4] = m1.x; mv[5] = m1.y; mv[6] = m1.z; mv[7] = m1.w;
}

// k_out = bf16_rne(float(K) - mean[bi, col]) over the [b*sk rows, c8 groups of 8 channels] view
// of K, by nthreads threads (this one is tid). With nthreads >= c8, thread tid < R*c8 (R =
// nthreads / c8) owns channel group tid % c8 at rows tid / c8, + R, + 2R, ...; otherwise it owns
// groups tid, tid + nthreads, ... at every row. Each thread keeps its group's 8 mean values and
// moves to the next batch's when its row crosses into it, so no index is divided per group. G
// groups in flight per thread.
template <int G, bool NC>
__device__ __forceinline__ void sub_all(const uint4* k, const float* mean, uint4* k_out,
                                        int64_t tid, int64_t nthreads, int64_t b, int64_t sk,
                                        int64_t c8)
{
    const int64_t rows = b * sk, cols = c8 * 8;
    const bool by_rows = nthreads >= c8;
    const int64_t R = by_rows ? nthreads / c8 : 1;
    if (by_rows && tid >= R * c8) return;
    for (int64_t g8 = by_rows ? tid % c8 : tid; g8 < c8; g8 += by_rows ? c8 : nthreads) {
        const int64_t r0 = by_rows ? tid / c8 : 0;
        if (r0 >= rows) return;
        int64_t bi = r0 / sk, b_end = (bi + 1) * sk;
        float mv[8];
        load_mean8<NC>(mv, mean + bi * cols + g8 * 8);
        for (int64_t r = r0; r < rows; r += G * R) {
            uint4 x[G];
#pragma unroll
            for (int e = 0; e < G; ++e)
                if (r + e * R < rows) x[e] = load<NC>(k + (r + e * R) * c8 + g8);
#pragma unroll
            for (int e = 0; e < G; ++e) {
                const int64_t re = r + e * R;
                if (re < rows) {
                    if (re >= b_end) {  // first row of a later batch
                        bi = re / sk;
                        b_end = (bi + 1) * sk;
                        load_mean8<NC>(mv, mean + bi * cols + g8 * 8);
                    }
                    k_out[re * c8 + g8] = sub8(x[e], mv);
                }
            }
        }
    }
}

__global__ void __launch_bounds__(kSubThreads)
    k_sub_kernel(const uint4* __restrict__ k, const float* __restrict__ mean,
                 uint4* __restrict__ k_out, int64_t b, int64_t sk, int64_t c8)
{
    sub_all<8, true>(k, mean, k_out, (int64_t)blockIdx.x * kSubThreads + threadIdx.x,
                     (int64_t)gridDim.x * kSubThreads, b, sk, c8);
}

// The mean (phases 1 and 2 exactly as k_mean_onepass, so the same split gives the same bits),
// then k_out = K - mean over the whole tensor once every fold CTA has published its columns.
__global__ void __launch_bounds__(kThreads) k_mean_sub_onepass(const OnePass a)
{
    __shared__ float red[kFoldWarps][32];
    __shared__ float4 lred[kThreads * 2];
    __shared__ uint64_t full[kStages];
    __shared__ int abort_flag;
    extern __shared__ __align__(128) uint8_t ring[];
    if (!mean_phase1(a, lred, ring, full, &abort_flag)) return;
    publish_cta(a.flags, a.tag);
    const int64_t nf = n_fold(a);
    const int fold_ctas = (int)(nf < (int64_t)gridDim.x ? nf : (int64_t)gridDim.x);
    if ((int)blockIdx.x < fold_ctas) {
        if (!wait_all_published(a.flags, a.tag, (int)gridDim.x, fold_ctas, a.flags + kGo1,
                                a.status, a.timeout_ns))
            return;
        fold_mean(a, red);
        publish_cta(a.flags2, a.tag);
    }
    if (!wait_all_published(a.flags2, a.tag, fold_ctas, (int)gridDim.x, a.flags + kGo2, a.status,
                            a.timeout_ns))
        return;
    sub_all<8, false>(a.k, a.mean, a.k_out, (int64_t)blockIdx.x * kThreads + threadIdx.x,
                      (int64_t)gridDim.x * kThreads, a.b, a.sk, a.c8);
}

// Column-partitioned K mean (and, with SUB, K - mean), used when K has many (batch, 8-channel
// group) pairs: CTA c owns the G consecutive pairs p = bi * c8 + g8 in [c*G, c*G + G) and sums
// them over ALL sk rows itself, so no cross-CTA fold, scratch or grid-wide wait is needed.
// Thread t takes pair slot t % G at rows t / G, + L, + 2L, ... (L = 512 / G row lanes, G a power
// of two; sixteen 16-byte loads in flight, added in row order); the L lane sums of each pair are
// then added by a fixed tree in shared memory, so the mean is bit-identical from run to run. With
// SUB every thread then rewrites its rows as K - mean, re-reading them through L2.
template <bool SUB>
__global__ void __launch_bounds__(kThreads, 1)
    k_mean_cols(const uint4* __restrict__ k, float* __restrict__ mean, uint4* __restrict__ k_out,
                int64_t b, int64_t sk, int64_t c8, int G)
{
    __shared__ float4 red[kThreads * 2];  // [thread][2]: its 8 channel sums, then the tree's
    const int gs = threadIdx.x % G, ln = threadIdx.x / G, L = kThreads / G;
    const int64_t pair = (int64_t)blockIdx.x * G + gs;
    const bool active = pair < b * c8;
    const int64_t bi = active ? pair / c8 : 0, g8 = active ? pair - bi * c8 : 0;
    const uint4* src = k + (bi * sk) * c8 + g8;
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (active) {
        int64_t r = ln;
        for (; r + 15 * L < sk; r += 16 * L) {
            uint4 x[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = __ldg(src + (r + e * L) * c8);
#pragma unroll
            for (int e = 0; e < 16; ++e) acc_bf16x8(s, x[e]);
        }
        for (; r < sk; r += L) acc_bf16x8(s, __ldg(src + r * c8));
    }
    red[2 * threadIdx.x] = make_float4(s[0], s[1], s[2], s[3]);
    red[2 * threadIdx.x + 1] = make_float4(s[4], s[5], s[6], s[7]);
    __syncthreads();
    for (int w = L / 2; w > 0; w >>= 1) {  // lane ln += lane ln + w, same slot
        if (ln < w) {
            const int o = threadIdx.x + w * G;
            float4 a = red[2 * threadIdx.x], c = red[2 * threadIdx.x + 1];
            const float4 a2 = red[2 * o], c2 = red[2 * o + 1];
            a.x += a2.x; a.y += a2.y; a.z += a2.z; a.w += a2.w;
            c.x += c2.x; c.y += c2.y; c.z += c2.z; c.w += c2.w;
            red[2 * threadIdx.x] = a;
            red[2 * threadIdx.x + 1] = c;
        }
        __syncthreads();
    }
    const float4 t0 = red[2 * gs], t1 = red[2 * gs + 1];  // lane 0's sums of this slot
    const float n = (float)sk;
    float mv[8] = {__fdiv_rn(t0.x, n), __fdiv_rn(t0.y, n), __fdiv_rn(t0.z, n), __fdiv_rn(t0.w, n),
                   __fdiv_rn(t1.x, n), __fdiv_rn(t1.y, n), __fdiv_rn(t1.z, n), __fdiv_rn(t1.w, n)};
    if (active && ln == 0) {
        float4* m4 = reinterpret_cast<float4*>(mean + pair * 8);  // [b][cols] = pair-major
        m4[0] = make_float4(mv[0], mv[1], mv[2], mv[3]);
        m4[1] = make_float4(mv[4], mv[5], mv[6], mv[7]);
    }
    if constexpr (SUB) {
        if (!active) return;
        uint4* dst = k_out + (bi * sk) * c8 + g8;
        int64_t r = ln;
        for (; r + 7 * L < sk; r += 8 * L) {
            uint4 x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = __ldcg(src + (r + e * L) * c8);
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[(r + e * L) * c8] = sub8(x[e], mv);
        }
        for (; r < sk; r += L) dst[r * c8] = sub8(__ldcg(src + r * c8), mv);
    }
}

// ---- K mean of a strided view (k_smooth_mean_strided): 2-byte loads, any alignment ----
// Element (bi, s, g, c) of the view is k[bi*sb + s*ss + g*sh + c]. Phase A: CTA (chunk, bi,
// channel block) sums rows [chunk*rpc, +rpc) of kStrChannels channels, thread t owning channels
// cb*kStrChannels + t + kStrThreads*q (q < kStrPerThread); a warp's loads of one row are 32
// consecutive channels of one head (64 contiguous bytes), eight rows in flight per channel, added
// in row order. Phase B: CTA (bi, 32 channels); warp w adds the chunks of its fixed contiguous
// range in chunk order for its lane's channel, then the warp sums are added in warp order.
constexpr int kStrThreads = 256;
constexpr int kStrPerThread = 4;
constexpr int kStrChannels = kStrThreads * kStrPerThread;

__device__ __forceinline__ float bf16_at(const uint16_t* k, int64_t off)
{
    return __uint_as_float((uint32_t)__ldg(k + off) << 16);
}

__global__ void __launch_bounds__(kStrThreads)
    k_mean_strided_partial(const uint16_t* __restrict__ k, float* __restrict__ partial,
                           int64_t sk, int64_t d, int64_t cols, int64_t sb, int64_t ss,
                           int64_t sh, int64_t rpc, int nchunks)
{
    const int chunk = blockIdx.x;
    const int64_t bi = blockIdx.y;
    const int64_t t0 = (int64_t)chunk * rpc;
    const int64_t t1 = t0 + rpc < sk ? t0 + rpc : sk;
    int64_t off[kStrPerThread];
    bool on[kStrPerThread];
#pragma unroll
    for (int q = 0; q < kStrPerThread; ++q) {
        const int64_t c = (int64_t)blockIdx.z * kStrChannels + threadIdx.x + q * kStrThreads;
        on[q] = c < cols;
        const int64_t g = on[q] ? c / d : 0;
        off[q] = bi * sb + g * sh + (on[q] ? c - g * d : 0);
    }
    float acc[kStrPerThread] = {0.f, 0.f, 0.f, 0.f};
    int64_t t = t0;
    for (; t + 8 <= t1; t += 8) {
        float x[kStrPerThread][8];
#pragma unroll
        for (int q = 0; q < kStrPerThread; ++q)
#pragma unroll
            for (int e = 0; e < 8; ++e) x[q][e] = on[q] ? bf16_at(k, off[q] + (t + e) * ss) : 0.f;
#pragma unroll
        for (int q = 0; q < kStrPerThread; ++q)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[q] += x[q][e];
    }
    for (; t < t1; ++t)
#pragma unroll
        for (int q = 0; q < kStrPerThread; ++q)
            if (on[q]) acc[q] += bf16_at(k, off[q] + t * ss);
#pragma unroll
    for (int q = 0; q < kStrPerThread; ++q) {
        const int64_t c = (int64_t)blockIdx.z * kStrChannels + threadIdx.x + q * kStrThreads;
        if (on[q]) partial[(bi * nchunks + chunk) * cols + c] = acc[q];
    }
}

__global__ void __launch_bounds__(kStrThreads)
    k_mean_strided_fold(const float* __restrict__ partial, float* __restrict__ mean, int64_t cols,
                        int nchunks, float n_rows)
{
    constexpr int W = kStrThreads / 32;
    __shared__ float red[W][32];
    const int64_t nblk = (cols + 31) / 32;
    const int64_t bi = blockIdx.x / nblk;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t c = (blockIdx.x - bi * nblk) * 32 + lane;
    const int c_lo = (int)((int64_t)w * nchunks / W), c_hi = (int)((int64_t)(w + 1) * nchunks / W);
    float sum = 0.f;
    if (c < cols) {
        const float* src = partial + bi * nchunks * cols + c;
        int q = c_lo;
        for (; q + 8 <= c_hi; q += 8) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = src[(int64_t)(q + e) * cols];
#pragma unroll
            for (int e = 0; e < 8; ++e) sum += v[e];
        }
        for (; q < c_hi; ++q) sum += src[(int64_t)q * cols];
    }
    red[w][lane] = sum;
    __syncthreads();
    if (w == 0 && c < cols) {
        float tsum = 0.f;
#pragma unroll
        for (int q = 0; q < W; ++q) tsum += red[q][lane];
        mean[bi * cols + c] = __fdiv_rn(tsum, n_rows);
    }
}

// The column-partitioned split: G = the least power of two whose ceil(pairs / G) CTAs fit on
// the SMs; taken when that grid keeps at least half of the SMs busy and G >= kColsMinG (each
// CTA then reads G * 16 contiguous bytes of every row); else 0: the one-pass row-chunk kernel.
constexpr int kColsMinG = 2;
int cols_group(int64_t pairs, int n_sm)
{
    if (n_sm <= 0) return 0;
    int G = 1;
    while (G < kThreads && (pairs + G - 1) / G > n_sm) G <<= 1;
    const int64_t grid = (pairs + G - 1) / G;
    return (grid <= n_sm && 2 * grid >= n_sm && G >= kColsMinG) ? G : 0;
}

int launch_cols(const void* k, float* mean, void* k_out, int64_t b, int64_t sk, int64_t cols,
                int G, cudaStream_t st)
{
    const int64_t pairs = b * (cols / 8);
    const unsigned grid = (unsigned)((pairs + G - 1) / G);
    if (k_out)
        k_mean_cols<true><<<grid, kThreads, 0, st>>>(static_cast<const uint4*>(k), mean,
                                                      static_cast<uint4*>(k_out), b, sk,
                                                      cols / 8, G);
    else
        k_mean_cols<false><<<grid, kThreads, 0, st>>>(static_cast<const uint4*>(k), mean, nullptr,
                                                       b, sk, cols / 8, G);
    return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}

// Fixed scratch for k_smooth_mean_noalloc: file-scope device memory that every GPU loading this
// library holds until the process exits: 2^20 floats of partial sums (4 MiB), then one set of
// flag words (1024 + 32 64-bit words: one per CTA of the one-pass kernel, then the go words).
constexpr int64_t kNoAllocScratchFloats = (int64_t)1 << 20;
__device__ __align__(256) float g_kmean_scratch[kNoAllocScratchFloats + 2 * kFlagWords];

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
int onepass_grid(K kernel, std::atomic<int> (&cache)[64], int dyn_smem = 0)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 0;
    }
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        int per_sm = 0, sms = 0;
        if ((dyn_smem > 0 &&
             cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  dyn_smem) != cudaSuccess) ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, dyn_smem) !=
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

unsigned long long next_tag() { return next_call_tag(kTagKind); }

// Work split of the one-pass kernels: the rows of every (bi, column group of 4096 channels) cut
// into chunks, so that the grid's CTAs get about one item each; at least 16 rows per chunk (per
// row lane), at most max_chunks chunks (the scratch), at most 1024. With lanes_ok (the mean) and
// rows of at most 4096 channels (one column group), a chunk is one contiguous range of K: the
// bulk-copy phase 1 streams it, spread over kThreads / c8 row lanes. (The gate keeps the register
// path and one lane: its 2048-row sample is latency-bound, and row lanes made the gate of the
// b1 hk5 d128 65536-key workload slower, 17.7 vs 13.7 us, as fewer SMs then had loads in flight.)
struct Split {
    int64_t colgroups, rows_per_chunk, n_items;
    int nchunks, grid, lanes;
};

Split make_split(int64_t b, int64_t cols, int64_t n_rows, int64_t max_chunks, int grid_max,
                 bool lanes_ok)
{
    Split s;
    s.colgroups = (cols + kColsPerCta - 1) / kColsPerCta;
    const int64_t c8 = cols / 8;
    s.lanes = (lanes_ok && s.colgroups == 1) ? (int)(kThreads / c8) : 0;
    int64_t nch = (grid_max + b * s.colgroups - 1) / (b * s.colgroups);
    const int64_t per = 16 * (int64_t)(s.lanes > 0 ? s.lanes : 1);
    const int64_t by_rows = (n_rows + per - 1) / per;
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

int launch_onepass(void (*kernel)(const OnePass), OnePass& a, int grid, cudaStream_t st,
                   int dyn_smem = 0)
{
    void* args[] = {&a};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel), dim3((unsigned)grid),
                                    dim3(kThreads), args, (size_t)dyn_smem, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return B200ATTN_OK;
}

// The mean through the one-pass kernel with split sp, partials (room for sp.nchunks chunks) and
// flags (kFlagWords words) at the given device addresses; with k_out, the fused kernel, which
// also writes K - mean and takes a second set of kFlagWords words after the first.
int run_mean(const void* k, float* mean, void* k_out, int64_t b, int64_t sk, int64_t cols,
             const Split& sp, float* partial, unsigned long long* flags, int* status,
             cudaStream_t st)
{
    OnePass a{};
    a.k = static_cast<const uint4*>(k);
    a.partial = partial;
    a.flags = flags;
    a.flags2 = k_out ? flags + kFlagWords : nullptr;
    a.k_out = static_cast<uint4*>(k_out);
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
    a.lanes = sp.lanes;
    a.n_items = sp.n_items;
    a.n_rows_f = (float)sk;
    a.tag = next_tag();
    a.status = status;
    a.timeout_ns = 4000000000ull;
    return launch_onepass(k_out ? k_mean_sub_onepass : k_mean_onepass, a, sp.grid, st,
                          kRingBytes);
}

// k_smooth_mean and k_smooth_mean_sub: scratch (the split's partials, then two flag arrays) from
// the library pool on `st`, returned to it after the launch.
int mean_pooled(const void* k, float* mean, void* k_out, int64_t b, int64_t sk, int64_t cols,
                int grid_max, cudaStream_t st)
{
    int* status = status_word();
    if (!status || grid_max <= 0) return B200ATTN_ERR_CUDA;
    const Split sp = make_split(b, cols, sk, 1024, grid_max, true);
    const size_t part_bytes = (size_t)(b * sp.nchunks * cols) * sizeof(float);
    const size_t nbytes = part_bytes + 2 * kFlagWords * sizeof(unsigned long long);
    char* scratch = nullptr;
    cudaMemPool_t pool = scratch_pool();
    if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void**>(&scratch), nbytes, pool, st) !=
                     cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    const int rc =
        run_mean(k, mean, k_out, b, sk, cols, sp, reinterpret_cast<float*>(scratch),
                 reinterpret_cast<unsigned long long*>(scratch + part_bytes), status, st);
    if (cudaFreeAsync(scratch, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return rc;
}

std::atomic<int> g_mean_sub_grid[64];

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
    const int grid = onepass_grid(k_mean_onepass, g_mean_grid, kRingBytes);
    const int G = cols_group(b * (cols / 8), grid);
    if (G > 0)
        return launch_cols(k, mean, nullptr, b, sk, cols, G, static_cast<cudaStream_t>(stream));
    return mean_pooled(k, mean, nullptr, b, sk, cols, grid, static_cast<cudaStream_t>(stream));
}

extern "C" int k_smooth_mean_sub(const void* k, float* mean, void* k_out, int64_t b, int64_t hk,
                                 int64_t sk, int64_t d, void* stream)
{
    int64_t cols = 0;
    int rc = check_kmean_args(k, mean, b, hk, sk, d, &cols);
    if (rc != B200ATTN_OK || b == 0 || hk == 0) return rc;
    if (!k_out) return B200ATTN_ERR_NULL;
    if (!aligned(k_out, 16)) return B200ATTN_ERR_ALIGN;
    rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    // The mean's split must be the one k_smooth_mean takes (same bits): both grids are the SM
    // count whenever one CTA of each kernel fits on an SM, which the occupancy query confirms.
    const int grid = onepass_grid(k_mean_onepass, g_mean_grid, kRingBytes);
    const int G = cols_group(b * (cols / 8), grid);  // the same choice as k_smooth_mean's
    if (G > 0)
        return launch_cols(k, mean, k_out, b, sk, cols, G, static_cast<cudaStream_t>(stream));
    const int grid2 = onepass_grid(k_mean_sub_onepass, g_mean_sub_grid, kRingBytes);
    if (grid2 != grid) return B200ATTN_ERR_CUDA;
    return mean_pooled(k, mean, k_out, b, sk, cols, grid, static_cast<cudaStream_t>(stream));
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
    const int grid_max = onepass_grid(k_mean_onepass, g_mean_grid, kRingBytes);
    const int G = cols_group(b * (cols / 8), grid_max);  // no scratch at all on this path
    if (G > 0)
        return launch_cols(k, mean, nullptr, b, sk, cols, G, static_cast<cudaStream_t>(stream));
    float* scratch = noalloc_scratch();
    int* status = status_word();
    if (!scratch || !status || grid_max <= 0) return B200ATTN_ERR_CUDA;
    // The partials of as many chunks as fit in the fixed scratch; the flags after them. Every
    // partial the fold reads is written earlier in the same launch, and a flag counts only when
    // it carries this call's tag, so nothing needs clearing between calls.
    const Split sp =
        make_split(b, cols, sk, kNoAllocScratchFloats / (b * cols), grid_max, true);
    return run_mean(k, mean, nullptr, b, sk, cols, sp, scratch,
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
    const Split sp = make_split(b, cols, n_samp, 1024, grid_max, false);
    const size_t part_bytes = (size_t)(b * sp.nchunks * 2 * cols) * sizeof(float);
    const size_t nbytes = part_bytes + kFlagWords * sizeof(unsigned long long);
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
    a.lanes = 1;
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
    int64_t blocks = (n + 8 * kSubThreads - 1) / (8 * kSubThreads);
    if (blocks > 148 * 8) blocks = 148 * 8;
    k_sub_kernel<<<(unsigned)blocks, kSubThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k), mean, static_cast<uint4*>(k_out), b, sk, cols / 8);
    return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}

extern "C" int k_smooth_mean_strided(const void* k, float* mean, int64_t b, int64_t hk, int64_t sk,
                                     int64_t d, int64_t stride_b, int64_t stride_s,
                                     int64_t stride_h, void* stream)
{
    if (b < 0 || hk < 0 || sk <= 0 || stride_b < 0 || stride_s < 0 || stride_h < 0)
        return B200ATTN_ERR_SHAPE;
    if (!(d == 64 || d == 128 || d == 256)) return B200ATTN_ERR_HEADDIM;
    int64_t cols, n, last = 0, t;
    if (!numel({hk, d}, &cols) || !numel({b, cols}, &n) || b >= 65536 || sk >= ((int64_t)1 << 40) ||
        (cols + kStrChannels - 1) / kStrChannels >= 65536 || n >= ((int64_t)1 << 36))
        return B200ATTN_ERR_RANGE;
    // the largest element offset the view reaches must fit in int64
    if (b > 0 && hk > 0) {
        if (!mul_ok(b - 1, stride_b, &t) || (last += t) < 0 || !mul_ok(sk - 1, stride_s, &t) ||
            (last += t) < 0 || !mul_ok(hk - 1, stride_h, &t) || (last += t) < 0 ||
            (last += d) < 0 || last > INT64_MAX / 2)
            return B200ATTN_ERR_RANGE;
    }
    if (b == 0 || hk == 0) return B200ATTN_OK;
    if (!k || !mean) return B200ATTN_ERR_NULL;
    if (!aligned(k, 2) || !aligned(mean, 4)) return B200ATTN_ERR_ALIGN;
    // The contiguous layout at 16-byte alignment is k_smooth_mean itself (same kernels, same bits).
    if (stride_h == d && stride_s == cols && stride_b == sk * cols && aligned(k, 16) &&
        aligned(mean, 16))
        return k_smooth_mean(k, mean, b, hk, sk, d, stream);
    int rc = check_arch();
    if (rc != B200ATTN_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t cblocks = (cols + kStrChannels - 1) / kStrChannels;
    // about two CTAs per SM, at least 16 rows per chunk, at most 1024 chunks
    int64_t nch = (2 * 148 + b * cblocks - 1) / (b * cblocks);
    const int64_t by_rows = (sk + 15) / 16;
    if (nch > by_rows) nch = by_rows;
    if (nch > 1024) nch = 1024;
    if (nch < 1) nch = 1;
    const int64_t rpc = (sk + nch - 1) / nch;
    const int nchunks = (int)((sk + rpc - 1) / rpc);
    float* partial = nullptr;
    cudaMemPool_t pool = scratch_pool();
    const size_t nbytes = (size_t)(n * nchunks) * sizeof(float);
    if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void**>(&partial), nbytes, pool, st) !=
                     cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    k_mean_strided_partial<<<dim3((unsigned)nchunks, (unsigned)b, (unsigned)cblocks), kStrThreads,
                             0, st>>>(static_cast<const uint16_t*>(k), partial, sk, d, cols,
                                      stride_b, stride_s, stride_h, rpc, nchunks);
    k_mean_strided_fold<<<(unsigned)(b * ((cols + 31) / 32)), kStrThreads, 0, st>>>(
        partial, mean, cols, nchunks, (float)sk);
    rc = cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
    if (cudaFreeAsync(partial, st) != cudaSuccess) {
        cudaGetLastError();
        return B200ATTN_ERR_CUDA;
    }
    return rc;
}
