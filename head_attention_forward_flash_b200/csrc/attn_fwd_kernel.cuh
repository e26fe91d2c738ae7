// attn_fwd_kernel.cuh -- fused attention forward pass for sm_100a (B200).
//
// Computes O = softmax(scale * Q K^T [+ causal mask]) V and LSE = log sum exp(scale * Q K^T)
// per query row, for bf16 BSHD tensors with grouped-query heads, as the Triton "_attn_fwd"
// MHA forward of "Tune MHA config & small-head pipeline pathology" does (Motivation; shapes in
// "Source of shapes"): one CTA owns a 128-row query tile of one (batch, query head).
//
// Work split inside a CTA (192 threads):
//   warps 0-3  softmax: thread t owns query row t (= TMEM lane t). Writes its Q row into TMEM,
//              turns each S block into P (online softmax, exp2 with the scale folded into one
//              FMA, lazy rescaling of O), and finally normalises O and writes O and LSE.
//   warp 4     MMA issuer (one thread): S = Q K^T and O += P V on the tensor core, operands
//              A from TMEM (Q, then P), B from shared memory (K, V), accumulators in TMEM.
//   warp 5     TMA producer (one thread): streams K and V tiles through a ring of shared-memory
//              slots in the order the MMA warp consumes them: K0, K1, V0, K2, V1, ...
//
// Tensor memory columns (128 lanes x 32-bit): S0 | S1 (two BN-wide score buffers, so the next
// block's QK^T overlaps this block's softmax; P (bf16 pairs) overwrites the first BN/2 columns
// of its own S buffer) | O (DV columns, fp32) | Q (DQK/2 columns of bf16 pairs).
//
// Every mbarrier wait is bounded in time; a wait that gives up sets the device error word and a
// CTA-wide abort flag, every role then leaves its loop, in-flight TMA loads and MMAs are drained
// (again with a time bound), and tensor memory is freed before the CTA exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace b200 {

constexpr int kErrTimeout = 10;  // B200ATTN_ERR_TIMEOUT

struct AttnParams {
    const __nv_bfloat16* q;
    __nv_bfloat16* o;
    float* lse;  // may be null
    int64_t b, hq, hk, sq, sk;
    int64_t group;     // hq / hk
    float scale_log2;  // scale * log2(e)
    int n_qtiles;
    int* status;  // device error word
    unsigned long long timeout_ns;
};

template <int DQK_, int DV_, int BN_, int NSLOT_>
struct AttnTraits {
    static constexpr int DQK = DQK_;
    static constexpr int DV = DV_;
    static constexpr int BN = BN_;  // keys per block
    static constexpr int BM = 128;  // query rows per tile
    static constexpr int NSLOT = NSLOT_;
    static constexpr int QCH = DQK / 64;  // 128-byte (64-element) column chunks of a K row
    static constexpr int VCH = DV / 64;
    static constexpr uint32_t CHUNK_BYTES = BN * 128;  // one 64-column TMA box of a K or V tile
    static constexpr uint32_t K_TILE_BYTES = BN * DQK * 2;
    static constexpr uint32_t V_TILE_BYTES = BN * DV * 2;
    static constexpr uint32_t SLOT_BYTES = K_TILE_BYTES > V_TILE_BYTES ? K_TILE_BYTES
                                                                        : V_TILE_BYTES;
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t O_COL = 2 * BN;
    static constexpr uint32_t Q_COL = 2 * BN + DV;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(2 * BN + DV + DQK / 2 <= 512, "tensor memory budget");
    static_assert(DQK % 64 == 0 && DV % 64 == 0 && BN % 64 == 0 && BN <= 256 && DV <= 256, "");
    static constexpr uint32_t SLOTS_BYTES = NSLOT * SLOT_BYTES;
    static constexpr int NBAR = 2 * NSLOT + 7;
    static constexpr uint32_t SMEM_BYTES = 1024 + SLOTS_BYTES + NBAR * 8 + 16;
    static constexpr int NUM_THREADS = 192;
    static constexpr uint32_t IDESC_QK = make_idesc_bf16(128, BN, false, false);
    static constexpr uint32_t IDESC_PV = make_idesc_bf16(128, DV, false, true);
};

// Wait bounded only by time (used to drain in-flight copies / MMAs before exit, also after an
// abort, so it ignores the abort flag).
__device__ __noinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity,
                                             unsigned long long timeout_ns, int* status)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > timeout_ns) {
            atomicCAS(status, 0, kErrTimeout);
            return;
        }
    }
}

template <class T, bool CAUSAL>
__global__ void __launch_bounds__(T::NUM_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const AttnParams p)
{
    constexpr int BN = T::BN;
    constexpr int NSLOT = T::NSLOT;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);  // SW128 needs 1 KB
    const uint32_t slots = smem_addr(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::SLOTS_BYTES);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + T::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    auto bar_full = [&](int s) { return smem_addr(&bars[s]); };
    auto bar_empty = [&](int s) { return smem_addr(&bars[NSLOT + s]); };
    auto bar_s_full = [&](int s) { return smem_addr(&bars[2 * NSLOT + s]); };
    auto bar_p_full = [&](int s) { return smem_addr(&bars[2 * NSLOT + 2 + s]); };
    const uint32_t bar_pv_done = smem_addr(&bars[2 * NSLOT + 4]);
    const uint32_t bar_q_ready = smem_addr(&bars[2 * NSLOT + 5]);
    const uint32_t bar_mma_done = smem_addr(&bars[2 * NSLOT + 6]);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work unit: (batch, query head) from blockIdx.x; query tile from blockIdx.y, with the
    // tiles that see the most keys (causal) scheduled first.
    const int64_t bh = blockIdx.x;
    const int64_t bi = bh / p.hq;
    const int64_t h = bh - bi * p.hq;
    const int64_t g = h / p.group;
    const int64_t q0 = (int64_t)(p.n_qtiles - 1 - (int)blockIdx.y) * T::BM;
    const int64_t n_kv = (p.sk + BN - 1) / BN;
    int n_blocks, mask_from;
    if (CAUSAL) {
        const int64_t last_row = (q0 + T::BM - 1 < p.sq - 1) ? q0 + T::BM - 1 : p.sq - 1;
        const int64_t last_key = last_row + p.sk - p.sq;
        int64_t nb = last_key < 0 ? 0 : last_key / BN + 1;
        nb = nb < n_kv ? nb : n_kv;
        const int64_t first_lim = q0 + p.sk - p.sq + 1;  // keys < first_lim: allowed for all rows
        int64_t full = first_lim <= 0 ? 0 : first_lim / BN;
        full = full < p.sk / BN ? full : p.sk / BN;
        n_blocks = (int)nb;
        mask_from = (int)(full < nb ? full : nb);
    } else {
        n_blocks = (int)n_kv;
        mask_from = (int)(p.sk / BN);
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_s_full(s), 1);
            mbar_init(bar_p_full(s), 128);
        }
        mbar_init(bar_pv_done, 1);
        mbar_init(bar_q_ready, 128);
        mbar_init(bar_mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4) {
        tmem_alloc(smem_addr(tmem_holder), T::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 5 && lane == 0) {
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    const WaitCtx wc{abort_flag, p.status, p.timeout_ns};

    if (warp == 5) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0 && n_blocks > 0) {
            int it = 0;
            bool ok = true;
            auto load = [&](bool is_k, int j) {
                const int slot = it % NSLOT;
                const uint32_t phase = (uint32_t)(it / NSLOT) & 1u;
                if (!mbar_wait(bar_empty(slot), phase ^ 1u, wc, kErrTimeout)) {
                    ok = false;
                    return;
                }
                const uint32_t dst = slots + slot * T::SLOT_BYTES;
                mbar_arrive_expect_tx(bar_full(slot), is_k ? T::K_TILE_BYTES : T::V_TILE_BYTES);
                const int nch = is_k ? T::QCH : T::VCH;
                for (int ch = 0; ch < nch; ++ch)
                    tma_load_4d(dst + ch * T::CHUNK_BYTES, is_k ? (const void*)&tmap_k
                                                                : (const void*)&tmap_v,
                                bar_full(slot), ch * 64, (int)g, j * BN, (int)bi);
                ++it;
            };
            for (int j = 0; j < n_blocks && ok; ++j) {
                load(true, j);
                if (ok && j >= 1) load(false, j - 1);
            }
            if (ok) load(false, n_blocks - 1);
            // Nothing may be in flight when the CTA exits: wait for the last load of each slot.
            const int n_drain = it < NSLOT ? it : NSLOT;
            for (int d = 0; d < n_drain; ++d) {
                const int idx = it - 1 - d;
                mbar_wait_drain(bar_full(idx % NSLOT), (uint32_t)(idx / NSLOT) & 1u, p.timeout_ns,
                                p.status);
            }
        }
    } else if (warp == 4) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0 && n_blocks > 0) {
            bool ok = mbar_wait(bar_q_ready, 0, wc, kErrTimeout);
            tc_fence_after_sync();
            int it = 0;
            auto take = [&](uint32_t& addr, int& slot) -> bool {
                slot = it % NSLOT;
                const uint32_t phase = (uint32_t)(it / NSLOT) & 1u;
                ++it;
                if (!mbar_wait(bar_full(slot), phase, wc, kErrTimeout)) return false;
                addr = slots + slot * T::SLOT_BYTES;
                return true;
            };
            auto qk = [&](int j) {
                uint32_t kaddr;
                int slot;
                if (!take(kaddr, slot)) {
                    ok = false;
                    return;
                }
                const uint32_t d_tmem = tmem + T::S_COL + (uint32_t)(j & 1) * BN;
#pragma unroll
                for (int kk = 0; kk < T::DQK / 16; ++kk) {
                    const uint64_t bdesc = make_sdesc_sw128(
                        kaddr + (kk >> 2) * T::CHUNK_BYTES + (kk & 3) * 32, 16, 1024);
                    mma_ts(d_tmem, tmem + T::Q_COL + kk * 8, bdesc, T::IDESC_QK, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar_s_full(j & 1));
                tc_commit(bar_empty(slot));
            };
            auto pv = [&](int j) {
                if (!mbar_wait(bar_p_full(j & 1), (uint32_t)(j >> 1) & 1u, wc, kErrTimeout)) {
                    ok = false;
                    return;
                }
                tc_fence_after_sync();
                uint32_t vaddr;
                int slot;
                if (!take(vaddr, slot)) {
                    ok = false;
                    return;
                }
                const uint32_t p_tmem = tmem + T::S_COL + (uint32_t)(j & 1) * BN;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bdesc =
                        make_sdesc_sw128(vaddr + kk * 2048, T::CHUNK_BYTES, 1024);
                    mma_ts(tmem + T::O_COL, p_tmem + kk * 8, bdesc, T::IDESC_PV,
                           (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(bar_pv_done);
                tc_commit(bar_empty(slot));
            };
            for (int j = 0; j < n_blocks && ok; ++j) {
                qk(j);
                if (ok && j >= 1) pv(j - 1);
            }
            if (ok) pv(n_blocks - 1);
            tc_commit(bar_mma_done);  // drain every MMA this thread issued before teardown
            mbar_wait_drain(bar_mma_done, 0, p.timeout_ns, p.status);
        }
    } else {
        // ------------------------------ softmax warps 0-3 ------------------------------
        const int row = threadIdx.x;  // TMEM lane
        const int64_t i = q0 + row;
        const bool row_valid = i < p.sq;
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);

        // Q row -> TMEM (A operand of S = Q K^T): column c holds channels 2c (low) and 2c+1.
        {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q + ((bi * p.sq + (row_valid ? i : 0)) * p.hq + h) * T::DQK);
#pragma unroll
            for (int c = 0; c < T::DQK / 64; ++c) {
                uint32_t r[32];
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    uint4 x = row_valid ? __ldg(src + c * 8 + t) : make_uint4(0, 0, 0, 0);
                    r[4 * t + 0] = x.x;
                    r[4 * t + 1] = x.y;
                    r[4 * t + 2] = x.z;
                    r[4 * t + 3] = x.w;
                }
                tmem_st32(tl + T::Q_COL + c * 32, r);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_q_ready);
        }

        const float sl2 = p.scale_log2;
        const bool pos_scale = sl2 >= 0.f;
        const int64_t lim_row = CAUSAL ? i + p.sk - p.sq : p.sk - 1;
        const int64_t lim = lim_row < p.sk - 1 ? lim_row : p.sk - 1;  // last allowed key
        float m_ref = -INFINITY;  // exponent reference (log2 units); changes lazily
        float l = 0.f;            // sum of exp2(x - m_ref) over the keys seen so far
        bool ok = true;

        for (int j = 0; j < n_blocks; ++j) {
            const int sb = j & 1;
            ok = __all_sync(0xffffffffu,
                            mbar_wait(bar_s_full(sb), (uint32_t)(j >> 1) & 1u, wc, kErrTimeout));
            if (!ok) break;
            tc_fence_after_sync();
            uint32_t sraw[BN];
#pragma unroll
            for (int c = 0; c < BN / 32; ++c)
                tmem_ld32(tl + T::S_COL + sb * BN + c * 32,
                          *reinterpret_cast<uint32_t(*)[32]>(&sraw[c * 32]));
            tmem_wait_ld();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(sraw[c]);

            const bool masked_block = j >= mask_from;
            const int64_t kbase = (int64_t)j * BN;
            // Extreme of the raw scores in the direction of the scale's sign, valid keys only.
            float ext = pos_scale ? -INFINITY : INFINITY;
            if (masked_block) {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const bool v = kbase + c <= lim;
                    ext = v ? (pos_scale ? fmaxf(ext, s[c]) : fminf(ext, s[c])) : ext;
                }
            } else {
                if (pos_scale) {
#pragma unroll
                    for (int c = 0; c < BN; ++c) ext = fmaxf(ext, s[c]);
                } else {
#pragma unroll
                    for (int c = 0; c < BN; ++c) ext = fminf(ext, s[c]);
                }
            }
            const bool any_valid = pos_scale ? (ext != -INFINITY) : (ext != INFINITY);
            const float m_blk = any_valid ? ext * sl2 : -INFINITY;
            const float m_new = fmaxf(m_ref, m_blk);
            // Lazy rescale: keep the old reference while the running max stays within 2^8 of it;
            // the final O / l uses the same reference, so the result is exact either way.
            const bool need = m_new > m_ref + 8.0f;
            float alpha = 1.f;
            if (need) {
                alpha = ex2(m_ref - m_new);
                m_ref = m_new;
                l *= alpha;
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                // O holds blocks < j: wait for the previous P V, then scale O in place. When S_j
                // has landed, P V_{j-2} is complete (it was issued before Q K_j), so bar_pv_done
                // is in phase j-1 or j and the parity test on phase j-1 is unambiguous.
                ok = __all_sync(0xffffffffu, mbar_wait(bar_pv_done, (uint32_t)(j - 1) & 1u, wc,
                                                       kErrTimeout));
                if (!ok) break;
                tc_fence_after_sync();
#pragma unroll 1
                for (int c = 0; c < T::DV / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tl + T::O_COL + c * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        r[t] = __float_as_uint(__uint_as_float(r[t]) * alpha);
                    tmem_st32(tl + T::O_COL + c * 32, r);
                }
            }
            const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
            const float neg_m = -m_use;
            float rs = 0.f;
            uint32_t pk[BN / 2];
            if (masked_block) {
#pragma unroll
                for (int c = 0; c < BN / 2; ++c) {
                    const float p0 =
                        (kbase + 2 * c <= lim) ? ex2(fmaf(s[2 * c], sl2, neg_m)) : 0.f;
                    const float p1 =
                        (kbase + 2 * c + 1 <= lim) ? ex2(fmaf(s[2 * c + 1], sl2, neg_m)) : 0.f;
                    rs += p0 + p1;
                    pk[c] = pack_bf16x2(p0, p1);
                }
            } else {
#pragma unroll
                for (int c = 0; c < BN / 2; ++c) {
                    const float p0 = ex2(fmaf(s[2 * c], sl2, neg_m));
                    const float p1 = ex2(fmaf(s[2 * c + 1], sl2, neg_m));
                    rs += p0 + p1;
                    pk[c] = pack_bf16x2(p0, p1);
                }
            }
            l += rs;
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
                tmem_st32(tl + T::S_COL + sb * BN + c * 32,
                          *reinterpret_cast<const uint32_t(*)[32]>(&pk[c * 32]));
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_p_full(sb));
        }

        // ---- epilogue: O = O / l in bf16, LSE = ln 2 * (m_ref + log2 l)
        // The MMA thread commits bar_mma_done after its last P V. (bar_pv_done cannot be used
        // here: when S_{n-1} lands, up to two P V phases may still be pending, so a parity test
        // on it could pass a phase early.)
        if (n_blocks > 0 && ok) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_mma_done, 0u, wc, kErrTimeout));
            tc_fence_after_sync();
        }
        const bool have_o = n_blocks > 0 && ok;
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.o + ((bi * p.sq + (row_valid ? i : 0)) * p.hq + h) *
                                                        T::DV);
#pragma unroll 1
        for (int c = 0; c < T::DV / 32; ++c) {
            uint32_t r[32];
            if (have_o) {
                tmem_ld32(tl + T::O_COL + c * 32, r);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int t = 0; t < 32; ++t) r[t] = 0u;
            }
            uint32_t w[16];
#pragma unroll
            for (int t = 0; t < 16; ++t)
                w[t] = pack_bf16x2(__uint_as_float(r[2 * t]) * inv_l,
                                   __uint_as_float(r[2 * t + 1]) * inv_l);
            if (row_valid && ok) {
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    dst[c * 4 + t] = make_uint4(w[4 * t], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
            }
        }
        if (p.lse != nullptr && row_valid && ok)
            p.lse[(bi * p.hq + h) * p.sq + i] =
                l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }

    // ---- teardown: every tcgen05 access is complete (MMA drained, loads waited) ----
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 4) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, T::TMEM_COLS);
    }
}

}  // namespace b200
