// attn_fwd_kernel.cuh -- fused attention forward pass for sm_100a (B200).
//
// Computes O = softmax(scale * Q K^T [+ causal mask]) V and LSE = log sum exp(scale * Q K^T)
// per query row, for bf16 BSHD tensors with grouped-query heads: the Triton "_attn_fwd" MHA
// forward of "Tune MHA config & small-head pipeline pathology" (Motivation; shapes in "Source of
// shapes"), re-designed for the 5th-generation tensor core.
//
// Persistent kernel: one CTA per SM walks a list of work tiles (one 128-row query tile of one
// (batch, query head)), ordered so that the tiles that see the most keys (causal) come first.
// The pipeline does not drain between tiles.
//
// Roles (192 threads; at most two warps per SM sub-partition, so a softmax thread can keep its
// whole score row in registers):
//   warps 0-3  softmax + epilogue: thread t owns query row t (= TMEM lane t). Copies its Q row
//              from the shared-memory staging buffer into TMEM, turns each score block S into P
//              (online softmax: exp2 with the scale folded into one FMA, lazy rescaling of O),
//              and writes the finished O row (divided by the row sum) and LSE. A tile's epilogue
//              runs right after the next tile's first P is handed over, so the wait for the last
//              P V of the tile overlaps useful work.
//   warp 4     MMA issuer (one thread): S = Q K^T and O += P V, A operand from TMEM (Q, then P),
//              B operand from shared memory (K, V), fp32 accumulators in TMEM.
//   warp 5     TMA producer (one thread): the next tile's Q into the staging buffer, and K, V
//              tiles through a ring of shared-memory slots in the MMA warp's order
//              (K0, K1, V0, K2, V1, ...).
//
// Tensor memory (128 lanes x 512 columns of 32 bit): S0 | S1 (two BN-wide score buffers, so one
// block's Q K^T overlaps the previous block's softmax; P in bf16 pairs overwrites the first BN/2
// columns of its own S buffer) | O (DV fp32 columns) | Q (DQK/2 columns of bf16 pairs).
//
// Every mbarrier wait is bounded in time; a wait that gives up sets the device error word and a
// CTA-wide abort flag, every role then leaves its loops, in-flight TMA loads and MMAs are drained
// (with a time bound as well) and tensor memory is freed before the CTA exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace b200 {

constexpr int kErrTimeout = 10;  // B200ATTN_ERR_TIMEOUT

struct AttnParams {
    __nv_bfloat16* o;
    float* lse;  // may be null
    int64_t b, hq, hk, sq, sk;
    int64_t group;     // hq / hk
    int64_t n_qtiles;  // ceil(sq / 128)
    int64_t n_tiles;   // b * hq * n_qtiles
    float scale_log2;  // |scale| * log2(e); the sign of scale is applied by the MMA (negate A)
    uint32_t idesc_qk;
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
    static constexpr int QCH = DQK / 64;  // 128-byte (64-element) column chunks of a Q/K row
    static constexpr int VCH = DV / 64;
    static constexpr uint32_t CHUNK_BYTES = BN * 128;   // one 64-column TMA box of K or V
    static constexpr uint32_t QCHUNK_BYTES = BM * 128;  // one 64-column TMA box of Q
    static constexpr uint32_t Q_BYTES = BM * DQK * 2;
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
    // shared memory: [Q staging][K/V slots][barriers][TMEM base, abort flag]
    static constexpr uint32_t SLOTS_OFF = Q_BYTES;
    static constexpr uint32_t BARS_OFF = SLOTS_OFF + NSLOT * SLOT_BYTES;
    static constexpr int NBAR = 2 * NSLOT + 11;
    static constexpr uint32_t SMEM_BYTES = 1024 + BARS_OFF + NBAR * 8 + 16;
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

// One work tile: (batch, query head, 128-row query tile) and the key blocks it needs.
struct TileInfo {
    int64_t bi, h, g, q0;
    int n_blocks;   // key blocks with at least one allowed key for some row of the tile
    int mask_from;  // blocks >= mask_from need the per-key mask (causal diagonal, ragged tail)
};

template <int BN, bool CAUSAL>
__device__ __forceinline__ TileInfo tile_info(const AttnParams& p, int64_t u)
{
    TileInfo t;
    const int64_t bh_count = p.b * p.hq;
    const int64_t qi = u / bh_count;
    const int64_t qt = p.n_qtiles - 1 - qi;  // tiles that see the most keys first
    const int64_t bh = u - qi * bh_count;
    t.bi = bh / p.hq;
    t.h = bh - t.bi * p.hq;
    t.g = t.h / p.group;
    t.q0 = qt * 128;
    const int64_t n_kv = (p.sk + BN - 1) / BN;
    if (CAUSAL) {
        const int64_t last_row = (t.q0 + 127 < p.sq - 1) ? t.q0 + 127 : p.sq - 1;
        const int64_t last_key = last_row + p.sk - p.sq;
        int64_t nb = last_key < 0 ? 0 : last_key / BN + 1;
        nb = nb < n_kv ? nb : n_kv;
        const int64_t first_lim = t.q0 + p.sk - p.sq + 1;  // keys < first_lim: allowed for all
        int64_t full = first_lim <= 0 ? 0 : first_lim / BN;
        full = full < p.sk / BN ? full : p.sk / BN;
        t.n_blocks = (int)nb;
        t.mask_from = (int)(full < nb ? full : nb);
    } else {
        t.n_blocks = (int)n_kv;
        t.mask_from = (int)(p.sk / BN);
    }
    return t;
}

template <class T, bool CAUSAL>
__global__ void __launch_bounds__(T::NUM_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const AttnParams p)
{
    constexpr int BN = T::BN;
    constexpr int NSLOT = T::NSLOT;
    constexpr uint32_t FULL = 0xffffffffu;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);  // SW128 needs 1 KB
    const uint32_t sbase = smem_addr(smem);
    const uint32_t q_stage = sbase;
    const uint32_t slots = sbase + T::SLOTS_OFF;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BARS_OFF);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + T::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    auto bar = [&](int i) { return smem_addr(&bars[i]); };
    auto bar_full = [&](int s) { return bar(s); };
    auto bar_empty = [&](int s) { return bar(NSLOT + s); };
    auto bar_s_full = [&](int s) { return bar(2 * NSLOT + s); };
    auto bar_p_full = [&](int s) { return bar(2 * NSLOT + 2 + s); };
    const uint32_t bar_pv_done = bar(2 * NSLOT + 4);
    const uint32_t bar_q_full = bar(2 * NSLOT + 5);
    const uint32_t bar_q_empty = bar(2 * NSLOT + 6);
    const uint32_t bar_q_tmem = bar(2 * NSLOT + 7);
    const uint32_t bar_o_full = bar(2 * NSLOT + 8);
    const uint32_t bar_o_free = bar(2 * NSLOT + 9);
    const uint32_t bar_mma_done = bar(2 * NSLOT + 10);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

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
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_empty, 128);
        mbar_init(bar_q_tmem, 128);
        mbar_init(bar_o_full, 1);
        mbar_init(bar_o_free, 128);
        mbar_init(bar_mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 4) {
        tmem_alloc(smem_addr(tmem_holder), T::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 5 && lane == 0) {
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    const WaitCtx wc{abort_flag, p.status, p.timeout_ns};

    const int64_t u0 = blockIdx.x;
    const int64_t ustep = gridDim.x;

    // First tile of this CTA's list (from u) that has at least one key block, or -1.
    auto busy_from = [&](int64_t u) -> int64_t {
        for (; u < p.n_tiles; u += ustep)
            if (tile_info<BN, CAUSAL>(p, u).n_blocks > 0) return u;
        return -1;
    };

    if (warp >= 4) {
        if (warp == 5) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            int kv_it = 0;  // K/V items issued
            int q_cnt = 0;  // Q tiles issued
            bool ok = true;
            auto load_q = [&](int64_t u) {
                const TileInfo t = tile_info<BN, CAUSAL>(p, u);
                if (!mbar_wait(bar_q_empty, (uint32_t)(q_cnt & 1) ^ 1u, wc, kErrTimeout)) {
                    ok = false;
                    return;
                }
                mbar_arrive_expect_tx(bar_q_full, T::Q_BYTES);
                for (int ch = 0; ch < T::QCH; ++ch)
                    tma_load_4d(q_stage + ch * T::QCHUNK_BYTES, &tmap_q, bar_q_full, ch * 64,
                                (int)t.h, (int)t.q0, (int)t.bi);
                ++q_cnt;
            };
            auto load_kv = [&](bool is_k, const TileInfo& t, int j) {
                const int slot = kv_it % NSLOT;
                const uint32_t phase = (uint32_t)(kv_it / NSLOT) & 1u;
                if (!mbar_wait(bar_empty(slot), phase ^ 1u, wc, kErrTimeout)) {
                    ok = false;
                    return;
                }
                const uint32_t dst = slots + slot * T::SLOT_BYTES;
                mbar_arrive_expect_tx(bar_full(slot), is_k ? T::K_TILE_BYTES : T::V_TILE_BYTES);
                const int nch = is_k ? T::QCH : T::VCH;
                for (int ch = 0; ch < nch; ++ch)
                    tma_load_4d(dst + ch * T::CHUNK_BYTES,
                                is_k ? (const void*)&tmap_k : (const void*)&tmap_v,
                                bar_full(slot), ch * 64, (int)t.g, j * BN, (int)t.bi);
                ++kv_it;
            };
            // Items go out in the MMA warp's order: K of global block g, then V of block g-1
            // (also across tiles: a tile's last V follows the next tile's first K).
            bool pend = false;
            TileInfo pend_t{};
            int pend_j = 0;
            int64_t u = busy_from(u0);
            if (u >= 0) load_q(u);
            while (u >= 0 && ok) {
                const TileInfo t = tile_info<BN, CAUSAL>(p, u);
                const int64_t un = busy_from(u + ustep);
                for (int j = 0; j < t.n_blocks && ok; ++j) {
                    load_kv(true, t, j);
                    if (ok && pend) load_kv(false, pend_t, pend_j);
                    pend = true;
                    pend_t = t;
                    pend_j = j;
                    // Stage the next tile's Q as soon as this tile's Q has left the buffer.
                    if (ok && j == 0 && un >= 0) load_q(un);
                }
                u = un;
            }
            if (ok && pend) load_kv(false, pend_t, pend_j);
            // Nothing may be in flight when the CTA exits: wait for the last load of each slot
            // and for the last Q load.
            const int n_drain = kv_it < NSLOT ? kv_it : NSLOT;
            for (int d = 0; d < n_drain; ++d) {
                const int idx = kv_it - 1 - d;
                mbar_wait_drain(bar_full(idx % NSLOT), (uint32_t)(idx / NSLOT) & 1u, p.timeout_ns,
                                p.status);
            }
            if (q_cnt > 0)
                mbar_wait_drain(bar_q_full, (uint32_t)(q_cnt - 1) & 1u, p.timeout_ns, p.status);
        }
        } else {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            bool ok = true;
            int kv_it = 0;   // K/V items consumed
            int64_t gb = 0;  // global block counter (S buffer index and barrier phases)
            int tiles = 0;   // busy tiles started
            auto take = [&](uint32_t& addr, int& slot) -> bool {
                slot = kv_it % NSLOT;
                const uint32_t phase = (uint32_t)(kv_it / NSLOT) & 1u;
                ++kv_it;
                if (!mbar_wait(bar_full(slot), phase, wc, kErrTimeout)) return false;
                addr = slots + slot * T::SLOT_BYTES;
                return true;
            };
            auto qk = [&](int64_t gblk) {
                uint32_t kaddr;
                int slot;
                if (!take(kaddr, slot)) {
                    ok = false;
                    return;
                }
                const uint32_t d_tmem = tmem + T::S_COL + (uint32_t)(gblk & 1) * BN;
#pragma unroll
                for (int kk = 0; kk < T::DQK / 16; ++kk) {
                    const uint64_t bdesc = make_sdesc_sw128(
                        kaddr + (kk >> 2) * T::CHUNK_BYTES + (kk & 3) * 32, 16, 1024);
                    mma_ts(d_tmem, tmem + T::Q_COL + kk * 8, bdesc, p.idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar_s_full(gblk & 1));
                tc_commit(bar_empty(slot));
            };
            // P V for global block gblk; `first` / `last`: its position inside tile `tile_idx`.
            auto pv = [&](int64_t gblk, bool first, bool last, int tile_idx) {
                if (!mbar_wait(bar_p_full(gblk & 1), (uint32_t)(gblk >> 1) & 1u, wc,
                               kErrTimeout)) {
                    ok = false;
                    return;
                }
                if (first && tile_idx > 0 &&
                    !mbar_wait(bar_o_free, (uint32_t)(tile_idx - 1) & 1u, wc, kErrTimeout)) {
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
                const uint32_t p_tmem = tmem + T::S_COL + (uint32_t)(gblk & 1) * BN;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bdesc =
                        make_sdesc_sw128(vaddr + kk * 2048, T::CHUNK_BYTES, 1024);
                    mma_ts(tmem + T::O_COL, p_tmem + kk * 8, bdesc, T::IDESC_PV,
                           (!first || kk > 0) ? 1u : 0u);
                }
                tc_commit(bar_pv_done);
                tc_commit(bar_empty(slot));
                if (last) tc_commit(bar_o_full);
            };
            // The P V of a tile's last block is issued after the next tile's first Q K^T, so the
            // next tile's first S is computed while the softmax finishes this tile.
            bool pend = false, pend_first = false, pend_last = false;
            int pend_tile = 0;
            int64_t pend_g = 0;
            for (int64_t u = u0; u < p.n_tiles && ok; u += ustep) {
                const TileInfo t = tile_info<BN, CAUSAL>(p, u);
                if (t.n_blocks == 0) continue;
                if (!mbar_wait(bar_q_tmem, (uint32_t)(tiles & 1), wc, kErrTimeout)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                for (int j = 0; j < t.n_blocks && ok; ++j) {
                    qk(gb);
                    if (!ok) break;
                    if (pend) pv(pend_g, pend_first, pend_last, pend_tile);
                    pend = true;
                    pend_g = gb;
                    pend_first = (j == 0);
                    pend_last = (j == t.n_blocks - 1);
                    pend_tile = tiles;
                    ++gb;
                }
                ++tiles;
            }
            if (ok && pend) pv(pend_g, pend_first, pend_last, pend_tile);
            tc_commit(bar_mma_done);  // drain every MMA this thread issued before teardown
            mbar_wait_drain(bar_mma_done, 0, p.timeout_ns, p.status);
        }
        }
    } else {
        // --------------------------- softmax + epilogue warps 0-3 ---------------------------
        const int row = threadIdx.x;  // TMEM lane
        const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
        const float sl2 = p.scale_log2;
        bool ok = true;
        int64_t gb = 0;
        int tiles = 0;  // busy tiles whose key blocks are done

        // Staged Q tile number qidx (128-byte swizzled rows, as TMA wrote them) -> this row's
        // TMEM columns; then release the staging buffer and tell the MMA warp.
        auto copy_q = [&](int qidx) -> bool {
            if (!__all_sync(FULL, mbar_wait(bar_q_full, (uint32_t)(qidx & 1), wc, kErrTimeout)))
                return false;
#pragma unroll
            for (int ch = 0; ch < T::QCH; ++ch) {
                uint32_t r[32];
                const uint8_t* rowp = smem + ch * T::QCHUNK_BYTES + row * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 x =
                        *reinterpret_cast<const uint4*>(rowp + ((c ^ (row & 7)) << 4));
                    r[4 * c + 0] = x.x;
                    r[4 * c + 1] = x.y;
                    r[4 * c + 2] = x.z;
                    r[4 * c + 3] = x.w;
                }
                tmem_st32(tl + T::Q_COL + ch * 32, r);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_q_tmem);
            mbar_arrive(bar_q_empty);
            return true;
        };

        // Epilogue of busy tile number tile_idx: wait for its last P V, read this row of O from
        // TMEM (then free the accumulator for the next tile), write O / l in bf16 and the LSE.
        auto epilogue = [&](const TileInfo& t, float m_ref, float l, int tile_idx) -> bool {
            if (!__all_sync(FULL, mbar_wait(bar_o_full, (uint32_t)(tile_idx & 1), wc,
                                            kErrTimeout)))
                return false;
            tc_fence_after_sync();
            const int64_t i = t.q0 + row;
            const bool row_valid = i < p.sq;
            uint4* dst = reinterpret_cast<uint4*>(
                p.o + ((t.bi * p.sq + (row_valid ? i : 0)) * p.hq + t.h) * T::DV);
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
            for (int c = 0; c < T::DV / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tl + T::O_COL + c * 32, r);
                tmem_wait_ld();
                if (c == T::DV / 32 - 1) {
                    // O has been read out: the next tile's first P V may overwrite it.
                    tc_fence_before_sync();
                    mbar_arrive(bar_o_free);
                }
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l,
                                       __uint_as_float(r[2 * e + 1]) * inv_l);
                if (row_valid) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[c * 4 + q4] =
                            make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
                }
            }
            if (row_valid && p.lse)
                p.lse[(t.bi * p.hq + t.h) * p.sq + i] =
                    l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
            return true;
        };

        bool pend = false;  // a finished tile whose epilogue has not run yet
        TileInfo pend_t{};
        float pend_m = 0.f, pend_l = 0.f;
        int pend_idx = 0;
        if (busy_from(u0) >= 0) ok = copy_q(0);
        for (int64_t u = u0; u < p.n_tiles && ok; u += ustep) {
            const TileInfo t = tile_info<BN, CAUSAL>(p, u);
            if (t.n_blocks == 0) {  // no key at all for any row of this tile: O = 0, LSE = -inf
                const int64_t i = t.q0 + row;
                if (i < p.sq) {
                    uint4* dst = reinterpret_cast<uint4*>(
                        p.o + ((t.bi * p.sq + i) * p.hq + t.h) * T::DV);
#pragma unroll 1
                    for (int c = 0; c < T::DV / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
                    if (p.lse) p.lse[(t.bi * p.hq + t.h) * p.sq + i] = -INFINITY;
                }
                continue;
            }
            const int64_t un = busy_from(u + ustep);
            const int64_t i = t.q0 + row;
            const int64_t lim_row = CAUSAL ? i + p.sk - p.sq : p.sk - 1;
            const int64_t lim = lim_row < p.sk - 1 ? lim_row : p.sk - 1;  // last allowed key
            float m_ref = -INFINITY;  // exponent reference (log2 units); moves lazily
            float l = 0.f;            // sum of exp2(x - m_ref) over the keys seen so far

            for (int j = 0; j < t.n_blocks; ++j, ++gb) {
                const int sb = (int)(gb & 1);
                ok = __all_sync(FULL, mbar_wait(bar_s_full(sb), (uint32_t)(gb >> 1) & 1u, wc,
                                                kErrTimeout));
                if (!ok) break;
                tc_fence_after_sync();
                if (j == t.n_blocks - 1 && un >= 0) {
                    // Every Q K^T of this tile is complete (its last S has landed), so the Q
                    // columns can take the next tile's Q now, ahead of this block's softmax.
                    ok = copy_q(tiles + 1);
                    if (!ok) break;
                }
                uint32_t sr[BN];
#pragma unroll
                for (int c = 0; c < BN / 32; ++c)
                    tmem_ld32(tl + T::S_COL + sb * BN + c * 32,
                              *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
                tmem_wait_ld();

                const bool masked_block = j >= t.mask_from;
                // keys kbase + c with c <= rel are allowed (rel < 0: none, rel >= BN - 1: all)
                int64_t rel64 = lim - (int64_t)j * BN;
                rel64 = rel64 < -1 ? -1 : (rel64 > BN ? BN : rel64);
                const int rel = (int)rel64;
                float mx[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) mx[a] = -INFINITY;
                if (masked_block) {
#pragma unroll
                    for (int c = 0; c < BN; ++c) {
                        const float s = (c <= rel) ? __uint_as_float(sr[c]) : -INFINITY;
                        mx[c & 3] = fmaxf(mx[c & 3], s);
                        sr[c] = __float_as_uint(s);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < BN; ++c)
                        mx[c & 3] = fmaxf(mx[c & 3], __uint_as_float(sr[c]));
                }
                const float bmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                const float m_blk = (bmax == -INFINITY) ? -INFINITY : bmax * sl2;
                const float m_new = fmaxf(m_ref, m_blk);
                // Lazy rescale: keep the old reference while the running max stays within 2^8 of
                // it; the final O / l uses the same reference, so the result is exact either way.
                const bool need = m_new > m_ref + 8.0f;
                float alpha = 1.f;
                if (need) {
                    alpha = ex2(m_ref - m_new);
                    m_ref = m_new;
                    l *= alpha;
                }
                if (j > 0 && __any_sync(FULL, need)) {
                    // O holds blocks < j: wait for the previous P V, then scale O in place. When
                    // S_gb has landed, P V of block gb-2 is complete (it was issued before this
                    // Q K^T), so bar_pv_done is in phase gb-1 or gb and the parity test on phase
                    // gb-1 is unambiguous.
                    ok = __all_sync(FULL, mbar_wait(bar_pv_done, (uint32_t)(gb - 1) & 1u, wc,
                                                    kErrTimeout));
                    if (!ok) break;
                    tc_fence_after_sync();
#pragma unroll 1
                    for (int c = 0; c < T::DV / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(tl + T::O_COL + c * 32, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st32(tl + T::O_COL + c * 32, r);
                    }
                }
                const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
                float acc[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) acc[a] = 0.f;
#pragma unroll
                for (int h2 = 0; h2 < BN / 64; ++h2) {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int e = h2 * 64 + 2 * c;
                        float p0 = ex2(fmaf(__uint_as_float(sr[e]), sl2, neg_m));
                        float p1 = ex2(fmaf(__uint_as_float(sr[e + 1]), sl2, neg_m));
                        if (masked_block) {  // masked keys hold -inf: exactly 0 for any scale
                            p0 = (e <= rel) ? p0 : 0.f;
                            p1 = (e + 1 <= rel) ? p1 : 0.f;
                        }
                        acc[(2 * c) & 3] += p0;
                        acc[(2 * c + 1) & 3] += p1;
                        pk[c] = pack_bf16x2(p0, p1);
                    }
                    tmem_st32(tl + T::S_COL + sb * BN + h2 * 32, pk);
                }
                l += (acc[0] + acc[1]) + (acc[2] + acc[3]);
                tmem_wait_st();
                tc_fence_before_sync();
                mbar_arrive(bar_p_full(sb));
                if (j == 0 && pend) {
                    // The previous tile's epilogue, now that this tile's first P is handed over.
                    pend = false;
                    ok = epilogue(pend_t, pend_m, pend_l, pend_idx);
                    if (!ok) break;
                }
            }
            if (!ok) break;
            pend = true;
            pend_t = t;
            pend_m = m_ref;
            pend_l = l;
            pend_idx = tiles;
            ++tiles;
        }
        if (ok && pend) ok = epilogue(pend_t, pend_m, pend_l, pend_idx);
    }

    // ---- teardown: every tcgen05 access is complete (MMAs drained, loads waited) ----
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 4) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, T::TMEM_COLS);
    }
}

}  // namespace b200
