// attn_fwd_kernel.cuh -- fused attention forward pass for sm_100a (B200).
//
// Computes O = softmax(scale * Q K^T [+ causal mask]) V and LSE = log sum exp(scale * Q K^T)
// per query row, for bf16 BSHD tensors with grouped-query heads: the Triton "_attn_fwd" MHA
// forward of "Tune MHA config & small-head pipeline pathology" (Motivation; shapes in "Source of
// shapes"), re-designed for the 5th-generation tensor core.
//
// Work unit: NT consecutive 128-row query tiles (NT = 1 or 2, per head dim and layout) of one
// (batch or packed sequence, query head). Every K/V tile brought into shared memory serves all
// NT query tiles, which halves the L2 -> SM traffic per FLOP when NT = 2. Persistent kernel: one
// CTA per SM takes units in rounds, in the order AttnParams::order selects (round robin, snake,
// or weight-major snake); within a head the units that see the most keys (causal) come first.
// The pipeline does not drain between units.
//
// Items: the pipeline steps through "items" (key block j, query tile t) in the order
// (0,0) (0,1) (1,0) (1,1) ... for NT = 2, or (0) (1) (2) ... for NT = 1. Item g uses score buffer
// g % 2, so one item's Q K^T runs on the tensor core while the previous item's softmax runs.
//
// Roles: NSM softmax warpgroups, then the MMA warp and the TMA warp. NSM = 1: 192 threads.
// NSM = 2: 384 threads (a third warpgroup holds the MMA and TMA warps and two idle warps, so
// that setmaxnreg can move registers from it to the softmax warpgroups).
//   softmax + epilogue warps: thread r owns row r (= TMEM lane r) of a query tile and keeps its
//              whole score row of the current item in registers. Turns each score block S into
//              P (online softmax: exp2 with the scale folded into one packed fp32x2 FMA, part of
//              the exp2 on the FMA pipe, lazy rescaling of O, row sums as packed fp32x2 adds),
//              and writes each tile's finished O rows (divided by the row sums) and LSE right
//              after handing over that tile's first P of the next unit. When Q lives in TMEM they
//              also copy each tile's Q from the shared-memory staging buffer into TMEM once the
//              tile's last Q K^T of the current unit has landed.
//              NSM = 1: warps 0-3 take every item in order. NSM = 2: warps 4t..4t+3 own query
//              tile t, so the two tiles' softmax run side by side.
//   warp 4*NSM   MMA issuer (one thread): S = Q K^T and O += P V. A operand: Q from TMEM or
//              shared memory, then P from TMEM; B operand: K, V from shared memory; fp32
//              accumulators in TMEM.
//   warp 4*NSM+1 TMA producer (one thread): each unit's Q into the staging buffer, and K, V
//              tiles through two rings of shared-memory slots, in the order the MMA warp takes
//              them.
//
// Template flags: CAUSAL; VARLEN (packed sequences: per-unit offsets from cu_seqlens); EXT
// (sliding window and sinks: a first key block per unit, a lower per-key bound, and each row's
// reference and sum started at the head's sink logit). Traits flag FP8: E4M3 Q, K, V with
// kind::f8f6f4 MMAs (K = 32 per instruction, the same 32 bytes of a row as bf16's K = 16), P
// rounded to E4M3 four per TMEM column, and per-(batch, head) descales folded into the exp2
// factor (Q, K) and the final division (V).
//
// Tensor memory (128 lanes x 512 columns of 32 bit): S0 | S1 (BN columns each; P in bf16 pairs
// overwrites the first BN/2 columns of its own S buffer, E4M3 quads the first BN/4) | O for each query tile (DV fp32
// columns each) | Q for each query tile when it lives in TMEM (DQK/2 columns of bf16 pairs).
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
constexpr int kMaxUnitClasses = 256;  // order 3: (sequence, rank) classes at most

struct AttnParams {
    __nv_bfloat16* o;
    float* lse;  // may be null
    // Dense: b batches of sq queries / sk keys. Packed sequences: b sequences, sq = the longest
    // query length (it sizes the unit grid), sk unused; sequence i owns query rows
    // cu_q[i] .. cu_q[i+1] and key rows cu_k[i] .. cu_k[i+1] of the packed tensors.
    int64_t b, hq, hk, sq, sk;
    const int* cu_q;
    const int* cu_k;
    int64_t total_q, total_k;
    // Sliding window: row i keeps only keys j >= i + sk - sq - window (window < 0: no window).
    // Sinks: one logit per query head that joins every row's softmax denominator (or null).
    int64_t window;
    const float* sinks;
    int64_t group;    // hq / hk
    int64_t n_qu;     // query units per (batch, head): ceil(sq / (NT * 128))
    int64_t n_units;  // b * hq * n_qu (below 2^31)
    FastDiv div_nqu, div_hq, div_group;  // by n_qu, hq and group
    // Order in which CTAs take units. Round r gives CTA c the position
    // r * grid + (r odd and order != 0 ? grid - 1 - c : c); position -> unit is the identity
    // (head-major, heaviest unit of a head first) for order 0 / 1, and for order 2 the
    // weight-major order (the k-th heaviest unit of every head, then the (k+1)-th ...). Order 3
    // (packed sequences): the (sequence, rank) classes sorted by decreasing cost, all query
    // heads of a class in turn.
    int order;
    FastDiv div_bh;  // by b * hq
    float scale_log2; // |scale| * log2(e); the sign of scale is applied by the MMA (negate A)
    uint32_t idesc_qk;
    int* status;      // device error word
    unsigned long long timeout_ns;
    int starve;       // failure test: the TMA producer loads nothing (see attn_debug_starve)
    int alt;          // two tiles: their softmax take turns block by block (else run freely)
    // E4M3 inputs: fp32 descales per (batch, head) of Q [b, hq], K and V [b, hk] (else null)
    const float* q_descale;
    const float* k_descale;
    const float* v_descale;
};

template <int DQK_, int DV_, int BN_, int NT_, int NSM_, bool Q_TMEM_, int NK_, int NV_,
          uint32_t EXP_FMA_PAIRS_ = 0, bool FP8_ = false, bool PIPE_ = false>
struct AttnTraits {
    static constexpr int DQK = DQK_;
    static constexpr int DV = DV_;
    static constexpr int BN = BN_;          // keys per block
    static constexpr int BM = 128;          // query rows per tile
    static constexpr int NT = NT_;          // query tiles per unit
    static constexpr int NSM = NSM_;        // softmax warpgroups: 1 (all tiles) or NT (one each)
    static constexpr bool Q_TMEM = Q_TMEM_; // Q as the TMEM A operand (else from shared memory)
    static constexpr int NK = NK_;          // K slots
    static constexpr int NV = NV_;          // V slots
    // E4M3 Q, K, V (kind::f8f6f4 MMAs, P in E4M3) instead of bf16 (kind::f16, P in bf16)
    static constexpr bool FP8 = FP8_;
    static constexpr int EB = FP8 ? 1 : 2;    // bytes per input element
    static constexpr int CE = 128 / EB;       // elements per 128-byte swizzled row chunk
    static constexpr int KSTEP = 32 / EB;     // K per MMA instruction: 32 bytes of a row
    static constexpr int QCH = DQK * EB / 128;  // 128-byte column chunks of a Q/K row
    static constexpr int VCH = DV * EB / 128;
    static constexpr uint32_t CHUNK_BYTES = BN * 128;   // one column chunk (TMA box) of K or V
    static constexpr uint32_t QCHUNK_BYTES = BM * 128;  // one column chunk (TMA box) of Q
    static constexpr uint32_t Q_TILE_BYTES = BM * DQK * EB;
    static constexpr uint32_t Q_BYTES = NT * Q_TILE_BYTES;
    static constexpr uint32_t K_TILE_BYTES = BN * DQK * EB;
    static constexpr uint32_t V_TILE_BYTES = BN * DV * EB;
    static_assert(!FP8 || (!Q_TMEM && (DQK * EB) % 128 == 0 && (DV * EB) % 128 == 0),
                  "E4M3 inputs: Q from shared memory, whole 128-byte row chunks");
    // PIPE (two tiles): every tile owns two score buffers and runs its own pipelined MMA order,
    // Q K^T of block j+1 before P V of block j, so the tensor core computes a tile's next S while
    // its softmax works on the current one and the two tiles' softmax run side by side. Without
    // PIPE two tiles share the two score buffers (one each), and NT = 1 alternates between them.
    static constexpr bool PIPE = PIPE_;
    static_assert(!PIPE || NT == 2, "");
    static constexpr int NSBUF = PIPE ? 2 * NT : 2;  // score buffers
    // One copy of the softmax body (two tiles, one score buffer each): a masked block first
    // sets its disallowed scores to -inf, then runs the body of the unmasked blocks. The other
    // layouts keep a second, masked body that skips chunks no row of the warp allows (measured
    // on B200: one body is 1-2.5 % faster at d128, d192/128 and E4M3, 4 % slower at d64).
    static constexpr bool ONE_BODY = NT == 2 && !PIPE;
    // tensor memory columns
    static constexpr uint32_t O_COL0 = NSBUF * BN;
    static constexpr uint32_t Q_COL0 = NSBUF * BN + NT * DV;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(NSBUF * BN + NT * DV + (Q_TMEM ? NT * DQK / 2 : 0) <= 512,
                  "tensor memory budget");
    static_assert(DQK % 64 == 0 && DV % 64 == 0 && BN % 64 == 0 && BN <= 256 && DV <= 256, "");
    static_assert(NT == 1 || NT == 2, "");
    // shared memory: [Q staging][K slots][V slots][O staging, if used][barriers][TMEM base,
    // abort flag]
    static constexpr uint32_t K_OFF = Q_BYTES;
    static constexpr uint32_t V_OFF = K_OFF + NK * K_TILE_BYTES;
    static constexpr uint32_t O_OFF = V_OFF + NV * V_TILE_BYTES;
    static constexpr int NBAR = 2 * NK + 2 * NV + 2 * NSBUF + 3 + 4 * NT;
    // The epilogue writes O through a shared-memory tile and TMA stores (one per warp and
    // 64-column box: slab o_slab(tile, box, warp % 4), 32 rows x 128 bytes) when the tiles fit
    // next to the rings; otherwise each thread stores its own row.
    static constexpr uint32_t O_STAGE_BYTES = NT * BM * DV * 2;
    // after the barriers: the TMEM base and the abort flag (16 bytes), then order 3's class list
    // and class costs (uint16 each)
    static constexpr uint32_t TAIL_BYTES = 16 + 4 * kMaxUnitClasses;
    static constexpr bool O_TMA = 1024 + O_OFF + O_STAGE_BYTES + NBAR * 8 + TAIL_BYTES <= 232448;
    static constexpr uint32_t o_slab(int tt, int bx, int w4)
    {
        return (uint32_t)(((tt * (DV / 64) + bx) * 4 + w4) * 4096);
    }
    static constexpr uint32_t BARS_OFF = O_OFF + (O_TMA ? O_STAGE_BYTES : 0);
    static constexpr uint32_t SMEM_BYTES = 1024 + BARS_OFF + NBAR * 8 + TAIL_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(NSM == NT, "one softmax warpgroup per query tile (and one MMA issuer each)");
    // Threads. One softmax warpgroup: warps 0-3 softmax, warp 4 MMA issuer, warp 5 TMA producer.
    // Two: warpgroup 0 holds the MMA issuers (warps 0 and 2) and the TMA producer (warp 1; warp
    // 3 idles), warpgroups 1 and 2 the softmax of tiles 0 and 1. The block is three full
    // warpgroups so that registers can move between them: at launch every thread has
    // LAUNCH_REGS (the cap for 384 threads); the issuers' warpgroup drops to AUX_REGS and the
    // softmax warpgroups rise to SOFTMAX_REGS, which keeps the block's total unchanged (a larger
    // total would never be granted). The issuers come first: the warp schedulers favour older
    // warps, and an issuer that waits for issue slots behind two busy softmax warps on its SM
    // sub-partition delays its tile's next S (measured on B200).
    static constexpr int NUM_THREADS = NSM == 1 ? 192 : 384;
    static constexpr int AUX_WG = NSM == 1 ? 1 : 0;  // the warpgroup of the MMA and TMA warps
    static constexpr int SM_WG0 = NSM == 1 ? 0 : 1;  // the first softmax warpgroup
    static constexpr int MMA_WARP = 4 * AUX_WG;      // MMA issuer (tile 0, or every tile when NT = 1)
    static constexpr int TMA_WARP = 4 * AUX_WG + 1;
    static constexpr int MMA_WARP2 = 4 * AUX_WG + 2; // NT = 2: issuer of tile 1's MMAs
    static constexpr int LAUNCH_REGS = 168;
    static constexpr int SOFTMAX_REGS = 224;
    static constexpr int AUX_REGS = 56;
    static_assert(NSM == 1 || 2 * 128 * SOFTMAX_REGS + 128 * AUX_REGS <= NUM_THREADS * LAUNCH_REGS,
                  "register split exceeds the launch allocation");
    // Score pairs whose exp2 runs on the FMA pipe (exp2_fma_pair) rather than the MUFU unit: bit
    // k set = pairs with index k mod 8 in each row, in the one-warpgroup softmax.
    static constexpr uint32_t EXP_FMA_PAIRS = EXP_FMA_PAIRS_;
    static constexpr uint32_t IDESC_QK =
        FP8 ? make_idesc_e4m3(128, BN, false, false) : make_idesc_bf16(128, BN, false, false);
    static constexpr uint32_t IDESC_PV =
        FP8 ? make_idesc_e4m3(128, DV, false, true) : make_idesc_bf16(128, DV, false, true);
};

// Wait bounded only by time (used to drain in-flight copies / MMAs before exit, also after an
// abort, so it ignores the abort flag).
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity,
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

// One work unit: (batch or sequence, query head, NT query tiles starting at row q0 of the
// sequence) and its key blocks.
struct UnitInfo {
    int64_t bi, h, g, q0;
    int64_t sq, sk;      // this sequence's query / key lengths
    int64_t qrow, krow;  // its first query / key row in the tensor maps' row dimension
    int64_t obase;       // O row of its query 0: O[(obase + i) * hq + h]
    int64_t lbase;       // LSE of its query i at lse[lbase + i]
    int bmap;            // the tensor maps' batch coordinate
    int j_begin;    // first key block with an allowed key for some row of the unit (window)
    int n_blocks;   // key blocks j_begin .. n_blocks-1 are visited
    int mask_lo;    // blocks < mask_lo need the window's lower per-key bound
    int mask_from;  // blocks >= mask_from need the per-key mask (causal diagonal, ragged tail)
};

template <int BN, int NT, bool CAUSAL, bool VARLEN, bool EXT>
__device__ __forceinline__ UnitInfo unit_info(const AttnParams& p, int64_t u)
{
    UnitInfo t;
    const uint32_t uu = (uint32_t)u;
    const uint32_t bh = fast_div(uu, p.div_nqu);
    const uint32_t qu = p.div_nqu.d - 1 - (uu - bh * p.div_nqu.d);  // within a head: most keys first
    const uint32_t bi = fast_div(bh, p.div_hq);
    const uint32_t h = bh - bi * p.div_hq.d;
    t.bi = bi;
    t.h = h;
    t.g = fast_div(h, p.div_group);
    t.q0 = qu * (NT * 128);
    if (VARLEN) {
        // offsets clamped into the packed tensors, so no row outside them is ever addressed
        int64_t qs = __ldg(p.cu_q + bi), qe = __ldg(p.cu_q + bi + 1);
        int64_t ks = __ldg(p.cu_k + bi), ke = __ldg(p.cu_k + bi + 1);
        qs = qs < 0 ? 0 : (qs > p.total_q ? p.total_q : qs);
        qe = qe < qs ? qs : (qe > p.total_q ? p.total_q : qe);
        ks = ks < 0 ? 0 : (ks > p.total_k ? p.total_k : ks);
        ke = ke < ks ? ks : (ke > p.total_k ? p.total_k : ke);
        t.sq = qe - qs;
        t.sk = ke - ks;
        // ranks count from this sequence's own last query tile, so that rank k of every
        // sequence is its k-th most expensive unit; ranks past its tiles are empty
        const int64_t rank = (int64_t)(p.div_nqu.d - 1 - qu);
        const int64_t nqu_seq = (t.sq + NT * 128 - 1) / (NT * 128);
        t.q0 = rank < nqu_seq ? (nqu_seq - 1 - rank) * (NT * 128) : t.sq;
        t.qrow = qs;
        t.krow = ks;
        t.obase = qs;
        t.lbase = (int64_t)h * p.total_q + qs;
        t.bmap = 0;
    } else {
        t.sq = p.sq;
        t.sk = p.sk;
        t.qrow = 0;
        t.krow = 0;
        t.obase = (int64_t)bi * p.sq;
        t.lbase = ((int64_t)bi * p.hq + h) * p.sq;
        t.bmap = (int)bi;
    }
    t.j_begin = 0;
    t.mask_lo = 0;
    if (t.q0 >= t.sq) {  // (packed sequences) no query row of this sequence here
        t.n_blocks = 0;
        t.mask_from = 0;
        return t;
    }
    const int64_t n_kv = (t.sk + BN - 1) / BN;
    if (CAUSAL) {
        const int64_t last_row = (t.q0 + NT * 128 - 1 < t.sq - 1) ? t.q0 + NT * 128 - 1 : t.sq - 1;
        const int64_t last_key = last_row + t.sk - t.sq;
        int64_t nb = last_key < 0 ? 0 : last_key / BN + 1;
        nb = nb < n_kv ? nb : n_kv;
        const int64_t first_lim = t.q0 + t.sk - t.sq + 1;  // keys < first_lim: allowed for all
        int64_t full = first_lim <= 0 ? 0 : first_lim / BN;
        full = full < t.sk / BN ? full : t.sk / BN;
        t.n_blocks = (int)nb;
        t.mask_from = (int)(full < nb ? full : nb);
    } else {
        t.n_blocks = (int)n_kv;
        t.mask_from = (int)(t.sk / BN);
    }
    if (EXT && p.window >= 0) {  // keys left of every row's window are never visited
        const int64_t last_row = (t.q0 + NT * 128 - 1 < t.sq - 1) ? t.q0 + NT * 128 - 1 : t.sq - 1;
        const int64_t lo_first = t.q0 + t.sk - t.sq - p.window;  // the unit's smallest bound
        const int64_t lo_last = last_row + t.sk - t.sq - p.window;  // and its largest
        int64_t jb = lo_first <= 0 ? 0 : lo_first / BN;
        jb = jb < t.n_blocks ? jb : t.n_blocks;
        t.j_begin = (int)jb;
        t.mask_lo = (int)(lo_last <= 0 ? 0 : (lo_last + BN - 1) / BN);
    }
    return t;
}

// The MMA forms of the traits' input type.
template <class T>
__device__ __forceinline__ void mma_ss_t(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t acc)
{
    if constexpr (T::FP8) mma_ss_f8(d, a, b, idesc, acc);
    else mma_ss(d, a, b, idesc, acc);
}

template <class T>
__device__ __forceinline__ void mma_ts_t(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                         uint32_t acc)
{
    if constexpr (T::FP8) mma_ts_f8(d, a, b, idesc, acc);
    else mma_ts(d, a, b, idesc, acc);
}

// S = Q K^T for one query tile and one key block: one MMA of M128 x N=BN x K=KSTEP per 32
// bytes of a row (DQK/16 for bf16, DQK/32 for E4M3). K (and Q when staged in shared memory)
// are K-major 128-byte swizzled tiles in 128-byte column chunks, so k-step kk starts (kk / 4)
// chunks and (kk % 4) * 32 bytes in. q is a TMEM column (Q in TMEM) or a shared-memory address.
template <class T>
__device__ __forceinline__ void issue_qk_mmas(uint32_t d_tmem, uint32_t q, uint32_t kaddr,
                                              uint32_t idesc)
{
    const uint64_t b0 = make_sdesc_sw128(kaddr, 16, 1024);
    if constexpr (T::Q_TMEM) {
#pragma unroll
        for (int kk = 0; kk < T::DQK / 16; ++kk)
            mma_ts(d_tmem, q + kk * 8,
                   sdesc_advance(b0, (kk >> 2) * T::CHUNK_BYTES + (kk & 3) * 32), idesc,
                   kk > 0 ? 1u : 0u);
    } else {
        const uint64_t a0 = make_sdesc_sw128(q, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < T::DQK * T::EB / 32; ++kk)
            mma_ss_t<T>(d_tmem, sdesc_advance(a0, (kk >> 2) * T::QCHUNK_BYTES + (kk & 3) * 32),
                   sdesc_advance(b0, (kk >> 2) * T::CHUNK_BYTES + (kk & 3) * 32), idesc,
                   kk > 0 ? 1u : 0u);
    }
}

// O += P V for one query tile and one key block: BN/KSTEP MMAs of M128 x N=DV x K=KSTEP with P
// from TMEM (8 columns = 32 bytes per k-step: 16 bf16 or 32 E4M3 weights of a row) and V an
// MN-major 128-byte swizzled tile (KSTEP keys = KSTEP * 128 bytes per k-step).
template <class T>
__device__ __forceinline__ void issue_pv_mmas(uint32_t o_tmem, uint32_t p_tmem, uint32_t vaddr,
                                              bool accumulate)
{
    const uint64_t b0 = make_sdesc_sw128(vaddr, T::CHUNK_BYTES, 1024);
#pragma unroll
    for (int kk = 0; kk < T::BN / T::KSTEP; ++kk)
        mma_ts_t<T>(o_tmem, p_tmem + kk * 8, sdesc_advance(b0, kk * T::KSTEP * 128), T::IDESC_PV,
                    (accumulate || kk > 0) ? 1u : 0u);
}

// EXT: the sliding window and the sinks of AttnParams are honoured (compiled out otherwise).
template <class T, bool CAUSAL, bool VARLEN, bool EXT>
__global__ void __launch_bounds__(T::NUM_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_o, const AttnParams p)
{
    constexpr int BN = T::BN;
    constexpr int NT = T::NT;
    // O through the staging tile and TMA stores, except for packed sequences, where a store box
    // could reach into the next sequence's rows
    constexpr bool OTMA = T::O_TMA && !VARLEN;
    constexpr int NK = T::NK;
    constexpr int NV = T::NV;
    constexpr uint32_t FULL = 0xffffffffu;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);  // SW128 needs 1 KB
    const uint32_t sbase = smem_addr(smem);
    const uint32_t q_stage = sbase;
    const uint32_t k_slots = sbase + T::K_OFF;
    const uint32_t v_slots = sbase + T::V_OFF;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::BARS_OFF);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + T::NBAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    uint16_t* vcls = reinterpret_cast<uint16_t*>(smem + T::BARS_OFF + T::NBAR * 8 + 16);

    auto bar = [&](int i) { return smem_addr(&bars[i]); };
    auto bar_kfull = [&](int s) { return bar(s); };
    auto bar_kempty = [&](int s) { return bar(NK + s); };
    auto bar_vfull = [&](int s) { return bar(2 * NK + s); };
    auto bar_vempty = [&](int s) { return bar(2 * NK + NV + s); };
    constexpr int B0 = 2 * NK + 2 * NV;
    constexpr int NSB = T::NSBUF;
    auto bar_s_full = [&](int s) { return bar(B0 + s); };
    auto bar_p_full = [&](int s) { return bar(B0 + NSB + s); };
    // per tile: its last P V is complete (NT = 1 and PIPE, where S(j+1) lands before P V(j))
    auto bar_pv_done = [&](int t) { return bar(B0 + 2 * NSB + t); };
    const uint32_t bar_q_full = bar(B0 + 2 * NSB + NT);
    const uint32_t bar_q_empty = bar(B0 + 2 * NSB + NT + 1);
    const uint32_t bar_mma_done = bar(B0 + 2 * NSB + NT + 2);
    constexpr int B1 = B0 + 2 * NSB + NT + 3;
    // per query tile: its Q is in TMEM / its O is final / its O has been read out
    auto bar_q_tmem = [&](int t) { return bar(B1 + t); };
    auto bar_o_full = [&](int t) { return bar(B1 + NT + t); };
    auto bar_o_free = [&](int t) { return bar(B1 + 2 * NT + t); };
    // Score buffer of tile tt's key block number jg (counted over all units), and the parity of
    // the phase of that buffer's barriers the block completes.
    auto sbuf_of = [&](int64_t jg, int tt) -> int {
        return T::PIPE ? tt * 2 + (int)(jg & 1) : (NT == 2 ? tt : (int)(jg & 1));
    };
    auto sphase_of = [&](int64_t jg) -> uint32_t {
        return (T::PIPE || NT == 1) ? (uint32_t)(jg >> 1) & 1u : (uint32_t)jg & 1u;
    };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NK; ++s) {
            mbar_init(bar_kfull(s), 1);
            mbar_init(bar_kempty(s), NT);  // one commit per MMA issuer
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(bar_vfull(s), 1);
            mbar_init(bar_vempty(s), NT);
        }
        for (int s = 0; s < NSB; ++s) {
            mbar_init(bar_s_full(s), 1);
            mbar_init(bar_p_full(s), 128);  // one warpgroup writes each P
        }
        for (int t = 0; t < NT; ++t) mbar_init(bar_pv_done(t), 1);
        mbar_init(bar_q_full, 1);
        // per-tile copy-out (Q in TMEM) / each issuer's last Q K^T of the unit
        mbar_init(bar_q_empty, T::Q_TMEM ? 128 * NT : NT);
        mbar_init(bar_mma_done, NT);
        for (int t = 0; t < NT; ++t) {
            mbar_init(bar_q_tmem(t), 128);
            mbar_init(bar_o_full(t), 1);
            mbar_init(bar_o_free(t), 128);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == T::MMA_WARP) {
        tmem_alloc(smem_addr(tmem_holder), T::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == T::TMA_WARP && lane == 0) {
        tma_prefetch_desc(&tmap_q);
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_v);
    }
    if constexpr (VARLEN) {
        // Order 3: every CTA sorts the (sequence, rank) classes by decreasing cost -- the key
        // blocks a class's units visit, plus 2 for a unit's fixed cost; ties in class order --
        // so that CTAs take the most expensive units first, whatever the sequence lengths.
        if (p.order == 3) {
            uint16_t* vcost = vcls + kMaxUnitClasses;
            const int nqu = (int)p.n_qu;
            const int ncls = (int)p.b * nqu;  // at most kMaxUnitClasses (checked on the host)
            for (int c = threadIdx.x; c < ncls; c += blockDim.x) {
                const int bi = c / nqu, k = c - (c / nqu) * nqu;
                const UnitInfo t =
                    unit_info<T::BN, T::NT, CAUSAL, VARLEN, EXT>(p, (int64_t)bi * p.hq * nqu + k);
                const int nb = t.n_blocks - t.j_begin;
                vcost[c] = (uint16_t)(nb > 0 ? (nb + 2 < 65535 ? nb + 2 : 65535) : 0);
            }
            __syncthreads();
            for (int c = threadIdx.x; c < ncls; c += blockDim.x) {
                const uint32_t w = vcost[c];
                int rank = 0;
                for (int c2 = 0; c2 < ncls; ++c2) {
                    const uint32_t w2 = vcost[c2];
                    rank += (w2 > w || (w2 == w && c2 < c)) ? 1 : 0;
                }
                vcls[rank] = (uint16_t)c;
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_holder;
    const WaitCtx wc{abort_flag, p.status, p.timeout_ns};
    // The unit this CTA takes in round r, or -1 when round r is past the last unit (and so is
    // every later round). Every unit is taken by exactly one (CTA, round).
    auto unit_of = [&](int64_t r) -> int64_t {
        const int64_t g = gridDim.x;
        const int64_t c = blockIdx.x;
        const int64_t pos = r * g + ((p.order != 0 && (r & 1)) ? g - 1 - c : c);
        if (pos >= p.n_units) return -1;
        if (VARLEN && p.order == 3) {
            const uint32_t cr = fast_div((uint32_t)pos, p.div_hq);  // class rank
            const uint32_t h = (uint32_t)pos - cr * p.div_hq.d;
            const uint32_t c = vcls[cr];
            const uint32_t bi = fast_div(c, p.div_nqu), k = c - bi * p.div_nqu.d;
            return ((int64_t)bi * p.hq + h) * p.div_nqu.d + k;
        }
        if (p.order == 2) {
            const uint32_t k = fast_div((uint32_t)pos, p.div_bh);  // rank within its head
            const uint32_t bh = (uint32_t)pos - k * p.div_bh.d;
            return (int64_t)bh * p.div_nqu.d + k;
        }
        return pos;
    };
    // First round from r whose unit has at least one key block, or -1.
    auto busy_from = [&](int64_t r) -> int64_t {
        for (;; ++r) {
            const int64_t u = unit_of(r);
            if (u < 0) return -1;
            const UnitInfo t = unit_info<BN, NT, CAUSAL, VARLEN, EXT>(p, u);
            if (t.n_blocks > t.j_begin) return r;
        }
    };

    if constexpr (T::NSM == 2) {
        if ((warp >> 2) == T::AUX_WG) setmaxnreg_dec<T::AUX_REGS>();  // registers to the softmax
    }
    if (warp == T::TMA_WARP) {
        // ------------------------------ TMA producer ------------------------------
        // Walks the MMA warp's item sequence and issues each load at the point the MMA warp
        // will first need it (K_j at the Q K^T of item (j, 0), V_j at the P V of item (j, 0)).
        // Failure test (p.starve): no tile is ever loaded, so every other role's first wait runs
        // out; they all leave through the bounded abort and drain path.
        if (lane == 0 && !p.starve) {
            int kq = 0, vq = 0;  // K / V items issued
            int q_cnt = 0;       // Q units issued
            bool ok = true;
            auto load_q = [&](int64_t u) {
                const UnitInfo t = unit_info<BN, NT, CAUSAL, VARLEN, EXT>(p, u);
                if (!mbar_wait(bar_q_empty, (uint32_t)(q_cnt & 1) ^ 1u, wc, kErrTimeout)) {
                    ok = false;
                    return;
                }
                mbar_arrive_expect_tx(bar_q_full, T::Q_BYTES);
                for (int tt = 0; tt < NT; ++tt)
                    for (int ch = 0; ch < T::QCH; ++ch)
                        tma_load_4d(q_stage + tt * T::Q_TILE_BYTES + ch * T::QCHUNK_BYTES, &tmap_q,
                                    bar_q_full, ch * T::CE, (int)t.h,
                                    (int)(t.qrow + t.q0 + tt * 128), t.bmap);
                ++q_cnt;
            };
            auto load_k = [&](const UnitInfo& t, int j) {
                const int slot = kq % NK;
                if (!mbar_wait(bar_kempty(slot), (uint32_t)((kq / NK) & 1) ^ 1u, wc,
                               kErrTimeout)) {
                    ok = false;
                    return;
                }
                const uint32_t dst = k_slots + slot * T::K_TILE_BYTES;
                mbar_arrive_expect_tx(bar_kfull(slot), T::K_TILE_BYTES);
                for (int ch = 0; ch < T::QCH; ++ch)
                    tma_load_4d(dst + ch * T::CHUNK_BYTES, &tmap_k, bar_kfull(slot), ch * T::CE,
                                (int)t.g, (int)(t.krow + (int64_t)j * BN), t.bmap);
                ++kq;
            };
            auto load_v = [&](const UnitInfo& t, int j) {
                const int slot = vq % NV;
                if (!mbar_wait(bar_vempty(slot), (uint32_t)((vq / NV) & 1) ^ 1u, wc,
                               kErrTimeout)) {
                    ok = false;
                    return;
                }
                const uint32_t dst = v_slots + slot * T::V_TILE_BYTES;
                mbar_arrive_expect_tx(bar_vfull(slot), T::V_TILE_BYTES);
                for (int ch = 0; ch < T::VCH; ++ch)
                    tma_load_4d(dst + ch * T::CHUNK_BYTES, &tmap_v, bar_vfull(slot), ch * T::CE,
                                (int)t.g, (int)(t.krow + (int64_t)j * BN), t.bmap);
                ++vq;
            };
            bool pend = false;  // the P V step still owed for the previous item
            UnitInfo pend_t{};
            int pend_j = 0, pend_tt = 0;
            int64_t r = busy_from(0);
            if (r >= 0) load_q(unit_of(r));
            while (r >= 0 && ok) {
                const UnitInfo t = unit_info<BN, NT, CAUSAL, VARLEN, EXT>(p, unit_of(r));
                const int64_t rn = busy_from(r + 1);
                const int64_t un = rn >= 0 ? unit_of(rn) : -1;
                // PIPE: each tile's issuer takes K(j+1) before V(j), as with one tile
                constexpr int NTP = T::PIPE ? 1 : NT;
                for (int j = t.j_begin; j < t.n_blocks && ok; ++j) {
                    for (int tt = 0; tt < NTP && ok; ++tt) {
                        if (tt == 0) load_k(t, j);  // the Q K^T step of item (j, tt)
                        if (ok && T::Q_TMEM && j == t.j_begin && tt == 0 && un >= 0)
                            load_q(un);  // the staging buffer was emptied into TMEM
                        if (ok && pend && pend_tt == 0) load_v(pend_t, pend_j);  // P V step
                        pend = true;
                        pend_t = t;
                        pend_j = j;
                        pend_tt = tt;
                    }
                }
                // With Q read from shared memory, the next unit's Q can only replace this one
                // after the unit's last Q K^T (the MMA warp commits bar_q_empty then).
                if (ok && !T::Q_TMEM && un >= 0) load_q(un);
                r = rn;
            }
            if (ok && pend && pend_tt == 0) load_v(pend_t, pend_j);
            // Nothing may be in flight when the CTA exits: wait for the last load of each slot
            // and for the last Q load.
            for (int d = 0; d < (kq < NK ? kq : NK); ++d) {
                const int idx = kq - 1 - d;
                mbar_wait_drain(bar_kfull(idx % NK), (uint32_t)(idx / NK) & 1u, p.timeout_ns,
                                p.status);
            }
            for (int d = 0; d < (vq < NV ? vq : NV); ++d) {
                const int idx = vq - 1 - d;
                mbar_wait_drain(bar_vfull(idx % NV), (uint32_t)(idx / NV) & 1u, p.timeout_ns,
                                p.status);
            }
            if (q_cnt > 0)
                mbar_wait_drain(bar_q_full, (uint32_t)(q_cnt - 1) & 1u, p.timeout_ns, p.status);
        }
    } else if (warp == T::MMA_WARP || (NT == 2 && warp == T::MMA_WARP2)) {
        // ------------------------------ MMA issuers ------------------------------
        // NT = 2: one warp per query tile (warp MMA_WARP issues tile 0's MMAs, warp MMA_WARP2
        // tile 1's), so the two tiles' instruction streams are issued side by side. Each tile has
        // one score buffer, so its chain is Q K^T(j), then P V(j) once P(j) is out, then
        // Q K^T(j+1). NT = 1: one warp; its tile alternates between the two score buffers, so
        // Q K^T(g+1) is issued before P V(g).
        // The whole warp runs the loop (waits included) with warp-uniform values; one elected
        // lane issues each batch of MMAs and its commits.
        {
            const int my_tt = (warp == T::MMA_WARP) ? 0 : 1;
            bool ok = true;
            int kq = 0, vq = 0;  // K / V blocks taken
            int64_t jg = 0;      // key blocks stepped through (all units)
            int units = 0;       // busy units started
            auto wait_all = [&](uint32_t bar, uint32_t parity) {
                return __all_sync(FULL, mbar_wait(bar, parity, wc, kErrTimeout));
            };
            // Q K^T of tile tt's current block into score buffer sb. Every issuer takes K(j)
            // itself: the slot is freed when all NT issuers have committed kempty.
            auto qk = [&](int sb, bool first, int tt, bool last_item) {
                if (T::Q_TMEM && first) {  // this tile's Q of the new unit must be in TMEM
                    if (!wait_all(bar_q_tmem(tt), (uint32_t)(units & 1))) {
                        ok = false;
                        return;
                    }
                    tc_fence_after_sync();
                }
                const int kslot = kq % NK;
                const uint32_t phase = (uint32_t)(kq / NK) & 1u;
                ++kq;
                if (!wait_all(bar_kfull(kslot), phase)) {
                    ok = false;
                    return;
                }
                if (elect_one()) {
                    issue_qk_mmas<T>(tmem + (uint32_t)sb * BN,
                                     T::Q_TMEM ? tmem + T::Q_COL0 + tt * (T::DQK / 2)
                                               : q_stage + tt * T::Q_TILE_BYTES,
                                     k_slots + kslot * T::K_TILE_BYTES, p.idesc_qk);
                    tc_commit(bar_s_full(sb));
                    tc_commit(bar_kempty(kslot));
                    if (!T::Q_TMEM && last_item) tc_commit(bar_q_empty);
                }
                __syncwarp();
            };
            // P V of tile tt's block whose P is in score buffer sb (phase ph), of busy unit
            // number uidx.
            auto pv = [&](int sb, uint32_t ph, bool first, int tt, bool last_block, int uidx) {
                if (!wait_all(bar_p_full(sb), ph)) {
                    ok = false;
                    return;
                }
                if (first && uidx > 0 && !wait_all(bar_o_free(tt), (uint32_t)(uidx - 1) & 1u)) {
                    ok = false;
                    return;
                }
                tc_fence_after_sync();
                const int vslot = vq % NV;
                const uint32_t phase = (uint32_t)(vq / NV) & 1u;
                ++vq;
                if (!wait_all(bar_vfull(vslot), phase)) {
                    ok = false;
                    return;
                }
                if (elect_one()) {
                    issue_pv_mmas<T>(tmem + T::O_COL0 + tt * T::DV, tmem + (uint32_t)sb * BN,
                                     v_slots + vslot * T::V_TILE_BYTES, !first);
                    if (NT == 1 || T::PIPE) tc_commit(bar_pv_done(tt));
                    tc_commit(bar_vempty(vslot));
                    if (last_block) tc_commit(bar_o_full(tt));
                }
                __syncwarp();
            };
            // NT = 1 and PIPE: the P V of each block is issued after the next block's Q K^T (also
            // across units), so the tensor core computes the next S while the softmax works on
            // this one.
            bool pend = false, pend_last = false, pend_first = false;
            int pend_u = 0, pend_sb = 0;
            uint32_t pend_ph = 0;
            for (int64_t r = 0; ok; ++r) {
                const int64_t u = unit_of(r);
                if (u < 0) break;
                const UnitInfo t = unit_info<BN, NT, CAUSAL, VARLEN, EXT>(p, u);
                if (t.n_blocks <= t.j_begin) continue;
                if (!T::Q_TMEM) {  // the unit's Q in the staging buffer (read by the MMA)
                    if (!wait_all(bar_q_full, (uint32_t)(units & 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                }
                for (int j = t.j_begin; j < t.n_blocks && ok; ++j, ++jg) {
                    const bool first = j == t.j_begin, last = j == t.n_blocks - 1;
                    if constexpr (NT == 2 && !T::PIPE) {
                        qk(my_tt, first, my_tt, last);
                        if (ok) pv(my_tt, (uint32_t)jg & 1u, first, my_tt, last, units);
                    } else {
                        const int tt = T::PIPE ? my_tt : 0;
                        qk(sbuf_of(jg, tt), first, tt, last);
                        if (!ok) break;
                        if (pend) pv(pend_sb, pend_ph, pend_first, tt, pend_last, pend_u);
                        pend = true;
                        pend_sb = sbuf_of(jg, tt);
                        pend_ph = sphase_of(jg);
                        pend_first = first;
                        pend_last = last;
                        pend_u = units;
                    }
                }
                ++units;
            }
            if ((NT == 1 || T::PIPE) && ok && pend)
                pv(pend_sb, pend_ph, pend_first, T::PIPE ? my_tt : 0, pend_last, pend_u);
            // drain every MMA this warp issued before teardown
            if (elect_one()) tc_commit(bar_mma_done);
            __syncwarp();
            mbar_wait_drain(bar_mma_done, 0, p.timeout_ns, p.status);
        }
    } else if ((warp >> 2) != T::AUX_WG) {
        // ------ softmax + epilogue warpgroups (warps 0-3 with one, 4-11 with two warpgroups) ------
        // NSM = 1: the warpgroup takes every query tile's items in order. NSM = 2: warpgroup w
        // takes the items of query tile w. Either way each thread keeps its whole score row of
        // the current item in registers (one TMEM read, a single pass).
        if constexpr (T::NSM == 2) setmaxnreg_inc<T::SOFTMAX_REGS>();
        constexpr int NTW = T::NSM == 1 ? NT : 1;  // query tiles this warpgroup handles
        const int wg = (warp >> 2) - T::SM_WG0;
        const int w4 = warp & 3;                  // TMEM lanes 32*w4 .. 32*w4+31
        const int row = threadIdx.x & 127;        // TMEM lane = row of the query tile
        const uint32_t tl = tmem + ((uint32_t)(w4 * 32) << 16);
        float sl2 = p.scale_log2;  // per unit with E4M3 inputs (times the Q and K descales)
        auto tile_of = [&](int k) { return T::NSM == 1 ? k : wg; };
        bool ok = true;
        int64_t jg = 0;  // key blocks stepped through so far (all units); item g = jg * NT + tile
        int units = 0;   // busy units whose items are done

        // Staged Q of busy unit number qidx, tile tt (128-byte swizzled rows, as TMA wrote them)
        // -> this row's TMEM columns of that tile; then tell the MMA warp and the producer.
        auto copy_q = [&](int qidx, int tt) -> bool {
            if (!__all_sync(FULL, mbar_wait(bar_q_full, (uint32_t)(qidx & 1), wc, kErrTimeout)))
                return false;
#pragma unroll
            for (int ch = 0; ch < T::QCH; ++ch) {
                uint32_t r[32];
                const uint8_t* rowp = smem + tt * T::Q_TILE_BYTES + ch * T::QCHUNK_BYTES + row * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 x = *reinterpret_cast<const uint4*>(rowp + ((c ^ (row & 7)) << 4));
                    r[4 * c + 0] = x.x;
                    r[4 * c + 1] = x.y;
                    r[4 * c + 2] = x.z;
                    r[4 * c + 3] = x.w;
                }
                tmem_st32(tl + T::Q_COL0 + tt * (T::DQK / 2) + ch * 32, r);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_q_tmem(tt));
            mbar_arrive(bar_q_empty);
            return true;
        };

        // Epilogue of tile tt of busy unit number uidx: wait for that tile's last P V, read this
        // row of its O from TMEM (then free the accumulator), write O / l in bf16 and the LSE.
        auto epilogue = [&](int64_t u, int tt, float m_ref, float l, int uidx) -> bool {
            const UnitInfo t = unit_info<BN, NT, CAUSAL, VARLEN, EXT>(p, u);
            if (!__all_sync(FULL,
                            mbar_wait(bar_o_full(tt), (uint32_t)(uidx & 1), wc, kErrTimeout)))
                return false;
            tc_fence_after_sync();
            const int64_t i = t.q0 + tt * 128 + row;
            const bool row_valid = i < t.sq;
            // E4M3 inputs: the V descale joins the final division
            const float vds = T::FP8 ? __ldg(p.v_descale + t.bi * p.hk + t.g) : 1.f;
            const float inv_l = l > 0.f ? vds / l : 0.f;
            if constexpr (OTMA) {
                // This warp's 32 rows go to its own slab of the staging tile (one 32-row, 128-byte
                // swizzled box per 64 columns), then one lane stores the slab with TMA; rows past
                // sq are clipped by the tensor map. The slab is reused only after the previous
                // store from it has been read out.
                if (lane == 0) bulk_wait_read_all();
                __syncwarp();
                const int r32 = row & 31;
#pragma unroll 1
                for (int c = 0; c < T::DV / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tl + T::O_COL0 + tt * T::DV + c * 32, r);
                    tmem_wait_ld();
                    if (c == T::DV / 32 - 1) {
                        // this tile's O has been read out: the next unit's P V may overwrite it
                        tc_fence_before_sync();
                        mbar_arrive(bar_o_free(tt));
                    }
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l,
                                           __uint_as_float(r[2 * e + 1]) * inv_l);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int u16 = c * 4 + q4;  // 16-byte unit of the row
                        uint8_t* slab = smem + T::O_OFF + T::o_slab(tt, u16 >> 3, w4);
                        *reinterpret_cast<uint4*>(slab + r32 * 128 + (((u16 & 7) ^ (r32 & 7)) << 4)) =
                            make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                const int64_t row0 = t.q0 + tt * 128 + w4 * 32;
                if (lane == 0 && row0 < t.sq) {
#pragma unroll
                    for (int bx = 0; bx < T::DV / 64; ++bx)
                        tma_store_4d(&tmap_o, sbase + T::O_OFF + T::o_slab(tt, bx, w4), bx * 64,
                                     (int)t.h, (int)(t.qrow + row0), t.bmap);
                    bulk_commit_group();
                }
            } else {
                uint4* dst = reinterpret_cast<uint4*>(
                    p.o + ((t.obase + (row_valid ? i : 0)) * p.hq + t.h) * T::DV);
#pragma unroll 1
                for (int c = 0; c < T::DV / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tl + T::O_COL0 + tt * T::DV + c * 32, r);
                    tmem_wait_ld();
                    if (c == T::DV / 32 - 1) {
                        // this tile's O has been read out: the next unit's P V may overwrite it
                        tc_fence_before_sync();
                        mbar_arrive(bar_o_free(tt));
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
            }
            if (row_valid && p.lse)
                p.lse[t.lbase + i] =
                    l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
            return true;
        };

        // One key block of one query tile: mask (MASKED only), row max, lazy rescale, exp2 and
        // row sums, P into tensor memory. MASKED is a compile-time flag, so the common block
        // with every key allowed runs one straight-line body with no per-chunk branches.
        int64_t lim[NTW] = {};  // last allowed key of this thread's row in each tile
        int64_t lol[NTW] = {};  // first allowed key (the window's lower bound), may be negative
        float m_ref[NTW] = {};  // exponent reference (log2 units); moves lazily
        float l[NTW] = {};      // sum of exp2(x - m_ref) over the keys seen so far
        int j_begin = 0;
        // ONE_BODY layouts: keys j*BN + c with lor <= c <= rel are allowed; every other score of
        // the block becomes -inf (its max term and its p = exp2(-inf) then vanish). Chunks that
        // every row of the warp allows entirely are left as they are.
        auto mask_scores = [&](uint32_t(&sr)[BN], int k, int j) {
            int64_t rel64 = lim[k] - (int64_t)j * BN;
            rel64 = rel64 < -1 ? -1 : (rel64 > BN ? BN : rel64);
            int lor = 0;  // no lower bound without a window
            if (EXT) {
                int64_t lor64 = lol[k] - (int64_t)j * BN;
                lor = (int)(lor64 < 0 ? 0 : (lor64 > BN ? BN : lor64));
            }
            const int rel = (int)rel64;
            const int rel_lo = __reduce_min_sync(FULL, rel);
            const int lor_hi = EXT ? __reduce_max_sync(FULL, lor) : 0;
#pragma unroll
            for (int ch = 0; ch < BN / 32; ++ch) {
                if (ch * 32 + 31 <= rel_lo && ch * 32 >= lor_hi) continue;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int c = ch * 32 + e;
                    sr[c] = (c <= rel && c >= lor) ? sr[c] : 0xff800000u;
                }
            }
        };
        auto softmax_block = [&](const bool MASKED, uint32_t(&sr)[BN], int k, int tt, int j,
                                 int64_t jgb, uint32_t s_col) -> bool {
            // Keys j*BN + c with lor <= c <= rel are allowed. Per 32-key chunk the warp takes
            // one of three uniform paths: every row of the warp allows the whole chunk
            // (nothing to do), none allows any of it (skipped below: no max, P = 0 without
            // exp2), or the chunk holds some row's bound: then the disallowed scores become
            // -inf, so the max ignores them and their p = exp2(-inf) is exactly 0 (the scale
            // factor is never 0: the launch clamps it to at least 2^-100).
            uint32_t skip = 0;  // bit ch: no row of this warp allows a key of chunk ch
            if (MASKED) {
                int64_t rel64 = lim[k] - (int64_t)j * BN;
                rel64 = rel64 < -1 ? -1 : (rel64 > BN ? BN : rel64);
                int lor = 0;  // no lower bound without a window
                if (EXT) {
                    int64_t lor64 = lol[k] - (int64_t)j * BN;
                    lor = (int)(lor64 < 0 ? 0 : (lor64 > BN ? BN : lor64));
                }
                const int rel = (int)rel64;
                const int rel_lo = __reduce_min_sync(FULL, rel);
                const int rel_hi = __reduce_max_sync(FULL, rel);
                const int lor_lo = EXT ? __reduce_min_sync(FULL, lor) : 0;
                const int lor_hi = EXT ? __reduce_max_sync(FULL, lor) : 0;
#pragma unroll
                for (int ch = 0; ch < BN / 32; ++ch) {
                    if (ch * 32 > rel_hi || ch * 32 + 31 < lor_lo) {
                        skip |= 1u << ch;
                        continue;
                    }
                    if (ch * 32 + 31 <= rel_lo && ch * 32 >= lor_hi) continue;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int c = ch * 32 + e;
                        sr[c] = (c <= rel && c >= lor) ? sr[c] : 0xff800000u;
                    }
                }
            }
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int ch = 0; ch < BN / 32; ++ch) {
                if (MASKED && ((skip >> ch) & 1u)) continue;
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    mx[c & 3] = fmax3(mx[c & 3], __uint_as_float(sr[ch * 32 + 2 * c]),
                                      __uint_as_float(sr[ch * 32 + 2 * c + 1]));
            }
            const float bmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            const float m_blk = (bmax == -INFINITY) ? -INFINITY : bmax * sl2;
            const float m_new = fmaxf(m_ref[k], m_blk);
            // Lazy rescale: keep the old reference while the running max stays within 2^8 of
            // it; the final O / l uses the same reference, so the result is exact.
            const bool need = m_new > m_ref[k] + 8.0f;
            float alpha = 1.f;
            if (need) {
                alpha = ex2(m_ref[k] - m_new);
                m_ref[k] = m_new;
                l[k] *= alpha;
            }
            if (j > j_begin && __any_sync(FULL, need)) {
                // O holds blocks < j of this tile: scale it in place once its last P V is
                // complete. With two tiles sharing the score buffers that P V was issued by this
                // tile's issuer before this block's Q K^T, so it is complete now that S has
                // landed (a commit covers all earlier MMAs of its thread). With one tile, or with
                // PIPE, it was issued after this block's Q K^T: wait for it on the tile's
                // bar_pv_done (one phase per block; that barrier is then in the phase of block
                // jg-1 or jg, so the parity test on jg-1 is unambiguous).
                if (NT == 1 || T::PIPE) {
                    if (!__all_sync(FULL, mbar_wait(bar_pv_done(tt), (uint32_t)(jgb - 1) & 1u, wc,
                                                    kErrTimeout)))
                        return false;
                    tc_fence_after_sync();
                }
#pragma unroll 1
                for (int c = 0; c < T::DV / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tl + T::O_COL0 + tt * T::DV + c * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                    tmem_st32(tl + T::O_COL0 + tt * T::DV + c * 32, r);
                }
            }
            const float neg_m = (m_ref[k] == -INFINITY) ? 0.f : -m_ref[k];
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ch = 0; ch < BN / 32; ++ch) {
                uint32_t pk[16];
                if (MASKED && ((skip >> ch) & 1u)) {  // no row of this warp allows a key here
#pragma unroll
                    for (int c = 0; c < 16; ++c) pk[c] = 0u;
                } else {
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int e = ch * 32 + 2 * c;
                        float x0, x1;
                        fma2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1]), sl2, neg_m, x0,
                             x1);
                        float p0, p1;
                        if ((T::EXP_FMA_PAIRS >> (c & 7)) & 1u) {
                            exp2_fma_pair(x0, x1, p0, p1);
                        } else {
                            p0 = ex2(x0);
                            p1 = ex2(x1);
                        }
                        add2(acc[(2 * c) & 3], acc[(2 * c + 1) & 3], p0, p1);
                        if constexpr (T::FP8) {  // four E4M3 weights per column
                            const uint32_t h2 = pack_e4m3x2(p0, p1);
                            if (c & 1) pk[c >> 1] |= h2 << 16;
                            else pk[c >> 1] = h2;
                        } else {
                            pk[c] = pack_bf16x2(p0, p1);
                        }
                    }
                }
                // P chunk ch (16 columns of bf16 pairs, or 8 of E4M3 quads) overwrites S columns
                // already read
                if constexpr (T::FP8) tmem_st8(s_col + ch * 8, pk);
                else tmem_st16(s_col + ch * 16, pk);
            }
            l[k] += (acc[0] + acc[1]) + (acc[2] + acc[3]);
            return true;
        };

        bool pend = false;  // a finished unit whose epilogues have not run yet
        int64_t pend_u = 0;
        float pend_m[NTW], pend_l[NTW];
#pragma unroll
        for (int k = 0; k < NTW; ++k) pend_m[k] = pend_l[k] = 0.f;
        int pend_idx = 0;
        if (T::Q_TMEM && busy_from(0) >= 0)
            for (int k = 0; k < NTW && ok; ++k) ok = copy_q(0, tile_of(k));
        for (int64_t r = 0; ok; ++r) {
            const int64_t u = unit_of(r);
            if (u < 0) break;
            const UnitInfo t = unit_info<BN, NT, CAUSAL, VARLEN, EXT>(p, u);
            if (t.n_blocks <= t.j_begin) {  // no key for any row of this unit: O = 0, LSE = -inf
                // (or the head's sink logit)
#pragma unroll
                for (int k = 0; k < NTW; ++k) {
                    const int64_t i = t.q0 + tile_of(k) * 128 + row;
                    if (i < t.sq) {
                        uint4* dst = reinterpret_cast<uint4*>(
                            p.o + ((t.obase + i) * p.hq + t.h) * T::DV);
#pragma unroll 1
                        for (int c = 0; c < T::DV / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
                        if (p.lse)
                            p.lse[t.lbase + i] =
                                (EXT && p.sinks) ? __ldg(p.sinks + t.h) : -INFINITY;
                    }
                }
                continue;
            }
            const bool has_next = busy_from(r + 1) >= 0;
            if constexpr (T::FP8) {
                // S holds sums of code products; the descales fold into the exp2 factor, kept at
                // 2^-100 or more as on the host (a NaN product also becomes 2^-100)
                const float f = p.scale_log2 * __ldg(p.q_descale + t.bi * p.hq + t.h) *
                                __ldg(p.k_descale + t.bi * p.hk + t.g);
                sl2 = f > 0x1p-100f ? f : 0x1p-100f;
            }
            // A sink logit starts every row with that logit as reference and exp2(0) = 1 in
            // the sum: it then joins the denominator exactly, through every lazy rescale.
            const bool has_sink = EXT && p.sinks != nullptr;
            const float sink_l2 =
                has_sink ? __ldg(p.sinks + t.h) * 1.4426950408889634f : -INFINITY;
#pragma unroll
            for (int k = 0; k < NTW; ++k) {
                const int64_t i = t.q0 + tile_of(k) * 128 + row;
                const int64_t lim_row = CAUSAL ? i + t.sk - t.sq : t.sk - 1;
                lim[k] = lim_row < t.sk - 1 ? lim_row : t.sk - 1;
                lol[k] = (EXT && p.window >= 0) ? i + t.sk - t.sq - p.window : (int64_t)-1 << 40;
                m_ref[k] = sink_l2;
                l[k] = has_sink ? 1.f : 0.f;
            }
            j_begin = t.j_begin;
            const int n_blocks = t.n_blocks, mask_lo = t.mask_lo, mask_from = t.mask_from;

            for (int j = j_begin; j < n_blocks && ok; ++j, ++jg) {
#pragma unroll
                for (int k = 0; k < NTW; ++k) {
                    const int tt = tile_of(k);
                    const int sb = sbuf_of(jg, tt);  // score buffer
                    const uint32_t s_col = tl + sb * BN;
                    // The two tiles' softmax take turns: tile 1's block jg after tile 0's, tile 0's
                    // block jg after tile 1's block jg-1 (p_full of the other tile completes once
                    // per block, and cannot run a phase ahead of this wait). With E4M3 inputs the
                    // turn is taken after this block's S has landed and been loaded (measured on
                    // B200: +2.8 % for E4M3, 4-14 % slower for bf16 at d128 and d192/128).
                    constexpr bool TURN = NT == 2 && !T::PIPE;
                    constexpr bool TURN_LATE = TURN && T::FP8;
                    auto take_turn = [&]() -> bool {
                        bool w = true;
                        if (tt == 1)
                            w = mbar_wait(bar_p_full(0), (uint32_t)(jg & 1), wc, kErrTimeout);
                        else if (jg > 0)
                            w = mbar_wait(bar_p_full(1), (uint32_t)((jg - 1) & 1), wc,
                                          kErrTimeout);
                        return __all_sync(FULL, w);
                    };
                    if (TURN && !TURN_LATE && p.alt) {
                        ok = take_turn();
                        if (!ok) break;
                    }
                    ok = __all_sync(FULL, mbar_wait(bar_s_full(sb), sphase_of(jg), wc,
                                                    kErrTimeout));
                    if (!ok) break;
                    tc_fence_after_sync();
                    if (T::Q_TMEM && j == n_blocks - 1 && has_next) {
                        // This tile's last Q K^T of the unit is complete (its S has landed), so
                        // its Q columns can take the next unit's Q now, ahead of this softmax.
                        ok = copy_q(units + 1, tt);
                        if (!ok) break;
                    }
                    uint32_t sr[BN];
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c)
                        tmem_ld32(s_col + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
                    tmem_wait_ld();
                    if (TURN_LATE && p.alt) {
                        ok = take_turn();
                        if (!ok) break;
                    }
                    if constexpr (T::ONE_BODY) {
                        if ((EXT && j < mask_lo) || j >= mask_from) mask_scores(sr, k, j);
                        ok = softmax_block(false, sr, k, tt, j, jg, s_col);
                    } else if ((EXT && j < mask_lo) || j >= mask_from) {
                        ok = softmax_block(true, sr, k, tt, j, jg, s_col);
                    } else {
                        ok = softmax_block(false, sr, k, tt, j, jg, s_col);
                    }
                    if (!ok) break;
                    tmem_wait_st();
                    tc_fence_before_sync();
                    mbar_arrive(bar_p_full(sb));
                    if (j == j_begin && pend) {
                        // Tile tt of the previous unit, now that its successor's first P is out.
                        ok = epilogue(pend_u, tt, pend_m[k], pend_l[k], pend_idx);
                        if (k == NTW - 1) pend = false;
                        if (!ok) break;
                    }
                }
            }
            if (!ok) break;
            pend = true;
            pend_u = u;
#pragma unroll
            for (int k = 0; k < NTW; ++k) {
                pend_m[k] = m_ref[k];
                pend_l[k] = l[k];
            }
            pend_idx = units;
            ++units;
        }
        if (ok && pend)
            for (int k = 0; k < NTW && ok; ++k)
                ok = epilogue(pend_u, tile_of(k), pend_m[k], pend_l[k], pend_idx);
        // every O store this warp issued is complete before the CTA exits
        if (OTMA && lane == 0) bulk_wait_all();
    }

    // ---- teardown: every tcgen05 access is complete (MMAs drained, loads waited) ----
    tc_fence_before_sync();
    __syncthreads();
    if (warp == T::MMA_WARP) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem, T::TMEM_COLS);
    }
}

}  // namespace b200
