/*
 * b200attn.h -- C ABI of the B200 (sm_100a) fused attention forward library (libb200attn.so).
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller. The library never frees or
 *     keeps a caller pointer after the call returns.
 *   - Tensors are contiguous, BSHD, row-major (last dimension fastest):
 *       Q [b, sq, hq, dqk], K [b, sk, hk, dqk], V [b, sk, hk, dv], O [b, sq, hq, dv]  (bf16)
 *       LSE [b, hq, sq] (fp32, natural log), K mean [b, hk, d] (fp32);
 *     attn_fwd_varlen packs sequences along the row axis instead ([total, h, d], LSE [hq, total]);
 *     the FP8 recipe takes the same BSHD shapes as E4M3 codes (uint8) with fp32 descales
 *     [b, h] (fp8_quantize, attn_fwd_fp8).
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Work is
 *     enqueued asynchronously on it; the call does not synchronise.
 *   - Return value: B200ATTN_OK (0) on success, otherwise one of the status codes below.
 *     Argument checks run on the host before any CUDA call; when one fails nothing is launched
 *     and no output byte is written. attn_status_string() names every code.
 *   - Sizes are int64_t. Every byte offset the kernels form is 64-bit; extents that the tensor
 *     memory accelerator (TMA) cannot address are refused with B200ATTN_ERR_RANGE rather than
 *     truncated (the lesson of "MHA v4: fixes, refactor, new kernel, perf tweaks", the note on
 *     uint32 kernel-argument strides that truncated silently above 4 GiB).
 *   - Kernels never read past a tensor's logical end: tile loads past an edge are clipped and
 *     zero-filled by TMA, and stores are predicated (the same page's notes on speculative
 *     reads past the logical sequence).
 *   - Concurrency: calls from several host threads, or on several streams, may overlap; no two
 *     of them share scratch memory (k_smooth_mean_noalloc excepted: see there), and the
 *     library's per-device caches are atomics. Two things are shared by every attention launch
 *     on a device: the device error word -- attn_debug_status() reports and clears a
 *     bounded-wait timeout from whichever launch set it -- and the failure test that
 *     attn_debug_starve() arms, which applies to the next attention launch of the process,
 *     whatever thread makes it.
 */
#ifndef B200ATTN_H
#define B200ATTN_H

#include <stdint.h>

#if defined(__GNUC__)
#define B200ATTN_API __attribute__((visibility("default")))
#else
#define B200ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum b200attn_status {
    B200ATTN_OK = 0,
    B200ATTN_ERR_NULL = 1,     /* a required pointer is NULL for a non-empty tensor */
    B200ATTN_ERR_SHAPE = 2,    /* a size is negative, or hk <= 0 / sk < 0 */
    B200ATTN_ERR_GQA = 3,      /* hq is not a multiple of hk */
    B200ATTN_ERR_HEADDIM = 4,  /* (dqk, dv) not in {(64,64),(128,128),(192,128),(256,256)}
                                  ((128,128) only for attn_fwd_fp8); for the K mean and
                                  fp8_quantize, d not in {64, 128, 256} */
    B200ATTN_ERR_ALIGN = 5,    /* a pointer below its required alignment: 16 bytes for bf16
                                  and E4M3 tensors and the K mean, 4 bytes for LSE, sinks
                                  and descales */
    B200ATTN_ERR_RANGE = 6,    /* a size, byte extent or stride overflows int64 or TMA limits */
    B200ATTN_ERR_SCALE = 7,    /* scale is NaN or infinite */
    B200ATTN_ERR_ARCH = 8,     /* the current device is not compute capability 10.0 (sm_100) */
    B200ATTN_ERR_CUDA = 9,     /* a CUDA runtime / driver call or a kernel launch failed */
    B200ATTN_ERR_TIMEOUT = 10, /* a kernel gave up on a bounded wait (see attn_debug_status) */
    B200ATTN_ERR_SCRATCH = 11, /* b*hk*d exceeds the fixed scratch of k_smooth_mean_noalloc */
};

/*
 * attn_fwd -- fused attention forward pass with per-row log-sum-exp.
 *
 * Computes, for every batch bi < b, query head h < hq, query row i < sq, with kv head
 * g = h / (hq / hk) (consecutive query heads share a kv head; grouped-query attention):
 *     J = { j < sk : causal == 0  or  j <= i + sk - sq }       (bottom-right causal alignment)
 *     s_j = scale * <Q[bi,i,h,:], K[bi,j,g,:]>
 *     O[bi,i,h,:] = sum_{j in J} softmax_J(s)_j * V[bi,j,g,:]        (rounded to bf16, RNE)
 *     LSE[bi,h,i] = log(sum_{j in J} exp(s_j))                       (fp32, natural log)
 * A row with an empty J (causal with i < sq - sk) gets O = 0 and LSE = -inf.
 * This is the multi-head attention forward pass that the Triton "_attn_fwd" kernel of
 * "Tune MHA config & small-head pipeline pathology" computes (Motivation; shape notation
 * M = sq, N = sk, K = d_head_qk, d_v, HQ/HK and causal c0/c1 in "Source of shapes" and the
 * tables after Final status); the pages do not write the formula, and this is its standard
 * reading.
 *
 *   q, k, v  device bf16, 16-byte aligned, shapes as above. Read only.
 *   out      device bf16 [b, sq, hq, dv], 16-byte aligned. Fully written.
 *   lse      device fp32 [b, hq, sq], 4-byte aligned, or NULL to skip the LSE.
 *   b, hq, sq  may be 0 (nothing is launched). sk may be 0 (every row is empty).
 *   hk       > 0, hq % hk == 0.
 *   dqk, dv  one of (64,64), (128,128), (192,128), (256,256).
 *   causal   0 or nonzero.
 *   scale    finite; usually 1/sqrt(dqk).
 * Allocates nothing. Concurrency as in the conventions above.
 */
B200ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
             int64_t b, int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
             int causal, float scale, void* stream);

/*
 * attn_fwd_window_sink -- attn_fwd with a sliding window and per-head attention sinks.
 *
 * As attn_fwd, with two changes to each row's softmax (the "GPT-OSS sink+sliding-window" shapes
 * named in "Tune MHA config & small-head pipeline pathology", Source of shapes; the pages define
 * neither, and this is the usual reading):
 *     window   J additionally keeps only keys j >= i + sk - sq - window_left (the row's
 *              diagonal key and the window_left keys before it); window_left < 0: no window.
 *     sinks    fp32 [hq] logits (in the units of scale * <q, k>), or NULL. sigma_h joins the
 *              denominator without a value:  m = max(max_J s_j, sigma_h),
 *              O = sum_J exp(s_j - m) V_j / (exp(sigma_h - m) + sum_J exp(s_j - m)),
 *              LSE = log(exp(sigma_h) + sum_J exp(s_j)); an empty J gives O = 0, LSE = sigma_h.
 * Key blocks left of every row's window are never loaded or multiplied.
 *
 *   sinks    device fp32, 4-byte aligned, or NULL. Read only.
 *   other arguments, layouts, errors, allocation and concurrency as in attn_fwd.
 */
B200ATTN_API int attn_fwd_window_sink(const void* q, const void* k, const void* v, void* out,
                                      float* lse, const float* sinks, int64_t b, int64_t hq,
                                      int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
                                      int causal, int64_t window_left, float scale, void* stream);

/*
 * attn_fwd_varlen -- attn_fwd over b packed sequences of different lengths.
 *
 * Sequence i (i < b) owns query rows cu_seqlens_q[i] .. cu_seqlens_q[i+1]-1 of q / out and key
 * rows cu_seqlens_k[i] .. cu_seqlens_k[i+1]-1 of k / v; with sq_i, sk_i its lengths, every
 * query row r = i0 + i of it gets attn_fwd's result for its own sequence alone (same J with
 * sq_i, sk_i in place of sq, sk -- bottom-right causal alignment per sequence; an empty J
 * gives O = 0, LSE = -inf). This is the "varlen" layout of the shape tables of "Tune MHA config
 * & small-head pipeline pathology" (Source of shapes; the varlen rows after Final status),
 * which print no packing convention; this is the usual one (cumulative offsets, one entry per
 * sequence boundary).
 *
 *   q        device bf16 [total_q, hq, dqk];  k: [total_k, hk, dqk];  v: [total_k, hk, dv].
 *   out      device bf16 [total_q, hq, dv]. Rows of every sequence are written; rows that
 *            belong to no sequence are left unchanged.
 *   lse      device fp32 [hq, total_q] (head-major), or NULL.
 *   cu_seqlens_q, cu_seqlens_k  device int32 [b + 1], 4-byte aligned, non-decreasing row
 *            offsets into the packed tensors (usually 0 .. total_q / total_k; rows outside
 *            [cu[0], cu[b]) belong to no sequence). Read by the kernel only (the host never
 *            dereferences them). Offsets outside [0, total] are clamped into it, so no row
 *            outside the tensors is ever addressed.
 *   max_sq   at least the longest query length (it sizes the grid); query rows of a sequence
 *            beyond max_sq are not computed.
 *   b, total_q, max_sq  may be 0 (nothing is launched); total_k may be 0 (every row empty).
 *   hk, hq, dqk, dv, causal, scale  as in attn_fwd.
 * Errors as attn_fwd; also ERR_RANGE when total_q, total_k or b * hq * ceil(max_sq / 128)
 * reaches 2^31. Allocates nothing. Concurrency as in the conventions above.
 */
B200ATTN_API int attn_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                 int64_t b, int64_t hq, int64_t hk, int64_t total_q,
                                 int64_t total_k, int64_t max_sq, int64_t dqk, int64_t dv,
                                 int causal, float scale, void* stream);

/*
 * k_smooth_mean -- fp32 channel mean of K over its sequence axis.
 *     mean[bi,g,c] = (1/sk) * sum_{s < sk} K[bi,s,g,c]
 * The per-(batch, head) moments of K over its key axis, folded per head in a fixed order, that
 * "[HIP] Mha v4: run the K-smoothing gate as one HIP call" computes in two deterministic kernels
 * behind one host call (Summary; commit message). Here the sample is every key and no gate is
 * applied. Sums run in fp32 over sequence chunks, then the chunk partials are folded in a fixed
 * order, so repeated calls give bit-identical results. One launch: when K has many (batch,
 * 8-channel group) pairs, each CTA sums its own pairs over every key (no cross-CTA fold, no
 * scratch); otherwise the sums over key chunks and their fold are two phases of one cooperative
 * launch with a bounded grid-wide wait between them (a wait that runs out sets the error word
 * read by attn_debug_status).
 *
 *   k     device bf16 [b, sk, hk, d], 16-byte aligned.
 *   mean  device fp32 [b, hk, d], 16-byte aligned. Fully written.
 *   d     64, 128 or 256 (the head dims the page's host check accepts). sk > 0.
 * Takes its partial-sum scratch (b * hk * d * chunks floats, at most 4 MiB per 1024 channels)
 * from a library-owned stream-ordered memory pool on `stream` and frees it on the same stream,
 * so concurrent calls on different streams never share scratch. The pool keeps freed memory for
 * later calls (it is created on the first call on a device and lives until the process exits).
 */
B200ATTN_API int k_smooth_mean(const void* k, float* mean, int64_t b, int64_t hk, int64_t sk, int64_t d,
                  void* stream);

/*
 * k_smooth_mean_noalloc -- k_smooth_mean for callers that must not allocate device memory.
 *
 * No counterpart on the reference pages: this entry point exists for callers that cannot let a
 * library allocate during a call -- for example a serving process that reserves all device
 * memory for its own pool at start-up (so a cudaMallocAsync inside the call could fail, or
 * stall the stream while the driver maps memory), or code that must keep its memory use fixed
 * and known in advance. It computes the same mean as k_smooth_mean with the same kernels; where
 * those fold partial sums, it takes them from a fixed file-scope device array of 2^20 floats
 * (4 MiB) that
 * every GPU which loads this library holds until the process exits. It never calls cudaMalloc,
 * cudaFree or any allocating routine.
 *
 *   Arguments, layout and alignment as for k_smooth_mean.
 *   Limit: b * hk * d <= 2^20 (one fp32 partial row per batch must fit); larger problems are
 *   refused with B200ATTN_ERR_SCRATCH before anything is launched. Long sequences are folded in
 *   fewer, longer chunks so that the partials always fit.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current; make that first call before any stream capture.
 *   Every call on a device shares the one array and leaves its contents behind: calls whose
 *   kernels overlap on the GPU (for example on two streams) race, so serialise them.
 */
B200ATTN_API int k_smooth_mean_noalloc(const void* k, float* mean, int64_t b, int64_t hk,
                                       int64_t sk, int64_t d, void* stream);

/*
 * k_smooth_mean_strided -- k_smooth_mean of a strided view of K: a slice of its heads or keys, a
 * view into a larger buffer, or one whose address or strides are not 16-byte aligned.
 *     mean[bi,g,c] = (1/sk) * sum_{s < sk} K(bi, s, g, c),
 *     K(bi, s, g, c) = k[bi*stride_b + s*stride_s + g*stride_h + c]   (bf16 elements)
 * "[HIP] Mha v4: run the K-smoothing gate as one HIP call" (PR Self-Review: PR-specific question;
 * Changed op tests; commit message): the op's host check takes BSHD K whose last dimension is
 * contiguous, misaligned views take a scalar-load path, and its test covers head-sliced and
 * misaligned K views. Here: when the view is the contiguous layout (stride_h = d,
 * stride_s = hk*d, stride_b = sk*hk*d) and k and mean are 16-byte aligned, this is
 * k_smooth_mean (same kernels, same bits). Otherwise two launches on `stream`: fp32 partial sums
 * per (batch, chunk of keys) with 2-byte loads, added in key order, then a fold of the chunks in
 * chunk order, so repeated calls give bit-identical results.
 *
 *   k         device bf16, 2-byte aligned; element (bi, s, g, c) as above. The channel stride
 *             is 1 (the page's contiguous last dimension).
 *   stride_b, stride_s, stride_h  element strides >= 0 (any values; views may overlap).
 *   mean      device fp32 [b, hk, d], 4-byte aligned. Fully written.
 *   d         64, 128 or 256. sk > 0.
 * Errors as for k_smooth_mean, plus B200ATTN_ERR_SHAPE for a negative stride and
 * B200ATTN_ERR_RANGE when the largest element offset of the view overflows int64. Scratch
 * (b * hk * d * chunks floats) from the library's stream-ordered pool, as k_smooth_mean.
 * Concurrency as in the conventions above.
 */
B200ATTN_API int k_smooth_mean_strided(const void* k, float* mean, int64_t b, int64_t hk,
                                       int64_t sk, int64_t d, int64_t stride_b, int64_t stride_s,
                                       int64_t stride_h, void* stream);

/*
 * k_smooth_gate -- the K-smoothing gate: sampled channel mean of K and a per-head decision.
 *
 * "[HIP] Mha v4: run the K-smoothing gate as one HIP call" (Summary, commit message) runs the
 * gate as per-(batch*head, chunk) moments over a strided sample of the keys, then a per-head
 * fold and the gate, as two deterministic kernels behind one call; it prints neither the stride
 * nor the threshold. Reading:
 *     sample   keys s = 0, stride, 2*stride, ... < sk, stride = ceil(sk / 2048) (every key when
 *              sk <= 2048); n sampled keys
 *     mu[bi,g,c] = (1/n) sum_s K[bi,s,g,c],   e[bi,g,c] = (1/n) sum_s K[bi,s,g,c]^2
 *     ratio[bi,g] = sum_c mu^2 / sum_c e   (the share of K's energy in its channel mean; 0 when
 *                                           the sampled K is all zero)
 *     gate[bi,g] = ratio >= threshold
 *     mean[bi,g,c] = gate ? mu : 0   (fp32; feed it to k_smooth_sub: where the gate is off,
 *                                     K' = K)
 * All sums in fp32 in a fixed order: the outputs are bit-identical from run to run. The two
 * steps run as phases of one cooperative launch with a bounded grid-wide wait between them.
 *
 *   k          device bf16 [b, sk, hk, d], 16-byte aligned. Read only.
 *   mean       device fp32 [b, hk, d], 16-byte aligned. Fully written.
 *   gate       device int32 [b, hk] (0 / 1), 4-byte aligned. Fully written.
 *   ratio      device fp32 [b, hk], 4-byte aligned, or NULL. Fully written when given.
 *   threshold  finite (NaN / inf -> ERR_SCALE).
 *   b, hk, sk, d  as in k_smooth_mean (sk > 0, d in {64, 128, 256}).
 * Scratch: taken from and returned to a library-owned stream-ordered memory pool on `stream`
 * (as k_smooth_mean). Concurrency as in the conventions above.
 */
B200ATTN_API int k_smooth_gate(const void* k, float* mean, int32_t* gate, float* ratio, int64_t b,
                               int64_t hk, int64_t sk, int64_t d, float threshold, void* stream);

/*
 * k_smooth_sub -- subtract the channel mean from K: k_out = bf16_rne(float(K) - mean),
 * with mean[bi,g,c] broadcast over the sequence axis. This makes the smoothed K that the
 * attention pass then reads ("mean subtracted before attention"). k_out must not overlap k.
 *
 *   k, k_out  device bf16 [b, sk, hk, d], 16-byte aligned.   mean  device fp32 [b, hk, d],
 *             16-byte aligned.
 * Allocates nothing.
 */
B200ATTN_API int k_smooth_sub(const void* k, const float* mean, void* k_out, int64_t b, int64_t hk,
                 int64_t sk, int64_t d, void* stream);

/*
 * k_smooth_mean_sub -- k_smooth_mean and k_smooth_sub in one launch: the K channel mean and the
 * smoothed K' = bf16_rne(float(K) - mean) that the attention pass then reads. Bit-identical to
 * k_smooth_mean followed by k_smooth_sub with that mean. The cooperative launch sums the key
 * chunks, folds the mean, and then writes K'. It re-reads K from L2 when K fits there.
 *
 *   k      device bf16 [b, sk, hk, d], 16-byte aligned. Read only.
 *   mean   device fp32 [b, hk, d], 16-byte aligned. Fully written.
 *   k_out  device bf16 [b, sk, hk, d], 16-byte aligned. Fully written. Must not overlap k or mean.
 *   b, hk, sk, d  as in k_smooth_mean (sk > 0, d in {64, 128, 256}).
 * Scratch: taken from and returned to a library-owned stream-ordered memory pool on `stream`
 * (as k_smooth_mean). Concurrency as in the conventions above.
 */
B200ATTN_API int k_smooth_mean_sub(const void* k, float* mean, void* k_out, int64_t b, int64_t hk,
                                   int64_t sk, int64_t d, void* stream);

/*
 * fp8_quantize -- E4M3 codes of a bf16 BSHD tensor with one fp32 scale per (batch, head), for the
 * FP8 attention recipe ("[HIP] Mha v4: run the K-smoothing gate as one HIP call", Summary: the
 * quantized recipes apply the K-smoothing gate before quantizing K; "Tune MHA config &
 * small-head pipeline pathology", the FP8 rows after Final status). The pages give neither the
 * quantisation nor the scale layout. Reading (per-head amax scaling, OCP E4M3):
 *     x'      = mean ? fp32(x - mean[bi,hh,c]) : x          (one fp32 subtraction, RNE)
 *     amax    = max |x'| over the head's [s, d] slice
 *     descale[bi,hh] = amax > 0 ? fp32(amax / 448) : 1
 *     code    = E4M3_satfinite_rne(fp32(x' * f)),  f = amax > 0 ? min(fp32(448 / amax), FLT_MAX) : 1
 * E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormals, no infinities, largest
 * finite 448; ties round to the even code; magnitudes past 448 saturate. The codes are exact
 * (bit-identical to any correct implementation of these steps) and deterministic.
 *
 *   x         device bf16 [b, s, h, d], 16-byte aligned, finite. Read only.
 *   mean      device fp32 [b, h, d], 16-byte aligned (K smoothing: the output of k_smooth_mean or
 *             k_smooth_gate), or NULL.
 *   x8        device uint8 [b, s, h, d], 16-byte aligned. Fully written. Must not overlap x.
 *   descale   device fp32 [b, h], 4-byte aligned. Fully written.
 *   b, h      >= 0 (0: nothing to do);  s >= 0 (0: every descale is 1);  d in {64, 128, 256}.
 * Scratch: taken from and returned to a library-owned stream-ordered memory pool on `stream`.
 * One cooperative launch (per-chunk amax, a grid-wide wait, then fold and convert). Concurrency
 * as in the conventions above.
 */
B200ATTN_API int fp8_quantize(const void* x, const float* mean, void* x8, float* descale,
                              int64_t b, int64_t s, int64_t h, int64_t d, void* stream);

/*
 * attn_fwd_fp8 -- attn_fwd on E4M3 inputs with per-(batch, head) descales (the FP8 recipe; see
 * fp8_quantize for the format and the scale reading).
 *
 * Computes attn_fwd's O and LSE for the decoded inputs
 *     Q = code * q_descale[bi,h],  K = code * k_descale[bi,g],  V = code * v_descale[bi,g].
 * Q K^T and P V run as E4M3 tensor-core products with fp32 accumulation. The descales of Q and
 * K fold into the exp2 factor, and that of V into the final division. The softmax weights P
 * are rounded to E4M3 for the P V product; the row sums keep the unrounded weights. Per output
 * element this moves O by at most (2^-4 sum_j w_j |V_jc| + 2^-10 sum_j |V_jc|) / sum_j w_j
 * (w_j = exp(s_j - max s)) beyond attn_fwd's own rounding. LSE is as in attn_fwd.
 *
 *   q8       device uint8 [b, sq, hq, dqk];  k8: [b, sk, hk, dqk];  v8: [b, sk, hk, dv];
 *            16-byte aligned, E4M3 codes (no NaN codes). Read only.
 *   q_descale  device fp32 [b, hq];  k_descale, v_descale: [b, hk]; 4-byte aligned, positive
 *            and finite. The exp2 factor |scale| * log2(e) * q_descale * k_descale is kept at
 *            2^-100 or more, as attn_fwd keeps its own (the sign of scale is applied by the MMA).
 *   out, lse as in attn_fwd (O in bf16).
 *   dqk, dv  (128, 128) only (else B200ATTN_ERR_HEADDIM).
 *   other arguments, errors, allocation and concurrency as in attn_fwd.
 */
B200ATTN_API int attn_fwd_fp8(const void* q8, const void* k8, const void* v8,
                              const float* q_descale, const float* k_descale,
                              const float* v_descale, void* out, float* lse, int64_t b,
                              int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk,
                              int64_t dv, int causal, float scale, void* stream);

/* Static description of a status code (never NULL). */
B200ATTN_API const char* attn_status_string(int status);

/*
 * attn_debug_status -- synchronise `stream`, then return and clear the device-side error word
 * that kernels set when a bounded wait gives up (B200ATTN_ERR_TIMEOUT) instead of hanging.
 * Returns B200ATTN_OK when no kernel has reported an error since the last call on this device.
 */
B200ATTN_API int attn_debug_status(void* stream);

/*
 * attn_debug_starve -- failure test of the bounded waits (no counterpart on the pages; their
 * stalls were found by timing only). Arms the next attention launch of this process (any entry
 * point, any stream) so that its TMA producer loads nothing and every wait of the other roles is
 * limited to timeout_us: they all give up, leave through the abort path (in-flight work drained,
 * tensor memory freed), the launch completes, and attn_debug_status then reports
 * B200ATTN_ERR_TIMEOUT. The device and its context stay usable; the launch's outputs are
 * undefined. No fault, trap or hang is involved.
 *   timeout_us  1 .. 1000000 (else B200ATTN_ERR_RANGE).
 */
B200ATTN_API int attn_debug_starve(int64_t timeout_us);

#ifdef __cplusplus
}
#endif

#endif /* B200ATTN_H */
