"""FP8 (E4M3) attention recipe: codes, the per-head quantiser and attention over decoded inputs.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the tests, the smoke check and the
benchmark's CPU-baseline arm may import it. It shares no code with the CUDA library.

What the pages fix and what is read into them ("[HIP] Mha v4: run the K-smoothing gate as one HIP
call", Summary and the commit message; "Tune MHA config & small-head pipeline pathology", the
quantized recipes after Final status): the FP8 recipe runs attention on 8-bit E4M3 Q, K and V
and applies the K-smoothing gate before quantizing K. The pages do not give the quantisation
or the scale layout. The reading taken here is the plainest one:

  * E4M3 is the OCP 8-bit floating-point format (the "FN" variant): a sign bit, 4 exponent bits
    with bias 7 and 3 mantissa bits. Exponent field 0 holds subnormals (m/8) * 2^-6. S.1111.111
    is NaN. There are no infinities. The largest finite magnitude is 1.75 * 2^8 = 448.
  * One fp32 scale per (batch, head) of each tensor: descale = amax / 448 over the head's
    [s, d] slice. The codes are E4M3(x * (448 / amax)), rounded to nearest with ties to even
    and saturated to +-448 (448 / amax and the product are fp32 operations, rounded to
    nearest). An all-zero slice takes descale 1 and factor 1. A factor that overflows fp32 is
    clamped to the largest finite fp32.
  * K smoothing: with a channel mean given, each element is first replaced by
    fp32(K - mean), one fp32 subtraction rounded to nearest. Its amax and codes follow from
    that value.
  * The attention computes the bf16 definition of attn_oracle.c on the decoded values
    Q = code * q_descale[b, h], K = code * k_descale[b, g] and V = code * v_descale[b, g]. In
    fp64 these products are exact.

Parity: pinned by tests/test_oracle_fp8.py. Decoding is checked against torch's independent
float8_e4m3fn conversion for all 256 codes. Encoding is checked against the same conversion on
every midpoint and on random values, and against closed forms for saturation and signed zero.
The quantiser is checked against its error bound and the amax -> 448 rule. The attention is
checked against the pinned bf16 oracle on exactly representable inputs and against a
brute-force softmax.
"""
from __future__ import annotations

import numpy as np

from . import _ptr, default_threads, load_library

E4M3_MAX = 448.0
_F32_MAX = np.float32(np.finfo(np.float32).max)


def e4m3_decode(codes) -> np.ndarray:
    """fp64 value of each E4M3 code (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


# The 127 non-negative finite values in code order (codes 0x00 .. 0x7E), which is also
# ascending value order.
_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))


def e4m3_encode(y) -> np.ndarray:
    """E4M3 code of each finite value of y: nearest value, ties to the even code (the code's
    last bit is the mantissa's last bit), magnitudes past 448 saturated to 448, and the sign
    kept, also for zero."""
    y = np.asarray(y, dtype=np.float64)
    if not np.all(np.isfinite(y)):
        raise ValueError("e4m3_encode takes finite values")
    a = np.minimum(np.abs(y), E4M3_MAX)
    hi = np.searchsorted(_POS, a, side="left")  # first value >= a
    hi = np.minimum(hi, len(_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a == _POS[hi], hi, code)  # exact hits (also a = 0)
    return (code | np.where(np.signbit(y), 0x80, 0)).astype(np.uint8)


def _bf16_to_f32(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def quantize(x_bits, b, s, h, d, mean32=None):
    """Quantise a bf16 BSHD tensor [b, s, h, d] (raw bits) to E4M3 codes with one scale per
    (batch, head). Returns (codes uint8 [b, s, h, d], descale float32 [b, h]). mean32
    ([b, h, d] fp32) is subtracted first (K smoothing)."""
    x = _bf16_to_f32(x_bits).reshape(b, s, h, d)
    if mean32 is not None:
        m = np.ascontiguousarray(mean32, dtype=np.float32).reshape(b, 1, h, d)
        x = np.subtract(x, m, dtype=np.float32)
    if s == 0:
        amax = np.zeros((b, h), dtype=np.float32)
    else:
        amax = np.abs(x).max(axis=(1, 3)).astype(np.float32)  # [b, h]
    pos = amax > 0
    with np.errstate(divide="ignore", over="ignore"):
        inv = np.where(pos, np.float32(E4M3_MAX) / np.where(pos, amax, np.float32(1)),
                       np.float32(1)).astype(np.float32)
    inv = np.minimum(inv, _F32_MAX).astype(np.float32)
    descale = np.where(pos, amax / np.float32(E4M3_MAX), np.float32(1)).astype(np.float32)
    y = np.multiply(x, inv.reshape(b, 1, h, 1), dtype=np.float32)
    return e4m3_encode(y), descale


def dequantize(codes, descale, b, s, h, d) -> np.ndarray:
    """fp64 values code * descale[b, h] of a BSHD code tensor."""
    v = e4m3_decode(np.asarray(codes).reshape(b, s, h, d))
    return v * np.asarray(descale, dtype=np.float64).reshape(b, 1, h, 1)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def attn_full(q8, k8, v8, q_descale, k_descale, v_descale, b, hq, hk, sq, sk, dqk, dv, causal,
              scale, nthreads=None, lib=None):
    """O (fp64 [b, sq, hq, dv]) and LSE (fp64 [b, hq, sq]) of the attention definition on the
    decoded, descaled E4M3 inputs."""
    lib = lib or load_library()
    q = _f64(dequantize(q8, q_descale, b, sq, hq, dqk))
    k = _f64(dequantize(k8, k_descale, b, sk, hk, dqk))
    v = _f64(dequantize(v8, v_descale, b, sk, hk, dv))
    o = np.zeros((b, sq, hq, dv), dtype=np.float64)
    lse = np.zeros((b, hq, sq), dtype=np.float64)
    rc = lib.oracle_attn_full_f64(_ptr(q), _ptr(k), _ptr(v), b, hq, hk, sq, sk, dqk, dv,
                                  int(causal), float(scale), _ptr(o), _ptr(lse),
                                  int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_attn_full_f64 failed with code {rc}")
    return o, lse


def attn_rows(q8, k8, v8, q_descale, k_descale, v_descale, b, hq, hk, sq, sk, dqk, dv, causal,
              scale, rows, nthreads=None, lib=None):
    """O (fp64 [nrows, dv]) and LSE (fp64 [nrows]) for the (batch, head, query) triples in
    rows, on the decoded, descaled E4M3 inputs."""
    q = _f64(dequantize(q8, q_descale, b, sq, hq, dqk))
    k = _f64(dequantize(k8, k_descale, b, sk, hk, dqk))
    v = _f64(dequantize(v8, v_descale, b, sk, hk, dv))
    return attn_rows_decoded(q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale, rows,
                             nthreads=nthreads, lib=lib)


def attn_rows_decoded(q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale, rows, nthreads=None,
                      lib=None):
    """attn_rows on inputs already decoded by dequantize (fp64 BSHD arrays)."""
    lib = lib or load_library()
    q, k, v = _f64(q), _f64(k), _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.zeros((n, dv), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = lib.oracle_attn_rows_f64(_ptr(q), _ptr(k), _ptr(v), b, hq, hk, sq, sk, dqk, dv,
                                  int(causal), float(scale), _ptr(rows), n, _ptr(o), _ptr(lse),
                                  int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_attn_rows_f64 failed with code {rc}")
    return o, lse


def p_rounding_bound(q8, k8, v8, q_descale, k_descale, v_descale, b, hq, hk, sq, sk, dqk, dv,
                     causal, scale, rows) -> np.ndarray:
    """Per selected row and channel, a bound on how far O can move when each softmax weight is
    rounded to E4M3 before the P V product, while the row sum l keeps the unrounded weights.

    An implementation computes p_j = 2^(s_j log2(e) - r) for a reference r no larger than the
    row's maximum m (a lazily updated running maximum; p_j <= 2^8 then stays finite in E4M3).
    One E4M3 rounding of p_j errs by at most 2^-4 p_j in the normal range and 2^-10 below it.
    In units of the exact weights w_j = exp(s_j - m), with l = sum w_j, the error of O_c is
    therefore at most (2^-4 sum_j w_j |v_jc| + 2^-10 sum_j |v_jc|) / l. The bound does not
    include O's own rounding to bf16. Returns fp64 [nrows, dv]."""
    q = dequantize(q8, q_descale, b, sq, hq, dqk)
    k = dequantize(k8, k_descale, b, sk, hk, dqk)
    v = np.abs(dequantize(v8, v_descale, b, sk, hk, dv))
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    out = np.zeros((rows.shape[0], dv))
    group = hq // hk
    for r, (bi, h, i) in enumerate(rows):
        g = h // group
        n = min(sk, i + sk - sq + 1) if causal else sk
        if n <= 0:
            continue
        s = scale * (k[bi, :n, g, :] @ q[bi, i, h, :])
        w = np.exp(s - s.max())
        out[r] = (2.0 ** -4 * (w @ v[bi, :n, g, :]) + 2.0 ** -10 * v[bi, :n, g, :].sum(axis=0)) / w.sum()
    return out
