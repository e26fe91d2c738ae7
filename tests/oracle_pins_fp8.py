"""Pins of the FP8 (E4M3) oracle module against what does not come from it: torch's own
float8_e4m3fn conversion (an independent implementation of the same format), closed forms of
the OCP E4M3 definition, the already pinned bf16 attention oracle on exactly representable
inputs, and a brute-force softmax. Each pin takes the module under test (the real oracle.fp8
or a copy with a planted mistake) and raises AssertionError when it disagrees."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Closed forms of the E4M3 definition: 1.0, the largest finite value, the smallest subnormal,
# the smallest normal, the largest subnormal, negative zero, -1.75, and 2^-3.
KNOWN = {0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0x07: 7 * 2.0 ** -9,
         0x80: -0.0, 0xBE: -1.75, 0x20: 0.125}


def torch_decode(codes) -> np.ndarray:
    c = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return c.view(torch.float8_e4m3fn).float().double().numpy()


def torch_encode(y) -> np.ndarray:
    """torch's round-to-nearest-even cast (valid for |y| <= 464, where it does not overflow)."""
    t = torch.from_numpy(np.ascontiguousarray(y, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_decode_matches_torch(f):
    c = np.arange(256, dtype=np.uint8)
    d, t = f.e4m3_decode(c), torch_decode(c)
    nan = np.isnan(t)
    assert np.array_equal(np.isnan(d), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(d[~nan], t[~nan])
    assert np.array_equal(np.signbit(d[~nan]), np.signbit(t[~nan]))


def pin_decode_closed_forms(f):
    for code, val in KNOWN.items():
        got = float(f.e4m3_decode(np.array([code], dtype=np.uint8))[0])
        assert got == val and np.signbit(got) == np.signbit(val), (hex(code), got, val)


def pin_encode_matches_torch(f):
    rng = np.random.default_rng(11)
    y = (rng.standard_normal(100000) * np.exp2(rng.uniform(-16, 9, 100000))).astype(np.float32)
    y = y[np.abs(y) <= 464]
    assert np.array_equal(f.e4m3_encode(y), torch_encode(y))
    # every finite value maps to its own code, and every midpoint between neighbours to the
    # neighbour with the even code (ties to even), for both signs
    pos = torch_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.array_equal(f.e4m3_encode(pos), np.arange(0x7F, dtype=np.uint8))
    mid = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (pos[:-1] + pos[1:]) / 2)  # exact in fp32
    want = np.where(np.arange(0x7E) % 2 == 0, np.arange(0x7E), np.arange(1, 0x7F)).astype(np.uint8)
    assert np.array_equal(f.e4m3_encode(mid), want)
    assert np.array_equal(f.e4m3_encode(-mid), want | 0x80)
    assert np.array_equal(torch_encode(mid), want)


def pin_encode_saturates_and_keeps_sign(f):
    big = np.array([448.0, 460.0, 465.0, 1e6, 3.0e38], dtype=np.float32)
    assert np.array_equal(f.e4m3_encode(big), np.full(5, 0x7E, dtype=np.uint8))
    assert np.array_equal(f.e4m3_encode(-big), np.full(5, 0xFE, dtype=np.uint8))
    tiny = np.array([0.0, -0.0, 2.0 ** -11, -(2.0 ** -11), 2.0 ** -10, -(2.0 ** -10)], dtype=np.float32)
    assert f.e4m3_encode(tiny).tolist() == [0x00, 0x80, 0x00, 0x80, 0x00, 0x80]


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def pin_quantize_bound_and_amax(f):
    b, s, h, d = 2, 96, 3, 64
    rng = np.random.default_rng(12)
    x = rng.standard_normal((b, s, h, d)) * np.array([1.0, 30.0, 1e-3]).reshape(1, 1, h, 1)
    x[1, :, 2, :] = 0.0  # an all-zero head slice
    bits = _bf16_bits(x)
    xv = oracle.bf16_to_f64(bits).reshape(b, s, h, d)
    codes, ds = f.quantize(bits, b, s, h, d)
    assert codes.shape == (b, s, h, d) and codes.dtype == np.uint8
    assert ds.shape == (b, h) and ds.dtype == np.float32
    amax = np.abs(xv).max(axis=(1, 3))
    nz = amax > 0
    assert np.all(ds[~nz] == 1.0) and np.all(codes[1, :, 2, :] == 0)
    # descale = amax / 448 up to one fp32 rounding
    assert np.all(np.abs(ds[nz] - amax[nz] / 448.0) <= amax[nz] / 448.0 * 2.0 ** -23)
    # reconstruction: one E4M3 rounding (half a step: 2^-4 relative, 2^-10 absolute below the
    # normal range) of x / descale, plus fp32 roundings of the factor and the product
    dec = torch_decode(codes) * ds.astype(np.float64).reshape(b, 1, h, 1)
    dsb = ds.astype(np.float64).reshape(b, 1, h, 1)
    bound = np.abs(xv) * (2.0 ** -4 + 2.0 ** -20) + dsb * 2.0 ** -10
    assert np.all(np.abs(dec - xv) <= bound)
    # each head's largest magnitude lands on +-448
    for bi in range(b):
        for hh in range(h):
            if not nz[bi, hh]:
                continue
            sl = xv[bi, :, hh, :]
            idx = np.unravel_index(np.argmax(np.abs(sl)), sl.shape)
            assert codes[bi, idx[0], hh, idx[1]] & 0x7F == 0x7E


def pin_quantize_codes_match_torch(f):
    # the codes are torch's E4M3 cast of fp32(x * fp32(448 / amax))
    b, s, h, d = 1, 64, 2, 128
    rng = np.random.default_rng(13)
    x = rng.standard_normal((b, s, h, d)) * 3.0
    bits = _bf16_bits(x)
    codes, ds = f.quantize(bits, b, s, h, d)
    xt = torch.from_numpy(oracle.bf16_to_f64(bits).reshape(b, s, h, d)).float()
    amax = xt.abs().amax(dim=(1, 3))
    inv = torch.tensor(448.0, dtype=torch.float32) / amax
    y = (xt * inv.reshape(b, 1, h, 1)).numpy()
    assert np.array_equal(codes, torch_encode(y))


def pin_quantize_mean_shift(f):
    # x + c with a per-(batch, head, channel) shift c, all exactly representable: subtracting
    # mean = c must give back exactly the codes of x
    b, s, h, d = 2, 40, 2, 64
    rng = np.random.default_rng(14)
    x = rng.integers(-64, 65, size=(b, s, h, d)) * 2.0 ** -6
    c = rng.choice([2.0, 3.0, -3.0, -2.5, 2.25], size=(b, h, d))
    shifted = x + c[:, None, :, :]
    bits_x, bits_s = _bf16_bits(x), _bf16_bits(shifted)
    assert np.array_equal(oracle.bf16_to_f64(bits_s).reshape(b, s, h, d), shifted)
    c0, d0 = f.quantize(bits_x, b, s, h, d)
    c1, d1 = f.quantize(bits_s, b, s, h, d, mean32=c.astype(np.float32))
    assert np.array_equal(c0, c1) and np.array_equal(d0, d1)


def _codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    return np.where((c & 0x7F) == 0x7F, c & 0xF0, c).astype(np.uint8)  # no NaN codes


def pin_attention_equals_bf16_oracle(f, lib=None):
    # power-of-two descales: every decoded value is exact in bf16, so the FP8 attention must be
    # the (separately pinned) bf16 oracle on those values
    b, hq, hk, sq, sk, dqk, dv = 2, 4, 2, 40, 56, 64, 64
    rng = np.random.default_rng(15)
    q8, k8, v8 = _codes(rng, (b, sq, hq, dqk)), _codes(rng, (b, sk, hk, dqk)), _codes(rng, (b, sk, hk, dv))
    dq = np.exp2(rng.integers(-7, -3, size=(b, hq))).astype(np.float32)
    dk = np.exp2(rng.integers(-7, -3, size=(b, hk))).astype(np.float32)
    dvv = np.exp2(rng.integers(-6, -2, size=(b, hk))).astype(np.float32)
    qv = torch_decode(q8) * dq.reshape(b, 1, hq, 1)
    kv = torch_decode(k8) * dk.reshape(b, 1, hk, 1)
    vv = torch_decode(v8) * dvv.reshape(b, 1, hk, 1)
    for causal in (False, True):
        o, lse = f.attn_full(q8, k8, v8, dq, dk, dvv, b, hq, hk, sq, sk, dqk, dv, causal, 0.3,
                             lib=lib)
        o_ref, lse_ref = oracle.attn_full(_bf16_bits(qv), _bf16_bits(kv), _bf16_bits(vv), b, hq,
                                          hk, sq, sk, dqk, dv, causal, 0.3, lib=lib)
        assert np.allclose(o, o_ref, rtol=0, atol=1e-12)
        assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)


def pin_attention_brute_force(f, lib=None):
    # arbitrary descales: numpy full-matrix softmax over torch-decoded values
    b, hq, hk, sq, sk, dqk, dv = 1, 6, 2, 24, 33, 128, 128
    rng = np.random.default_rng(16)
    q8, k8, v8 = _codes(rng, (b, sq, hq, dqk)), _codes(rng, (b, sk, hk, dqk)), _codes(rng, (b, sk, hk, dv))
    dq = rng.uniform(0.001, 0.01, size=(b, hq)).astype(np.float32)
    dk = rng.uniform(0.001, 0.01, size=(b, hk)).astype(np.float32)
    dvv = rng.uniform(0.01, 0.1, size=(b, hk)).astype(np.float32)
    qv = torch_decode(q8) * dq.astype(np.float64).reshape(b, 1, hq, 1)
    kv = torch_decode(k8) * dk.astype(np.float64).reshape(b, 1, hk, 1)
    vv = torch_decode(v8) * dvv.astype(np.float64).reshape(b, 1, hk, 1)
    rows = np.array([[0, h, i] for h in range(hq) for i in (0, 7, sq - 1)])
    scale = 1.0 / np.sqrt(dqk)
    o, lse = f.attn_rows(q8, k8, v8, dq, dk, dvv, b, hq, hk, sq, sk, dqk, dv, True, scale, rows,
                         lib=lib)
    for r, (bi, h, i) in enumerate(rows):
        g = h // (hq // hk)
        n = i + sk - sq + 1
        s = scale * (kv[bi, :n, g, :] @ qv[bi, i, h, :])
        m = s.max()
        w = np.exp(s - m)
        assert np.allclose(o[r], (w @ vv[bi, :n, g, :]) / w.sum(), rtol=0, atol=1e-12)
        assert abs(lse[r] - (m + np.log(w.sum()))) <= 1e-12


ALL_PINS = [pin_decode_matches_torch, pin_decode_closed_forms, pin_encode_matches_torch,
            pin_encode_saturates_and_keeps_sign, pin_quantize_bound_and_amax,
            pin_quantize_codes_match_torch, pin_quantize_mean_shift,
            pin_attention_equals_bf16_oracle, pin_attention_brute_force]
