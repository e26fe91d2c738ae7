"""The FP8 (E4M3) oracle against its pins, a mutation check of those pins, and the accuracy
property that motivates K smoothing before quantisation (CPU only)."""
import importlib.util
import os
import sys

import numpy as np
import pytest

import oracle
from oracle import fp8
from oracle_pins_fp8 import ALL_PINS, _bf16_bits

import workloads


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_fp8_oracle_pin(pin):
    pin(fp8)


# Plausible mistakes in the FP8 module; each must fail at least one pin.
MUTANTS = {
    "exponent_bias_8": ("np.exp2(e - 7.0)", "np.exp2(e - 8.0)"),
    "subnormal_scale": ("m / 8.0 * 2.0 ** -6", "m / 8.0 * 2.0 ** -7"),
    "ties_away_from_zero": ("(d_hi == d_lo) & (hi % 2 == 0)", "(d_hi == d_lo)"),
    "zero_loses_sign": ("np.where(np.signbit(y), 0x80, 0)", "np.where(y < 0, 0x80, 0)"),
    "descale_inverted": ("amax / np.float32(E4M3_MAX), np.float32(1)",
                         "np.float32(E4M3_MAX) / np.where(pos, amax, np.float32(1)), np.float32(1)"),
    "mean_added": ("x = np.subtract(x, m, dtype=np.float32)", "x = np.add(x, m, dtype=np.float32)"),
    "v_descale_dropped": ("v = _f64(dequantize(v8, v_descale, b, sk, hk, dv))\n    o = np.zeros((b, sq",
                          "v = _f64(dequantize(v8, np.ones_like(v_descale), b, sk, hk, dv))\n    o = np.zeros((b, sq"),
    "k_descale_from_q": ("k = _f64(dequantize(k8, k_descale, b, sk, hk, dqk))\n    v = _f64(dequantize(v8, v_descale, b, sk, hk, dv))\n    return attn_rows_decoded",
                         "k = _f64(dequantize(k8, q_descale[:, :hk], b, sk, hk, dqk))\n    v = _f64(dequantize(v8, v_descale, b, sk, hk, dv))\n    return attn_rows_decoded"),
}


def _load_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(fp8.__file__).read()
    assert src.count(old) == 1, f"mutation anchor not found: {old}"
    path = tmp_path / f"fp8_{name}.py"
    path.write_text(src.replace(old, new))
    mod_name = f"oracle._fp8_mutant_{name}"
    spec = importlib.util.spec_from_file_location(mod_name, str(path))
    mod = importlib.util.module_from_spec(spec)
    sys.modules[mod_name] = mod
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.modules.pop(mod_name, None)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8_pins_catch_planted_mistake(tmp_path, name):
    mod = _load_mutant(tmp_path, name)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"


def test_k_smoothing_reduces_fp8_error():
    """With per-channel offsets in K (the K-mean workload's recipe), quantising K' = K - mean
    instead of K shrinks the logit error that K's codes cause: the offsets set K's amax, so
    without smoothing the codes spend their range on them. Subtracting the mean moves each
    row's logits by one constant, which the softmax ignores, so the error is measured against
    the matching exact logits. The attention output is no worse either."""
    b, hq, hk, s, d = 1, 2, 2, 256, 128
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, d, d, seed=321, kmean=True)
    qb, kb, vb = (workloads.bf16_bits(t) for t in (q, k, v))
    qv = oracle.bf16_to_f64(qb).reshape(b, s, hq, d)
    kv = oracle.bf16_to_f64(kb).reshape(b, s, hk, d)
    scale = 1.0 / np.sqrt(d)
    o_ref, _ = oracle.attn_full(qb, kb, vb, b, hq, hk, s, s, d, d, False, scale)
    q8, dq = fp8.quantize(qb, b, s, hq, d)
    v8, dv = fp8.quantize(vb, b, s, hk, d)
    logit_rms, o_err = {}, {}
    for smooth in (False, True):
        mean32 = oracle.k_mean(kb, b, hk, s, d)[1] if smooth else None
        k8, dk = fp8.quantize(kb, b, s, hk, d, mean32=mean32)
        exact = kv - (mean32.astype(np.float64)[:, None] if smooth else 0.0)
        dk_err = fp8.dequantize(k8, dk, b, s, hk, d) - exact  # [b, s, hk, d]
        e = scale * np.einsum("bihc,bjhc->bhij", qv, dk_err)  # hq == hk here
        logit_rms[smooth] = float(np.sqrt(np.mean(e ** 2)))
        o, _ = fp8.attn_full(q8, k8, v8, dq, dk, dv, b, hq, hk, s, s, d, d, False, scale)
        o_err[smooth] = float(np.max(np.abs(o - o_ref)))
    assert logit_rms[True] < 0.7 * logit_rms[False], logit_rms
    assert o_err[True] <= o_err[False], o_err


def test_quantize_edge_shapes():
    # one row, and a zero-length sequence: descale 1, no codes
    for s in (1, 0):
        x = np.full((1, s, 2, 64), 0.5)
        codes, ds = fp8.quantize(_bf16_bits(x), 1, s, 2, 64)
        assert codes.shape == (1, s, 2, 64)
        if s:
            assert np.all(codes == 0x7E) and np.allclose(ds, 0.5 / 448, rtol=2 ** -23)
        else:
            assert np.all(ds == 1.0)


def test_p_rounding_bound_holds_for_emulated_rounding():
    """Emulate the rounding the bound covers -- weights against a stale reference r <= m,
    rounded to E4M3 (torch's cast), row sum from the unrounded weights -- and check the bound."""
    import torch

    b, hq, hk, sq, sk, d = 1, 2, 1, 48, 48, 64
    rng = np.random.default_rng(17)
    q8, k8, v8 = (np.where((c & 0x7F) == 0x7F, 0, c).astype(np.uint8)
                  for c in (rng.integers(0, 256, size=sh) for sh in
                            [(b, sq, hq, d), (b, sk, hk, d), (b, sk, hk, d)]))
    dq, dk, dv = (np.full((b, n), 2.0 ** -6, dtype=np.float32) for n in (hq, hk, hk))
    rows = np.array([[0, h, i] for h in range(hq) for i in range(sq)])
    bound = fp8.p_rounding_bound(q8, k8, v8, dq, dk, dv, b, hq, hk, sq, sk, d, d, True, 0.4, rows)
    o_exact, _ = fp8.attn_rows(q8, k8, v8, dq, dk, dv, b, hq, hk, sq, sk, d, d, True, 0.4, rows)
    q = fp8.dequantize(q8, dq, b, sq, hq, d)
    k = fp8.dequantize(k8, dk, b, sk, hk, d)
    v = fp8.dequantize(v8, dv, b, sk, hk, d)
    worst = 0.0
    for r, (_, h, i) in enumerate(rows):
        s = 0.4 * (k[0, : i + 1, 0, :] @ q[0, i, h, :]) * np.log2(np.e)
        for stale in (0.0, 3.5, 7.9):  # the reference may trail the maximum by up to 8
            p = np.exp2(s - (s.max() - stale))
            pr = torch.from_numpy(p.astype(np.float32)).to(torch.float8_e4m3fn).double().numpy()
            o = (pr @ v[0, : i + 1, 0, :]) / p.sum()
            err = np.abs(o - o_exact[r])
            assert np.all(err <= bound[r] * (1 + 1e-6) + 1e-12), (i, stale)
            worst = max(worst, float(np.max(err / np.maximum(bound[r], 1e-30))))
    assert worst > 0.05  # the bound is not vacuous
