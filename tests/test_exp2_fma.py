"""Host-side check of the FMA-pipe exp2 used by the d64 softmax (exp2_fma_pair, sm100_ptx.cuh).

The kernel's constants are read from the header and the algorithm is replayed in fp32 with
numpy: every fp32 step rounds once, as the packed fp32x2 instructions do. The bound is the
minimax error of the cubic (1.0e-4 relative), far below the bf16 rounding of P (2^-9).
"""
import pathlib
import re

import numpy as np

HDR = pathlib.Path(__file__).resolve().parents[1] / "head_attention_forward_flash_b200" / "csrc" / "sm100_ptx.cuh"


def constants():
    text = HDR.read_text()
    c = {}
    for k in ("kExp2C1", "kExp2C2", "kExp2C3"):
        m = re.search(rf"constexpr float {k} = ([0-9.eE+-]+)f;", text)
        assert m, k
        c[k] = np.float32(float(m.group(1)))
    return c["kExp2C1"], c["kExp2C2"], c["kExp2C3"]


def f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def exp2_fma(x):
    c1, c2, c3 = constants()
    x = np.maximum(f32(x), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = f32(x.astype(np.float64) + np.float64(magic))
    r = f32(t.astype(np.float64) - np.float64(magic))
    f = f32(x.astype(np.float64) - r.astype(np.float64))
    q = f32(np.float64(c3) * f + np.float64(c2))
    q = f32(q.astype(np.float64) * f + np.float64(c1))
    q = f32(q.astype(np.float64) * f + 1.0)
    bits = (t.view(np.uint32).astype(np.uint64) << np.uint64(23)) + q.view(np.uint32).astype(np.uint64)
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-126.0, 12.0, 400001)
    y = exp2_fma(x).astype(np.float64)
    rel = np.abs(y / np.exp2(f32(x).astype(np.float64)) - 1.0)
    assert rel.max() < 1.1e-4, rel.max()


def test_integers_are_exact_powers_of_two():
    j = np.arange(-126, 13, dtype=np.float64)
    assert np.array_equal(exp2_fma(j).astype(np.float64), np.exp2(j))


def test_masked_and_tiny_arguments_give_zero():
    x = np.array([-np.inf, -1e30, -200.0, -127.5, -127.0], dtype=np.float64)
    y = exp2_fma(x)
    assert np.all(y.view(np.uint32) == 0)  # +0 exactly, as ex2.approx.ftz gives


def test_results_are_finite_and_positive_between():
    x = np.linspace(-127.0, -120.0, 70001)
    y = exp2_fma(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0)
