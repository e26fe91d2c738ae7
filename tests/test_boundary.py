"""C-ABI boundary checks that need no GPU: the library loads, exports every function the header
declares, and refuses invalid arguments with the documented status before any CUDA call."""
import ctypes

import pytest

from libutil import ensure_built, header_functions

ensure_built()
import head_attention_forward_flash_b200 as b2  # noqa: E402

A = 0x10000  # a fake, 16-byte aligned, never-dereferenced address (checks fail before any use)


def test_exports_every_header_function():
    names = header_functions()
    assert set(names) == set(b2.EXPORTS), names
    raw = ctypes.CDLL(b2.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} not exported"


def test_status_strings():
    for code in range(0, 12):
        s = b2.lib.attn_status_string(code)
        assert s and s.decode() != "unknown status"
    assert b2.lib.attn_status_string(99).decode() == "unknown status"


def call(q=A, k=A, v=A, o=A, lse=A, b=1, hq=2, hk=1, sq=16, sk=16, dqk=64, dv=64, causal=0,
         scale=0.125):
    return b2.lib.attn_fwd(q, k, v, o, lse, b, hq, hk, sq, sk, dqk, dv, causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(b=-1), 2), (dict(sq=-3), 2), (dict(sk=-1), 2), (dict(hk=0), 2), (dict(hq=-2), 2),
    (dict(hq=3, hk=2), 3), (dict(hq=6, hk=4), 3),
    (dict(dqk=96, dv=96), 4), (dict(dqk=128, dv=64), 4), (dict(dqk=192, dv=192), 4),
    (dict(dqk=32, dv=32), 4),
    (dict(scale=float("nan")), 7), (dict(scale=float("inf")), 7),
    (dict(q=None), 1), (dict(o=None), 1), (dict(k=None), 1), (dict(v=None), 1),
    (dict(q=A + 8), 5), (dict(k=A + 2), 5), (dict(o=A + 4), 5), (dict(lse=A + 2), 5),
    (dict(b=1 << 40, hq=1 << 40, hk=1), 6), (dict(sq=1 << 31), 6),
    (dict(sk=1 << 33, b=1, hk=1), 6),
])
def test_attn_fwd_rejects(kw, code):
    assert call(**kw) == code


def test_empty_problem_is_a_no_op():
    # b, hq or sq == 0: nothing to compute, no pointer is touched, no CUDA call is made.
    assert call(b=0, q=None, k=None, v=None, o=None, lse=None) == 0
    assert call(sq=0, q=None, o=None, lse=None) == 0
    assert call(hq=0, hk=1, q=None, o=None, lse=None) == 0


def test_noalloc_mean_size_limit():
    # b * hk * d above the fixed 2^20-float scratch is refused before any CUDA call
    assert b2.lib.k_smooth_mean_noalloc(A, A, 1, 4097, 16, 256, None) == 11
    assert b2.lib.k_smooth_mean_noalloc(A, A, 1, 4, 16, 96, None) == 4


@pytest.mark.parametrize("fn", ["k_smooth_mean", "k_smooth_sub", "k_smooth_mean_sub"])
def test_k_mean_rejects(fn):
    f = getattr(b2.lib, fn)

    def c(k=A, m=A, b=1, hk=2, sk=8, d=64):
        if fn == "k_smooth_mean":
            return f(k, m, b, hk, sk, d, None)
        return f(k, m, A, b, hk, sk, d, None)

    assert c(d=96) == 4 and c(d=192) == 4
    assert c(sk=0) == 2 and c(b=-1) == 2 and c(hk=-1) == 2
    assert c(k=None) == 1 and c(m=None) == 1
    assert c(k=A + 8) == 5 and c(m=A + 4) == 5
    assert c(b=0) == 0 and c(hk=0) == 0
    if fn != "k_smooth_mean":
        assert f(A, A, None, 1, 2, 8, 64, None) == 1
        assert f(A, A, A + 2, 1, 2, 8, 64, None) == 5


def test_k_mean_strided_rejects():
    f = b2.lib.k_smooth_mean_strided

    def c(k=A, m=A, b=1, hk=2, sk=8, d=64, sb=2048, ss=256, sh=64):
        return f(k, m, b, hk, sk, d, sb, ss, sh, None)

    assert c(d=96) == 4 and c(d=192) == 4
    assert c(sk=0) == 2 and c(b=-1) == 2 and c(hk=-1) == 2
    assert c(sb=-1) == 2 and c(ss=-64) == 2 and c(sh=-1) == 2
    assert c(k=None) == 1 and c(m=None) == 1
    assert c(k=A + 1) == 5 and c(m=A + 2) == 5
    assert c(b=0) == 0 and c(hk=0) == 0
    assert c(ss=1 << 62) == 6 and c(b=2, sb=1 << 62) == 6
    assert c(hk=1 << 20, d=256) == 6  # more channel blocks than a grid dimension holds


def call_varlen(q=A, k=A, v=A, o=A, lse=A, cq=A, ck=A, b=2, hq=2, hk=1, tq=32, tk=32, max_sq=16,
                dqk=64, dv=64, causal=0, scale=0.125):
    return b2.lib.attn_fwd_varlen(q, k, v, o, lse, cq, ck, b, hq, hk, tq, tk, max_sq, dqk, dv,
                                  causal, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(b=-1), 2), (dict(tq=-1), 2), (dict(tk=-5), 2), (dict(max_sq=-1), 2), (dict(hk=0), 2),
    (dict(hq=3, hk=2), 3), (dict(dqk=128, dv=64), 4), (dict(dqk=32, dv=32), 4),
    (dict(scale=float("nan")), 7),
    (dict(q=None), 1), (dict(o=None), 1), (dict(k=None), 1), (dict(v=None), 1),
    (dict(cq=None), 1), (dict(ck=None), 1),
    (dict(q=A + 8), 5), (dict(v=A + 2), 5), (dict(lse=A + 2), 5), (dict(cq=A + 2), 5),
    (dict(ck=A + 1), 5),
    (dict(tq=1 << 31), 6), (dict(tk=1 << 31), 6), (dict(b=1 << 20, hq=1 << 10, hk=1, max_sq=1 << 10), 6),
])
def test_attn_fwd_varlen_rejects(kw, code):
    assert call_varlen(**kw) == code


def test_varlen_empty_problem_is_a_no_op():
    # no sequence, no query row or a zero longest length: nothing is computed or touched
    assert call_varlen(b=0, q=None, k=None, v=None, o=None, lse=None, cq=None, ck=None) == 0
    assert call_varlen(tq=0, q=None, o=None, lse=None, cq=None, ck=None) == 0
    assert call_varlen(max_sq=0, q=None, o=None, lse=None, cq=None, ck=None) == 0


def call_ws(q=A, k=A, v=A, o=A, lse=A, sinks=A, b=1, hq=2, hk=1, sq=16, sk=16, dqk=64, dv=64,
            causal=1, window=8, scale=0.125):
    return b2.lib.attn_fwd_window_sink(q, k, v, o, lse, sinks, b, hq, hk, sq, sk, dqk, dv, causal,
                                       window, scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(b=-1), 2), (dict(sk=-1), 2), (dict(hk=0), 2), (dict(hq=3, hk=2), 3),
    (dict(dqk=96, dv=96), 4), (dict(scale=float("inf")), 7),
    (dict(q=None), 1), (dict(k=None), 1), (dict(o=None), 1),
    (dict(q=A + 8), 5), (dict(sinks=A + 2), 5), (dict(lse=A + 1), 5),
    (dict(sq=1 << 31), 6),
])
def test_attn_fwd_window_sink_rejects(kw, code):
    assert call_ws(**kw) == code


def test_window_sink_empty_problem_is_a_no_op():
    assert call_ws(b=0, q=None, k=None, v=None, o=None, lse=None, sinks=None) == 0
    assert call_ws(sq=0, q=None, o=None, lse=None) == 0


def test_k_smooth_gate_rejects():
    f = b2.lib.k_smooth_gate

    def c(k=A, m=A, g=A, r=A, b=1, hk=2, sk=8, d=64, t=0.25):
        return f(k, m, g, r, b, hk, sk, d, t, None)

    assert c(d=96) == 4 and c(sk=0) == 2 and c(b=-1) == 2
    assert c(k=None) == 1 and c(m=None) == 1 and c(g=None) == 1
    assert c(k=A + 8) == 5 and c(m=A + 4) == 5 and c(g=A + 2) == 5 and c(r=A + 1) == 5
    assert c(t=float("nan")) == 7 and c(t=float("inf")) == 7
    assert c(b=0) == 0 and c(hk=0) == 0


def test_debug_starve_range():
    assert b2.lib.attn_debug_starve(0) == 6 and b2.lib.attn_debug_starve(2_000_000) == 6


def call_fp8(q=A, k=A, v=A, dq=A, dk=A, dv_=A, o=A, lse=A, b=1, hq=2, hk=1, sq=16, sk=16,
             dqk=128, dv=128, causal=1, scale=0.125):
    return b2.lib.attn_fwd_fp8(q, k, v, dq, dk, dv_, o, lse, b, hq, hk, sq, sk, dqk, dv, causal,
                               scale, None)


@pytest.mark.parametrize("kw,code", [
    (dict(b=-1), 2), (dict(sk=-1), 2), (dict(hk=0), 2), (dict(hq=3, hk=2), 3),
    (dict(dqk=64, dv=64), 4), (dict(dqk=192, dv=128), 4), (dict(dqk=256, dv=256), 4),
    (dict(scale=float("nan")), 7),
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(o=None), 1),
    (dict(dq=None), 1), (dict(dk=None), 1), (dict(dv_=None), 1),
    (dict(q=A + 8), 5), (dict(k=A + 1), 5), (dict(o=A + 2), 5), (dict(dq=A + 2), 5),
    (dict(dv_=A + 1), 5), (dict(lse=A + 3), 5),
    (dict(sq=1 << 31), 6), (dict(b=1 << 40, hq=1 << 40, hk=1), 6),
])
def test_attn_fwd_fp8_rejects(kw, code):
    assert call_fp8(**kw) == code


def test_fp8_empty_problem_is_a_no_op():
    assert call_fp8(b=0, q=None, k=None, v=None, dq=None, dk=None, dv_=None, o=None, lse=None) == 0
    assert call_fp8(sq=0, q=None, o=None, lse=None) == 0


def test_fp8_quantize_rejects():
    f = b2.lib.fp8_quantize

    def c(x=A, m=A, x8=A, ds=A, b=1, s=8, h=2, d=128):
        return f(x, m, x8, ds, b, s, h, d, None)

    assert c(d=96) == 4 and c(d=32) == 4 and c(b=-1) == 2 and c(s=-1) == 2 and c(h=-1) == 2
    assert c(x=None) == 1 and c(x8=None) == 1 and c(ds=None) == 1
    assert c(x=A + 8) == 5 and c(x8=A + 4) == 5 and c(m=A + 4) == 5 and c(ds=A + 2) == 5
    assert c(b=1 << 40, s=1 << 30) == 6
    assert c(b=0) == 0 and c(h=0) == 0
