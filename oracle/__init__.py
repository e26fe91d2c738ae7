"""CPU oracle for the attention forward pass and the K channel-mean pre-pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / reference arm are the only code allowed to import this package. The CUDA
library never imports, links or calls it, and it never imports the CUDA library.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, one left-to-right loop per sum; see
its header for the definition it follows). This module compiles it with gcc, loads it with
ctypes and marshals numpy arrays of raw bf16 bit patterns (uint16) in and fp64 results out.

The FP8 (E4M3) recipe -- codes, the per-head quantiser and attention on decoded inputs -- is in
``oracle.fp8`` (numpy, on top of the fp64-input entry points of ``attn_oracle.c``).

Parity status: every function here is pinned by ``tests/test_oracle.py`` against torch's fp64
scaled-dot-product attention and logsumexp, numpy's fp64 mean, torch's fp32->bf16 cast, closed
forms and invariants; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_p = ctypes.c_void_p


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle into a shared library (no -ffast-math: IEEE fp64, no reassociation)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-shared", "-fPIC", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _bind(lib):
    lib.oracle_attn_rows.argtypes = [_p, _p, _p] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double,
                                                               _p, _i64, _p, _p, ctypes.c_int]
    lib.oracle_attn_rows.restype = ctypes.c_int
    lib.oracle_attn_full.argtypes = [_p, _p, _p] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double,
                                                               _p, _p, ctypes.c_int]
    lib.oracle_attn_full.restype = ctypes.c_int
    lib.oracle_attn_rows_ex.argtypes = [_p, _p, _p] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double,
                                        _i64, _p, _p, _i64, _p, _p, ctypes.c_int]
    lib.oracle_attn_rows_ex.restype = ctypes.c_int
    lib.oracle_attn_full_ex.argtypes = [_p, _p, _p] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double,
                                        _i64, _p, _p, _p, ctypes.c_int]
    lib.oracle_attn_full_ex.restype = ctypes.c_int
    lib.oracle_attn_full_f64.argtypes = [_p, _p, _p] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double,
                                                                   _p, _p, ctypes.c_int]
    lib.oracle_attn_full_f64.restype = ctypes.c_int
    lib.oracle_attn_rows_f64.argtypes = [_p, _p, _p] + [_i64] * 7 + [ctypes.c_int, ctypes.c_double,
                                                                   _p, _i64, _p, _p, ctypes.c_int]
    lib.oracle_attn_rows_f64.restype = ctypes.c_int
    lib.oracle_k_mean.argtypes = [_p, _i64, _i64, _i64, _i64, _p, _p]
    lib.oracle_k_mean.restype = ctypes.c_int
    lib.oracle_k_gate.argtypes = [_p, _i64, _i64, _i64, _i64, ctypes.c_double, _p, _p, _p, _p]
    lib.oracle_k_gate.restype = ctypes.c_int
    lib.oracle_k_sub.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i64]
    lib.oracle_k_sub.restype = ctypes.c_int
    lib.oracle_bf16_rne.argtypes = [ctypes.c_double]
    lib.oracle_bf16_rne.restype = ctypes.c_uint16
    return lib


def load_library(path: str | None = None):
    """Load (building first if needed) the oracle library; ``path`` loads another build."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are raw bf16 bit patterns (numpy uint16)")
    return a


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _sinks(sinks, hq):
    if sinks is None:
        return None
    s = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64).reshape(-1))
    if s.shape[0] != hq:
        raise ValueError("sinks must hold one logit per query head")
    return s


def attn_rows(q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale, rows, nthreads=None, lib=None,
              window=-1, sinks=None):
    """O (fp64 [nrows, dv]) and LSE (fp64 [nrows]) for the (batch, head, query) triples in rows.

    window >= 0 limits row i to keys j >= i + sk - sq - window; sinks (one logit per query head)
    join each row's softmax denominator (see attn_oracle.c)."""
    lib = lib or load_library()
    q, k, v = _u16(q), _u16(k), _u16(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.zeros((n, dv), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    sk_arr = _sinks(sinks, hq)
    rc = lib.oracle_attn_rows_ex(_ptr(q), _ptr(k), _ptr(v), b, hq, hk, sq, sk, dqk, dv,
                                 int(causal), float(scale), int(window),
                                 _ptr(sk_arr) if sk_arr is not None else None, _ptr(rows), n,
                                 _ptr(o), _ptr(lse), int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_attn_rows failed with code {rc}")
    return o, lse


def attn_full(q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale, nthreads=None, lib=None,
              window=-1, sinks=None):
    """O (fp64 BSHD [b,sq,hq,dv]) and LSE (fp64 [b,hq,sq]) for every row (window and sinks as
    in attn_rows)."""
    lib = lib or load_library()
    q, k, v = _u16(q), _u16(k), _u16(v)
    o = np.zeros((b, sq, hq, dv), dtype=np.float64)
    lse = np.zeros((b, hq, sq), dtype=np.float64)
    sk_arr = _sinks(sinks, hq)
    rc = lib.oracle_attn_full_ex(_ptr(q), _ptr(k), _ptr(v), b, hq, hk, sq, sk, dqk, dv,
                                 int(causal), float(scale), int(window),
                                 _ptr(sk_arr) if sk_arr is not None else None, _ptr(o), _ptr(lse),
                                 int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_attn_full failed with code {rc}")
    return o, lse


def attn_varlen(q, k, v, cu_q, cu_k, hq, hk, dqk, dv, causal, scale, nthreads=None, lib=None):
    """Packed sequences: O (fp64 [total_q, hq, dv]) and LSE (fp64 [hq, total_q]).

    Sequence i is the dense problem on its own query rows cu_q[i] .. cu_q[i+1]-1 and key rows
    cu_k[i] .. cu_k[i+1]-1 -- the "varlen" layout of the shape tables of "Tune MHA config &
    small-head pipeline pathology" (Source of shapes; varlen rows after Final status), read as
    independent sequences packed along the row axis. Each sequence goes to attn_full with b = 1.
    Rows that belong to no sequence are NaN.
    """
    q = _u16(q).reshape(-1, hq, dqk)
    k = _u16(k).reshape(-1, hk, dqk)
    v = _u16(v).reshape(-1, hk, dv)
    total_q = q.shape[0]
    o = np.full((total_q, hq, dv), np.nan)
    lse = np.full((hq, total_q), np.nan)
    cu_q = [int(x) for x in cu_q]
    cu_k = [int(x) for x in cu_k]
    for i in range(len(cu_q) - 1):
        qs, qe, ks, ke = cu_q[i], cu_q[i + 1], cu_k[i], cu_k[i + 1]
        if qe <= qs:
            continue
        oi, li = attn_full(np.ascontiguousarray(q[qs:qe]), np.ascontiguousarray(k[ks:ke]),
                           np.ascontiguousarray(v[ks:ke]), 1, hq, hk, qe - qs, ke - ks, dqk, dv,
                           causal, scale, nthreads=nthreads, lib=lib)
        o[qs:qe] = oi[0]
        lse[:, qs:qe] = li[0]
    return o, lse


def k_mean(k, b, hk, sk, d, lib=None):
    """Channel mean of K over the sequence: (fp64 [b,hk,d], its fp32 rounding [b,hk,d])."""
    lib = lib or load_library()
    k = _u16(k)
    m64 = np.zeros((b, hk, d), dtype=np.float64)
    m32 = np.zeros((b, hk, d), dtype=np.float32)
    rc = lib.oracle_k_mean(_ptr(k), b, hk, sk, d, _ptr(m64), _ptr(m32))
    if rc != 0:
        raise ValueError(f"oracle_k_mean failed with code {rc}")
    return m64, m32


def k_gate(k, b, hk, sk, d, threshold, lib=None):
    """K-smoothing gate over the strided key sample (see attn_oracle.c): returns (mean fp64
    [b,hk,d], its fp32 rounding, ratio fp64 [b,hk], gate int32 [b,hk]); mean is the sampled
    channel mean where the gate is on, else 0."""
    lib = lib or load_library()
    k = _u16(k)
    m64 = np.zeros((b, hk, d), dtype=np.float64)
    m32 = np.zeros((b, hk, d), dtype=np.float32)
    r = np.zeros((b, hk), dtype=np.float64)
    gate = np.zeros((b, hk), dtype=np.int32)
    rc = lib.oracle_k_gate(_ptr(k), b, hk, sk, d, float(threshold), _ptr(m64), _ptr(m32), _ptr(r),
                           _ptr(gate))
    if rc != 0:
        raise ValueError(f"oracle_k_gate failed with code {rc}")
    return m64, m32, r, gate


def k_sub(k, mean32, b, hk, sk, d, lib=None):
    """K' = bf16_rne(K - mean) as raw bf16 bits [b,sk,hk,d]."""
    lib = lib or load_library()
    k = _u16(k)
    mean32 = np.ascontiguousarray(mean32, dtype=np.float32)
    out = np.zeros((b, sk, hk, d), dtype=np.uint16)
    rc = lib.oracle_k_sub(_ptr(k), _ptr(mean32), _ptr(out), b, hk, sk, d)
    if rc != 0:
        raise ValueError(f"oracle_k_sub failed with code {rc}")
    return out


def bf16_rne(x, lib=None) -> np.ndarray:
    """Round each fp64 value of x to bf16 (nearest, ties to even); returns the uint16 bits."""
    lib = lib or load_library()
    flat = np.asarray(x, dtype=np.float64).ravel()
    return np.array([lib.oracle_bf16_rne(float(t)) for t in flat], dtype=np.uint16).reshape(
        np.shape(x))


def bf16_to_f64(bits) -> np.ndarray:
    """Decode raw bf16 bit patterns to fp64 (a bf16 value is the top half of a binary32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
