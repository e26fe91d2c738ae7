"""Fused attention forward pass (with per-row log-sum-exp) on B200 (sm_100a) -- dense, packed
sequences, sliding window with sinks, and E4M3 inputs -- with the K channel-mean pre-pass, the
K-smoothing gate and the E4M3 quantiser, as a thin Python binding over the C ABI of
``libb200attn.so`` (declared in ``include/b200attn.h``).

The binding only marshals arguments: it checks dtypes/devices/contiguity, allocates outputs
with ``torch.empty`` and passes raw device pointers plus the current CUDA stream. Every step of
the computation runs in the library's CUDA kernels; there is no CPU or PyTorch fallback, and
importing this package fails loudly when the library is missing.

Raw C entry points, with the header's names and argument order, are exposed through ``lib``
(a ``ctypes.CDLL``): every name in ``EXPORTS`` (``lib.attn_fwd``, ``lib.attn_fwd_varlen``,
``lib.attn_fwd_window_sink``, ``lib.attn_fwd_fp8``, ``lib.fp8_quantize``, ``lib.k_smooth_gate``,
``lib.k_smooth_mean``, ``lib.k_smooth_mean_noalloc``, ``lib.k_smooth_mean_strided``,
``lib.k_smooth_sub``,
``lib.k_smooth_mean_sub``, ``lib.attn_status_string``, ``lib.attn_debug_status``, ``lib.attn_debug_starve``).
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libb200attn.so")

STATUS = {
    0: "OK", 1: "ERR_NULL", 2: "ERR_SHAPE", 3: "ERR_GQA", 4: "ERR_HEADDIM", 5: "ERR_ALIGN",
    6: "ERR_RANGE", 7: "ERR_SCALE", 8: "ERR_ARCH", 9: "ERR_CUDA", 10: "ERR_TIMEOUT",
    11: "ERR_SCRATCH",
}
EXPORTS = ("attn_fwd", "attn_fwd_varlen", "attn_fwd_window_sink", "attn_fwd_fp8", "fp8_quantize",
           "k_smooth_gate", "k_smooth_mean", "k_smooth_mean_noalloc", "k_smooth_mean_strided",
           "k_smooth_sub",
           "k_smooth_mean_sub", "attn_status_string", "attn_debug_status", "attn_debug_starve")


class B200AttnError(RuntimeError):
    def __init__(self, fn: str, status: int, message: str):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({message})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m head_attention_forward_flash_b200.build`"
            " (or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, ctypes.c_int,
                             ctypes.c_float, vp]
    lib.attn_fwd.restype = ctypes.c_int
    lib.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64,
                                    i64, ctypes.c_int, ctypes.c_float, vp]
    lib.attn_fwd_varlen.restype = ctypes.c_int
    lib.attn_fwd_window_sink.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64,
                                         ctypes.c_int, i64, ctypes.c_float, vp]
    lib.attn_fwd_window_sink.restype = ctypes.c_int
    lib.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64,
                                 ctypes.c_int, ctypes.c_float, vp]
    lib.attn_fwd_fp8.restype = ctypes.c_int
    lib.fp8_quantize.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, vp]
    lib.fp8_quantize.restype = ctypes.c_int
    lib.k_smooth_mean.argtypes = [vp, vp, i64, i64, i64, i64, vp]
    lib.k_smooth_mean.restype = ctypes.c_int
    lib.k_smooth_mean_noalloc.argtypes = [vp, vp, i64, i64, i64, i64, vp]
    lib.k_smooth_mean_noalloc.restype = ctypes.c_int
    lib.k_smooth_mean_strided.argtypes = [vp, vp, i64, i64, i64, i64, i64, i64, i64, vp]
    lib.k_smooth_mean_strided.restype = ctypes.c_int
    lib.k_smooth_gate.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, ctypes.c_float, vp]
    lib.k_smooth_gate.restype = ctypes.c_int
    lib.k_smooth_sub.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp]
    lib.k_smooth_sub.restype = ctypes.c_int
    lib.k_smooth_mean_sub.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp]
    lib.k_smooth_mean_sub.restype = ctypes.c_int
    lib.attn_status_string.argtypes = [ctypes.c_int]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_debug_status.argtypes = [vp]
    lib.attn_debug_status.restype = ctypes.c_int
    lib.attn_debug_starve.argtypes = [i64]
    lib.attn_debug_starve.restype = ctypes.c_int
    return lib


lib = _load()


def _check(fn: str, status: int):
    if status != 0:
        raise B200AttnError(fn, status, lib.attn_status_string(status).decode())


def _stream_ptr(t) -> int:
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


def _want(t, name, dims):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dims, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (BSHD)")


def _want_out(t, name, shape, dtype, device):
    """A caller-supplied output (or auxiliary) buffer: exactly ``shape`` and ``dtype``,
    contiguous and on ``device`` -- a smaller buffer would be written past its end."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name} must have shape {tuple(int(x) for x in shape)}, "
                         f"got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(ref, *named):
    for name, t in named:
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, expected {ref.device}")


def _attn_outputs(out, lse, return_lse, out_shape, lse_shape, device):
    """Allocates O and LSE, or checks the caller's buffers."""
    import torch
    if out is None:
        out = torch.empty(out_shape, dtype=torch.bfloat16, device=device)
    else:
        _want_out(out, "out", out_shape, torch.bfloat16, device)
    if lse is not None:
        _want_out(lse, "lse", lse_shape, torch.float32, device)
    elif return_lse:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=device)
    return out, lse


def attn_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
             return_lse: bool = True):
    """O = softmax(scale * Q K^T [+ causal mask]) V and the per-row LSE (natural log).

    q [b, sq, hq, dqk], k [b, sk, hk, dqk], v [b, sk, hk, dv]: contiguous bf16 CUDA tensors.
    Returns ``(out [b, sq, hq, dv] bf16, lse [b, hq, sq] fp32 or None)``.
    ``scale`` defaults to 1/sqrt(dqk).
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        _want(t, name, 4)
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    b, sq, hq, dqk = q.shape
    bk, sk, hk, dqk2 = k.shape
    bv, skv, hkv, dv = v.shape
    if bk != b or bv != b or dqk2 != dqk or skv != sk or hkv != hk:
        raise ValueError("inconsistent q/k/v shapes")
    _same_device(q, ("k", k), ("v", v))
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    out, lse = _attn_outputs(out, lse, return_lse, (b, sq, hq, dv), (b, hq, sq), q.device)
    st = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                      lse.data_ptr() if lse is not None else None, b, hq, hk, sq, sk, dqk, dv,
                      1 if causal else 0, float(scale), _stream_ptr(q))
    _check("attn_fwd", st)
    return out, lse


def attn_fwd_window_sink(q, k, v, causal: bool = False, window_left: int = -1, sinks=None,
                         scale: float | None = None, out=None, lse=None, return_lse: bool = True):
    """attn_fwd with a sliding window (row i keeps keys j >= i + sk - sq - window_left;
    window_left < 0: none) and optional per-head sink logits (fp32 CUDA tensor [hq]) that join
    every row's softmax denominator. Returns ``(out, lse)`` as attn_fwd."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        _want(t, name, 4)
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    b, sq, hq, dqk = q.shape
    bk, sk, hk, dqk2 = k.shape
    bv, skv, hkv, dv = v.shape
    if bk != b or bv != b or dqk2 != dqk or skv != sk or hkv != hk:
        raise ValueError("inconsistent q/k/v shapes")
    _same_device(q, ("k", k), ("v", v))
    if sinks is not None:
        _want_out(sinks, "sinks", (hq,), torch.float32, q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    out, lse = _attn_outputs(out, lse, return_lse, (b, sq, hq, dv), (b, hq, sq), q.device)
    st = lib.attn_fwd_window_sink(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  lse.data_ptr() if lse is not None else None,
                                  sinks.data_ptr() if sinks is not None else None, b, hq, hk, sq,
                                  sk, dqk, dv, 1 if causal else 0, int(window_left), float(scale),
                                  _stream_ptr(q))
    _check("attn_fwd_window_sink", st)
    return out, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, causal: bool = False,
                    scale: float | None = None, out=None, lse=None, return_lse: bool = True):
    """attn_fwd over packed sequences: sequence i owns query rows cu_seqlens_q[i] ..
    cu_seqlens_q[i+1]-1 and key rows cu_seqlens_k[i] .. cu_seqlens_k[i+1]-1.

    q [total_q, hq, dqk], k [total_k, hk, dqk], v [total_k, hk, dv]: contiguous bf16 CUDA
    tensors; cu_seqlens_q / cu_seqlens_k: int32 CUDA tensors of b + 1 offsets; max_seqlen_q: at
    least the longest query length. Returns ``(out [total_q, hq, dv] bf16, lse [hq, total_q] fp32
    or None)``. Rows that belong to no sequence are left as allocated.
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        _want(t, name, 3)
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        _want(t, name, 1)
        if t.dtype != torch.int32:
            raise TypeError(f"{name} must be int32")
    total_q, hq, dqk = q.shape
    total_k, hk, dqk2 = k.shape
    total_kv, hkv, dv = v.shape
    if dqk2 != dqk or total_kv != total_k or hkv != hk:
        raise ValueError("inconsistent q/k/v shapes")
    b = cu_seqlens_q.shape[0] - 1
    if b < 0 or cu_seqlens_k.shape[0] != b + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold b + 1 offsets")
    _same_device(q, ("k", k), ("v", v), ("cu_seqlens_q", cu_seqlens_q),
                 ("cu_seqlens_k", cu_seqlens_k))
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    out, lse = _attn_outputs(out, lse, return_lse, (total_q, hq, dv), (hq, total_q), q.device)
    st = lib.attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr() if lse is not None else None,
                             cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), b, hq, hk, total_q,
                             total_k, int(max_seqlen_q), dqk, dv, 1 if causal else 0,
                             float(scale), _stream_ptr(q))
    _check("attn_fwd_varlen", st)
    return out, lse


def _codes(t, name, dims):
    import torch
    _want(t, name, dims)
    if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
        raise TypeError(f"{name} must hold E4M3 codes (uint8 or float8_e4m3fn)")


def fp8_quantize(x, mean=None, out=None, descale=None):
    """E4M3 codes of a bf16 BSHD tensor x [b, s, h, d] with one fp32 descale per (batch, head)
    (amax / 448); ``mean`` ([b, h, d] fp32, e.g. from k_smooth_mean or k_smooth_gate) is
    subtracted first. Returns ``(codes [b, s, h, d] uint8, descale [b, h] fp32)``."""
    import torch
    _want(x, "x", 4)
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    b, s, h, d = x.shape
    if mean is not None:
        _want_out(mean, "mean", (b, h, d), torch.float32, x.device)
    if out is None:
        out = torch.empty((b, s, h, d), dtype=torch.uint8, device=x.device)
    else:
        if out.dtype == torch.float8_e4m3fn:
            out = out.view(torch.uint8)
        _want_out(out, "out", (b, s, h, d), torch.uint8, x.device)
    if descale is None:
        descale = torch.empty((b, h), dtype=torch.float32, device=x.device)
    else:
        _want_out(descale, "descale", (b, h), torch.float32, x.device)
    _check("fp8_quantize", lib.fp8_quantize(x.data_ptr(),
                                            mean.data_ptr() if mean is not None else None,
                                            out.data_ptr(), descale.data_ptr(), b, s, h, d,
                                            _stream_ptr(x)))
    return out, descale


def attn_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, causal: bool = False,
                 scale: float | None = None, out=None, lse=None, return_lse: bool = True):
    """attn_fwd on E4M3 inputs: q8 [b, sq, hq, 128], k8 [b, sk, hk, 128], v8 [b, sk, hk, 128]
    (uint8 or float8_e4m3fn CUDA tensors) with fp32 descales q_descale [b, hq], k_descale and
    v_descale [b, hk]. Returns ``(out [b, sq, hq, 128] bf16, lse [b, hq, sq] fp32 or None)``."""
    import torch
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _codes(t, name, 4)
    b, sq, hq, dqk = q8.shape
    bk, sk, hk, dqk2 = k8.shape
    bv, skv, hkv, dv = v8.shape
    if bk != b or bv != b or dqk2 != dqk or skv != sk or hkv != hk:
        raise ValueError("inconsistent q/k/v shapes")
    _same_device(q8, ("k8", k8), ("v8", v8))
    for name, t, n in (("q_descale", q_descale, hq), ("k_descale", k_descale, hk),
                       ("v_descale", v_descale, hk)):
        _want_out(t, name, (b, n), torch.float32, q8.device)
    if scale is None:
        scale = 1.0 / math.sqrt(dqk)
    out, lse = _attn_outputs(out, lse, return_lse, (b, sq, hq, dv), (b, hq, sq), q8.device)
    st = lib.attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), q_descale.data_ptr(),
                          k_descale.data_ptr(), v_descale.data_ptr(), out.data_ptr(),
                          lse.data_ptr() if lse is not None else None, b, hq, hk, sq, sk, dqk, dv,
                          1 if causal else 0, float(scale), _stream_ptr(q8))
    _check("attn_fwd_fp8", st)
    return out, lse


def k_smooth_mean(k, mean=None):
    """fp32 channel mean of K over its sequence axis: [b, hk, d]."""
    import torch
    _want(k, "k", 4)
    if k.dtype != torch.bfloat16:
        raise TypeError("k must be bfloat16")
    b, sk, hk, d = k.shape
    if mean is None:
        mean = torch.empty((b, hk, d), dtype=torch.float32, device=k.device)
    else:
        _want_out(mean, "mean", (b, hk, d), torch.float32, k.device)
    _check("k_smooth_mean",
           lib.k_smooth_mean(k.data_ptr(), mean.data_ptr(), b, hk, sk, d, _stream_ptr(k)))
    return mean


def k_smooth_mean_noalloc(k, mean):
    """k_smooth_mean without any device allocation inside the call (fixed library scratch);
    ``mean`` [b, hk, d] fp32 must be supplied by the caller."""
    import torch
    _want(k, "k", 4)
    if k.dtype != torch.bfloat16:
        raise TypeError("k must be bfloat16")
    b, sk, hk, d = k.shape
    _want_out(mean, "mean", (b, hk, d), torch.float32, k.device)
    _check("k_smooth_mean_noalloc", lib.k_smooth_mean_noalloc(k.data_ptr(), mean.data_ptr(), b, hk,
                                                              sk, d, _stream_ptr(k)))
    return mean


def k_smooth_mean_strided(k, mean=None):
    """k_smooth_mean of any 4-dim bf16 view ``k`` [b, sk, hk, d] of device memory whose last
    dimension is contiguous (a slice of heads or keys, an offset view): fp32 [b, hk, d]."""
    import torch
    if not isinstance(k, torch.Tensor):
        raise TypeError("k must be a torch.Tensor")
    if k.dim() != 4 or not k.is_cuda:
        raise ValueError("k must be a 4-dim CUDA tensor [b, sk, hk, d]")
    if k.dtype != torch.bfloat16:
        raise TypeError("k must be bfloat16")
    if k.shape[3] > 1 and k.stride(3) != 1:
        raise ValueError("k's last dimension must be contiguous")
    b, sk, hk, d = k.shape
    if mean is None:
        mean = torch.empty((b, hk, d), dtype=torch.float32, device=k.device)
    else:
        _want_out(mean, "mean", (b, hk, d), torch.float32, k.device)
    _check("k_smooth_mean_strided",
           lib.k_smooth_mean_strided(k.data_ptr(), mean.data_ptr(), b, hk, sk, d, k.stride(0),
                                     k.stride(1), k.stride(2), _stream_ptr(k)))
    return mean


def k_smooth_gate(k, threshold: float, mean=None, gate=None, ratio=None, return_ratio=True):
    """The K-smoothing gate over a strided sample of keys. k [b, sk, hk, d] bf16.

    Returns ``(mean [b, hk, d] fp32 -- the sampled channel mean where the gate is on, else 0 --,
    gate [b, hk] int32, ratio [b, hk] fp32 or None)``; pass ``mean`` to k_smooth_sub."""
    import torch
    _want(k, "k", 4)
    if k.dtype != torch.bfloat16:
        raise TypeError("k must be bfloat16")
    b, sk, hk, d = k.shape
    if mean is None:
        mean = torch.empty((b, hk, d), dtype=torch.float32, device=k.device)
    else:
        _want_out(mean, "mean", (b, hk, d), torch.float32, k.device)
    if gate is None:
        gate = torch.empty((b, hk), dtype=torch.int32, device=k.device)
    else:
        _want_out(gate, "gate", (b, hk), torch.int32, k.device)
    if ratio is not None:
        _want_out(ratio, "ratio", (b, hk), torch.float32, k.device)
    elif return_ratio:
        ratio = torch.empty((b, hk), dtype=torch.float32, device=k.device)
    st = lib.k_smooth_gate(k.data_ptr(), mean.data_ptr(), gate.data_ptr(),
                           ratio.data_ptr() if ratio is not None else None, b, hk, sk, d,
                           float(threshold), _stream_ptr(k))
    _check("k_smooth_gate", st)
    return mean, gate, ratio


def k_smooth_sub(k, mean, out=None):
    """bf16(K - mean) with the [b, hk, d] fp32 mean broadcast over the sequence axis."""
    import torch
    _want(k, "k", 4)
    if k.dtype != torch.bfloat16:
        raise TypeError("k must be bfloat16")
    b, sk, hk, d = k.shape
    _want_out(mean, "mean", (b, hk, d), torch.float32, k.device)
    if out is None:
        out = torch.empty_like(k)
    else:
        _want_out(out, "out", (b, sk, hk, d), torch.bfloat16, k.device)
    _check("k_smooth_sub", lib.k_smooth_sub(k.data_ptr(), mean.data_ptr(), out.data_ptr(), b, hk,
                                            sk, d, _stream_ptr(k)))
    return out


def k_smooth_mean_sub(k, mean=None, out=None):
    """k_smooth_mean and k_smooth_sub in one launch: returns ``(mean [b, hk, d] fp32,
    bf16(K - mean) [b, sk, hk, d])``, bit-identical to the two calls in sequence."""
    import torch
    _want(k, "k", 4)
    if k.dtype != torch.bfloat16:
        raise TypeError("k must be bfloat16")
    b, sk, hk, d = k.shape
    if mean is None:
        mean = torch.empty((b, hk, d), dtype=torch.float32, device=k.device)
    else:
        _want_out(mean, "mean", (b, hk, d), torch.float32, k.device)
    if out is None:
        out = torch.empty_like(k)
    else:
        _want_out(out, "out", (b, sk, hk, d), torch.bfloat16, k.device)
    _check("k_smooth_mean_sub", lib.k_smooth_mean_sub(k.data_ptr(), mean.data_ptr(), out.data_ptr(),
                                                      b, hk, sk, d, _stream_ptr(k)))
    return mean, out


def attn_debug_status(stream=None) -> int:
    """Synchronise and return/clear the device error word (0 = no kernel gave up a wait)."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    return int(lib.attn_debug_status(s))


def attn_debug_starve(timeout_us: int = 20000) -> None:
    """Failure test: the next attention launch loads nothing and every wait gives up after
    ``timeout_us``; attn_debug_status() then reports the timeout (status 10)."""
    _check("attn_debug_starve", lib.attn_debug_starve(int(timeout_us)))
