"""The binding refuses caller-supplied output buffers of the wrong shape, dtype or device before
anything is launched (an undersized buffer would be written past its end), for every entry point
that accepts one."""
import pytest
import torch

from libutil import ensure_built

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def b2():
    ensure_built()
    import head_attention_forward_flash_b200 as mod
    yield mod
    assert mod.attn_debug_status() == 0


def cuda(shape, dtype=torch.bfloat16):
    return torch.zeros(shape, dtype=dtype, device="cuda")


def test_attention_outputs_refused(b2):
    q, k, v = cuda((1, 16, 2, 64)), cuda((1, 16, 1, 64)), cuda((1, 16, 1, 64))
    good_o, good_l = cuda((1, 16, 2, 64)), cuda((1, 2, 16), torch.float32)
    bad = [dict(out=cuda((1, 15, 2, 64))), dict(out=cuda((1, 16, 2, 64), torch.float16)),
           dict(out=good_o, lse=cuda((1, 2, 15), torch.float32)),
           dict(out=good_o, lse=cuda((1, 16, 2), torch.float32)),
           dict(out=good_o, lse=cuda((1, 2, 16), torch.bfloat16)),
           dict(out=torch.zeros((1, 16, 2, 64), dtype=torch.bfloat16))]
    for kw in bad:
        with pytest.raises((ValueError, TypeError)):
            b2.attn_fwd(q, k, v, **kw)
        with pytest.raises((ValueError, TypeError)):
            b2.attn_fwd_window_sink(q, k, v, window_left=4, **kw)
    with pytest.raises(ValueError):
        b2.attn_fwd_window_sink(q, k, v, sinks=cuda((1,), torch.float32))
    o, l = b2.attn_fwd(q, k, v, out=good_o, lse=good_l)  # the exact buffers are accepted
    assert o.data_ptr() == good_o.data_ptr() and l.data_ptr() == good_l.data_ptr()


def test_varlen_outputs_refused(b2):
    q, k, v = cuda((20, 2, 64)), cuda((20, 1, 64)), cuda((20, 1, 64))
    cu = torch.tensor([0, 8, 20], dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        b2.attn_fwd_varlen(q, k, v, cu, cu, 12, out=cuda((19, 2, 64)))
    with pytest.raises(ValueError):
        b2.attn_fwd_varlen(q, k, v, cu, cu, 12, lse=cuda((20, 2), torch.float32))


def test_fp8_outputs_refused(b2):
    x = cuda((1, 16, 2, 128))
    with pytest.raises(ValueError):
        b2.fp8_quantize(x, out=cuda((1, 16, 2, 64), torch.uint8))
    with pytest.raises(ValueError):
        b2.fp8_quantize(x, descale=cuda((1, 1), torch.float32))
    with pytest.raises(ValueError):
        b2.fp8_quantize(x, mean=cuda((1, 2, 64), torch.float32))
    q8 = cuda((1, 16, 2, 128), torch.uint8)
    ds = cuda((1, 2), torch.float32)
    with pytest.raises(ValueError):
        b2.attn_fwd_fp8(q8, q8, q8, ds, ds, ds, out=cuda((1, 16, 2, 64)))
    with pytest.raises(ValueError):
        b2.attn_fwd_fp8(q8, q8, q8, ds, ds, cuda((1, 1), torch.float32))


def test_k_mean_and_gate_outputs_refused(b2):
    k = cuda((1, 32, 2, 64))
    for fn in (b2.k_smooth_mean, b2.k_smooth_mean_noalloc):
        with pytest.raises(ValueError):
            fn(k, cuda((1, 1, 64), torch.float32))
        with pytest.raises(TypeError):
            fn(k, cuda((1, 2, 64), torch.float64))
    with pytest.raises(ValueError):
        b2.k_smooth_gate(k, 0.25, mean=cuda((1, 2, 32), torch.float32))
    with pytest.raises(ValueError):
        b2.k_smooth_gate(k, 0.25, gate=cuda((1, 1), torch.int32))
    with pytest.raises(ValueError):
        b2.k_smooth_gate(k, 0.25, ratio=cuda((2, 1), torch.float32))
    with pytest.raises(ValueError):
        b2.k_smooth_sub(k, cuda((1, 2, 64), torch.float32), out=cuda((1, 31, 2, 64)))
    with pytest.raises(ValueError):
        b2.k_smooth_sub(k, cuda((1, 2, 63), torch.float32))
