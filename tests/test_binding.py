"""The Python binding's own argument checks (no GPU needed): every function refuses non-tensors,
tensors of the wrong rank and host tensors with a clear error before any CUDA call."""
import pytest
import torch

from libutil import ensure_built

ensure_built()
import head_attention_forward_flash_b200 as b2  # noqa: E402


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)  # a host tensor


CALLS = {
    "attn_fwd": lambda x: b2.attn_fwd(x, bf16(1, 4, 1, 64), bf16(1, 4, 1, 64)),
    "attn_fwd_window_sink": lambda x: b2.attn_fwd_window_sink(x, bf16(1, 4, 1, 64),
                                                              bf16(1, 4, 1, 64), window_left=2),
    "attn_fwd_varlen": lambda x: b2.attn_fwd_varlen(x, bf16(4, 1, 64), bf16(4, 1, 64),
                                                    torch.zeros(2, dtype=torch.int32),
                                                    torch.zeros(2, dtype=torch.int32), 4),
    "attn_fwd_fp8": lambda x: b2.attn_fwd_fp8(x, torch.zeros((1, 4, 1, 128), dtype=torch.uint8),
                                              torch.zeros((1, 4, 1, 128), dtype=torch.uint8),
                                              torch.ones(1, 1), torch.ones(1, 1), torch.ones(1, 1)),
    "fp8_quantize": lambda x: b2.fp8_quantize(x),
    "k_smooth_mean": lambda x: b2.k_smooth_mean(x),
    "k_smooth_gate": lambda x: b2.k_smooth_gate(x, 0.25),
    "k_smooth_sub": lambda x: b2.k_smooth_sub(x, torch.zeros((1, 1, 64))),
}
RANK = {"attn_fwd_varlen": 3}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_refuses_non_tensor(name):
    with pytest.raises(TypeError):
        CALLS[name]([[1.0]])


@pytest.mark.parametrize("name", sorted(CALLS))
def test_refuses_wrong_rank(name):
    with pytest.raises(ValueError, match="dims"):
        CALLS[name](bf16(4, 64))


@pytest.mark.parametrize("name", sorted(CALLS))
def test_refuses_host_tensor(name):
    rank = RANK.get(name, 4)
    shape = (4, 1, 64) if rank == 3 else (1, 4, 1, 128 if name == "attn_fwd_fp8" else 64)
    x = torch.zeros(shape, dtype=torch.uint8 if name == "attn_fwd_fp8" else torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        CALLS[name](x)


def test_debug_starve_range_from_python():
    with pytest.raises(b2.B200AttnError):
        b2.attn_debug_starve(0)


# Caller-supplied output buffers: exact shape, dtype, device and contiguity are required (a
# smaller buffer would be written past its end). The helpers run before any CUDA call, so they
# are checked here with host tensors standing for the expected device.
CPU = torch.device("cpu")


def test_output_buffer_exact_shape():
    b2._want_out(torch.empty((2, 3, 4, 64), dtype=torch.bfloat16), "out", (2, 3, 4, 64),
                 torch.bfloat16, CPU)
    for bad in ((2, 3, 4, 63), (2, 3, 3, 64), (1, 3, 4, 64), (2, 3, 4, 64, 1), (24, 64)):
        with pytest.raises(ValueError, match="shape"):
            b2._want_out(torch.empty(bad, dtype=torch.bfloat16), "out", (2, 3, 4, 64),
                         torch.bfloat16, CPU)


def test_output_buffer_dtype_device_contiguity():
    with pytest.raises(TypeError, match="float32"):
        b2._want_out(torch.empty((2, 4), dtype=torch.float16), "lse", (2, 4), torch.float32, CPU)
    with pytest.raises(ValueError, match="meta"):
        b2._want_out(torch.empty((2, 4), dtype=torch.float32, device="meta"), "lse", (2, 4),
                     torch.float32, CPU)
    with pytest.raises(ValueError, match="contiguous"):
        b2._want_out(torch.empty((4, 2), dtype=torch.float32).t(), "lse", (2, 4), torch.float32,
                     CPU)
    with pytest.raises(TypeError, match="Tensor"):
        b2._want_out([[0.0]], "mean", (1, 1), torch.float32, CPU)


def test_attention_outputs_checked_or_allocated():
    out, lse = b2._attn_outputs(None, None, True, (1, 8, 2, 64), (1, 2, 8), CPU)
    assert tuple(out.shape) == (1, 8, 2, 64) and out.dtype == torch.bfloat16
    assert tuple(lse.shape) == (1, 2, 8) and lse.dtype == torch.float32
    _, none = b2._attn_outputs(None, None, False, (1, 8, 2, 64), (1, 2, 8), CPU)
    assert none is None
    with pytest.raises(ValueError, match="shape"):  # an undersized O
        b2._attn_outputs(torch.empty((1, 7, 2, 64), dtype=torch.bfloat16), None, True,
                         (1, 8, 2, 64), (1, 2, 8), CPU)
    with pytest.raises(ValueError, match="shape"):  # LSE in the wrong layout
        b2._attn_outputs(None, torch.empty((1, 8, 2), dtype=torch.float32), True,
                         (1, 8, 2, 64), (1, 2, 8), CPU)
    with pytest.raises(ValueError, match="shape"):  # an LSE buffer passed with return_lse off
        b2._attn_outputs(None, torch.empty((1, 2, 7), dtype=torch.float32), False,
                         (1, 8, 2, 64), (1, 2, 8), CPU)
