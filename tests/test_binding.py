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
