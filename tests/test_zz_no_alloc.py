"""k_smooth_mean_noalloc, the allocation-free K channel mean, against k_smooth_mean.

Some callers cannot let a library allocate device memory during a call -- for example a serving
process that gives all device memory to its own pool at start-up, where an allocation inside
the call could fail or stall the stream. For them the library keeps the partial sums of this
one pre-pass in a fixed device array instead. These checks go through the C ABI: two calls in a
row must match the allocating entry point, and the CPU oracle, within the K-mean tolerance, also
at the largest size the fixed array takes (one chunk of partial sums); a problem too large for
the fixed array must be refused before anything is launched. The file is named so that pytest
collects it last.
"""
import numpy as np
import pytest
import torch

import oracle
from libutil import ensure_built
from workloads import bf16_bits, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def b2():
    ensure_built()
    import head_attention_forward_flash_b200 as mod
    return mod


@pytest.mark.parametrize("shape,seed", [((1, 16, 4096, 256), 4), ((2, 3, 1000, 128), 5),
                                        ((1, 1, 77, 64), 6), ((4, 1024, 40, 256), 7)])
def test_noalloc_mean_matches_allocating_mean_twice(b2, shape, seed):
    lib = b2.lib
    b, hk, sk, d = shape
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream().cuda_stream
    _, k, _ = make_inputs(b, 1, hk, 1, sk, d, d, seed=seed, kmean=True)
    kd = k.to(dev)
    ref = torch.empty((b, hk, d), dtype=torch.float32, device=dev)
    assert lib.k_smooth_mean(kd.data_ptr(), ref.data_ptr(), b, hk, sk, d, stream) == 0
    torch.cuda.synchronize()
    # the K-mean tolerance: 1e-5 relative to max(|mean|, mean over s of |K|)
    scale = torch.maximum(ref.abs(), kd.float().abs().mean(dim=1))
    m64, _ = oracle.k_mean(bf16_bits(k), b, hk, sk, d)
    for call in range(2):
        out = torch.full((b, hk, d), float("nan"), dtype=torch.float32, device=dev)
        rc = lib.k_smooth_mean_noalloc(kd.data_ptr(), out.data_ptr(), b, hk, sk, d, stream)
        assert rc == 0, lib.attn_status_string(rc)
        torch.cuda.synchronize()
        assert bool(torch.all((out - ref).abs() <= 1e-5 * scale)), f"call {call}"
        got = out.cpu().double().numpy()
        tol = 1e-5 * np.maximum(np.abs(m64), k.double().abs().mean(dim=1).numpy())
        assert np.all(np.abs(got - m64) <= tol), f"call {call} against the oracle"


def test_noalloc_python_binding(b2):
    """The binding's wrapper takes the caller's output buffer and allocates nothing."""
    dev = torch.device("cuda:0")
    _, k, _ = make_inputs(1, 1, 2, 1, 300, 128, 128, seed=8, kmean=True)
    kd = k.to(dev)
    out = torch.empty((1, 2, 128), dtype=torch.float32, device=dev)
    got = b2.k_smooth_mean_noalloc(kd, out)
    torch.cuda.synchronize()
    assert got.data_ptr() == out.data_ptr()
    m64, _ = oracle.k_mean(bf16_bits(k), 1, 2, 300, 128)
    tol = 1e-5 * np.maximum(np.abs(m64), k.double().abs().mean(dim=1).numpy())
    assert np.all(np.abs(out.cpu().double().numpy() - m64) <= tol)


def test_noalloc_refuses_problems_beyond_its_scratch(b2):
    fake = 0x10000  # never dereferenced: the size check fails before any launch
    assert b2.lib.k_smooth_mean_noalloc(fake, fake, 1, 8192, 16, 256, None) == 11
    assert b2.lib.k_smooth_mean_noalloc(fake, fake, 5, 1024, 16, 256, None) == 11
