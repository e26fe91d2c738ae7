"""k_smooth_mean_strided: the K channel mean of strided and misaligned views of K, against the
oracle, through the C ABI and the binding.

"[HIP] Mha v4: run the K-smoothing gate as one HIP call" (PR Self-Review: PR-specific question;
Changed op tests) takes BSHD K with a contiguous last dimension, sends misaligned views down a
scalar-load path, and tests head-sliced and misaligned K views. Here each view's mean must match
the oracle's mean of the same elements (copied out contiguously on the CPU) within the K-mean
tolerance, repeated calls must agree bit for bit, and the contiguous aligned layout must give
exactly k_smooth_mean's bits.
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


def check_against_oracle(view, got):
    """got [b, hk, d] on the GPU against the oracle's mean of the view's elements."""
    kc = view.cpu().contiguous()
    b, sk, hk, d = kc.shape
    m64, _ = oracle.k_mean(bf16_bits(kc), b, hk, sk, d)
    tol = 1e-5 * np.maximum(np.abs(m64), kc.double().abs().mean(dim=1).numpy())
    err = np.abs(got.cpu().double().numpy() - m64)
    assert np.all(err <= tol), float((err - tol).max())


def full_k(b, sk, hk, d, seed):
    _, k, _ = make_inputs(b, 1, hk, 1, sk, d, d, seed=seed, kmean=True)
    return k.to("cuda:0")


@pytest.mark.parametrize("b,sk,hk_full,h0,hk,d", [
    (1, 4096, 8, 2, 3, 128),    # a slice of the heads
    (2, 1000, 5, 4, 1, 256),    # the last head alone
    (1, 65536, 5, 1, 2, 128),   # long keys, many chunks
    (3, 77, 4, 0, 4, 64),       # every head (contiguous rows, still a batch-strided buffer)
])
def test_head_sliced_view(b2, b, sk, hk_full, h0, hk, d):
    k = full_k(b, sk, hk_full, d, seed=11 + h0)
    view = k[:, :, h0:h0 + hk, :]
    m1 = b2.k_smooth_mean_strided(view)
    m2 = b2.k_smooth_mean_strided(view)
    torch.cuda.synchronize()
    assert torch.equal(m1, m2)
    check_against_oracle(view, m1)


@pytest.mark.parametrize("offset", [1, 3, 8])
def test_misaligned_view(b2, offset):
    """A view that starts `offset` bf16 elements into a buffer (2 or 6 bytes off a 16-byte
    boundary for odd offsets): refused by k_smooth_mean, accepted here."""
    b, sk, hk, d = 2, 513, 3, 64
    src = full_k(1, b * sk + 1, hk, d, seed=20 + offset).reshape(-1)
    flat = src[offset:offset + b * sk * hk * d]
    view = flat.view(b, sk, hk, d)
    if offset % 8:
        assert view.data_ptr() % 16 != 0
        with pytest.raises(b2.B200AttnError):
            b2.k_smooth_mean(view)
    got = b2.k_smooth_mean_strided(view)
    check_against_oracle(view, got)


def test_key_sliced_and_batch_strided_view(b2):
    """Keys 100..2099 of every other batch of a larger K: non-unit batch and key offsets."""
    k = full_k(4, 2304, 2, 128, seed=31)
    view = k[::2, 100:2100]
    got = b2.k_smooth_mean_strided(view)
    check_against_oracle(view, got)


def test_contiguous_view_is_k_smooth_mean(b2):
    k = full_k(1, 4096, 16, 256, seed=41)
    ref = b2.k_smooth_mean(k)
    got = b2.k_smooth_mean_strided(k)
    torch.cuda.synchronize()
    assert torch.equal(ref, got)


def test_c_abi_with_explicit_strides(b2):
    """The raw entry point with hand-written element strides for a head slice, on the caller's
    output buffer."""
    b, sk, hk_full, d = 1, 3000, 6, 128
    k = full_k(b, sk, hk_full, d, seed=51)
    out = torch.full((b, 2, d), float("nan"), dtype=torch.float32, device=k.device)
    stream = torch.cuda.current_stream().cuda_stream
    ptr = k.data_ptr() + 3 * d * 2  # head 3
    rc = b2.lib.k_smooth_mean_strided(ptr, out.data_ptr(), b, 2, sk, d, sk * hk_full * d,
                                      hk_full * d, d, stream)
    assert rc == 0, b2.lib.attn_status_string(rc)
    torch.cuda.synchronize()
    check_against_oracle(k[:, :, 3:5, :], out)
