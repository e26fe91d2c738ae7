"""GPU parity of attn_fwd_window_sink (sliding window + attention sinks) against the oracle,
through the C-ABI."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from libutil import ensure_built

ensure_built()
import head_attention_forward_flash_b200 as b2  # noqa: E402

pytestmark = pytest.mark.gpu
TOL_O, TOL_LSE = 2e-2, 1e-3
DEV = "cuda"


def sinks_for(hq, seed):
    g = torch.Generator().manual_seed(seed)
    return (1.5 * torch.randn(hq, generator=g)).float()


def gpu(q, k, v, causal, window, sinks, scale):
    o, l = b2.attn_fwd_window_sink(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal,
                                   window_left=window,
                                   sinks=sinks.to(DEV) if sinks is not None else None, scale=scale)
    torch.cuda.synchronize()
    assert b2.attn_debug_status() == 0
    return o.float().cpu().numpy(), l.cpu().numpy()


def check(o, l, o_ref, l_ref):
    assert np.max(np.abs(o - o_ref)) <= TOL_O
    assert np.array_equal(np.isneginf(l), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    if fin.any():
        assert np.max(np.abs(l[fin] - l_ref[fin])) <= TOL_LSE


@pytest.mark.parametrize("dqk,dv", workloads.HEAD_DIMS)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("window", [0, 1, 63, 100, 300])
@pytest.mark.parametrize("with_sinks", [False, True])
def test_parity(dqk, dv, causal, window, with_sinks):
    b, hq, hk, sq, sk = 2, 4, 2, 200, 330  # sk > sq: the diagonal sits at key i + 130
    q, k, v = workloads.make_inputs(b, hq, hk, sq, sk, dqk, dv, seed=61 + window)
    sinks = sinks_for(hq, 7) if with_sinks else None
    scale = 1.0 / math.sqrt(dqk)
    o, l = gpu(q, k, v, causal, window, sinks, scale)
    o_ref, l_ref = oracle.attn_full(workloads.bf16_bits(q), workloads.bf16_bits(k),
                                    workloads.bf16_bits(v), b, hq, hk, sq, sk, dqk, dv, causal,
                                    scale, window=window,
                                    sinks=sinks.double().numpy() if sinks is not None else None)
    check(o, l, o_ref, l_ref)


def test_long_sequence_skips_blocks():
    """4096 keys with a 128-key window: most key blocks of every unit are never visited;
    sampled rows (first, last and seeded) of every head against the oracle."""
    b, hq, hk, s, d = 1, 4, 1, 4096, 64
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, d, d, seed=71)
    sinks = sinks_for(hq, 8)
    o, l = gpu(q, k, v, True, 128, sinks, 0.125)
    g = torch.Generator().manual_seed(72)
    pos = sorted({0, 1, 127, 128, 129, s - 1, *torch.randint(0, s, (20,), generator=g).tolist()})
    rows = np.array([(0, h, i) for h in range(hq) for i in pos], dtype=np.int64)
    o_ref, l_ref = oracle.attn_rows(workloads.bf16_bits(q), workloads.bf16_bits(k),
                                    workloads.bf16_bits(v), b, hq, hk, s, s, d, d, True, 0.125,
                                    rows, window=128, sinks=sinks.double().numpy())
    got_o = np.stack([o[0, i, h] for (_, h, i) in rows])
    got_l = np.array([l[0, h, i] for (_, h, i) in rows])
    assert np.max(np.abs(got_o - o_ref)) <= TOL_O
    assert np.max(np.abs(got_l - l_ref)) <= TOL_LSE


@pytest.mark.parametrize("dqk,dv", [(64, 64), (128, 128)])
def test_wide_window_is_plain_attention_bitwise(dqk, dv):
    b, hq, hk, s = 2, 4, 2, 300
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, dqk, dv, seed=73)
    o0, l0 = b2.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    o1, l1 = b2.attn_fwd_window_sink(q.to(DEV), k.to(DEV), v.to(DEV), causal=True,
                                     window_left=s)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)


def test_sink_closed_form_against_plain_kernel():
    """LSE with a sink is logaddexp(LSE without, sink) and O scales by exp(LSE - LSE_sink)."""
    b, hq, hk, s, d = 2, 4, 2, 257, 128
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, d, d, seed=75)
    sinks = sinks_for(hq, 9)
    o0, l0 = b2.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    o1, l1 = gpu(q, k, v, True, -1, sinks, 1.0 / math.sqrt(d))
    l0 = l0.cpu().double().numpy()
    expect = np.logaddexp(l0, sinks.double().numpy()[None, :, None])
    assert np.max(np.abs(l1 - expect)) <= TOL_LSE
    f = np.exp(l0 - expect).transpose(0, 2, 1)[..., None]
    assert np.max(np.abs(o1 - o0.float().cpu().numpy() * f)) <= TOL_O


def test_no_keys_with_sinks():
    b, hq, hk, sq, d = 1, 4, 2, 9, 64
    q = torch.randn(b, sq, hq, d).to(torch.bfloat16)
    k = torch.empty(b, 0, hk, d, dtype=torch.bfloat16)
    sinks = sinks_for(hq, 10)
    o, l = gpu(q, k, k, True, 5, sinks, 0.125)
    assert np.all(o == 0.0)
    assert np.allclose(l, np.broadcast_to(sinks.numpy()[None, :, None], l.shape))
