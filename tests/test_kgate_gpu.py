"""GPU parity of k_smooth_gate (the K-smoothing gate over a strided key sample) against the
oracle, through the C-ABI."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from libutil import ensure_built

ensure_built()
import head_attention_forward_flash_b200 as b2  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"
BAND = 1e-4  # |ratio - threshold| below this: either decision is valid


def k_inputs(b, hk, sk, d, seed, offset):
    g = torch.Generator().manual_seed(seed)
    noise = torch.randn(b, sk, hk, d, generator=g)
    off = offset * torch.randn(hk, d, generator=g)
    return (noise + off).to(torch.bfloat16)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("sk", [100, 2048, 2049, 4096, 5000])
@pytest.mark.parametrize("offset", [0.3, 2.0])
def test_gate_matches_oracle(d, sk, offset):
    b, hk, thr = 2, 3, 0.5
    k = k_inputs(b, hk, sk, d, seed=80 + sk + d, offset=offset)
    mean, gate, ratio = b2.k_smooth_gate(k.to(DEV), thr)
    torch.cuda.synchronize()
    mean, gate, ratio = mean.cpu().numpy(), gate.cpu().numpy(), ratio.cpu().numpy()
    _, _, r_ref, g_ref = oracle.k_gate(workloads.bf16_bits(k), b, hk, sk, d, thr)
    # the oracle's sampled mean of every head (threshold 0 turns every gate on)
    mu, _, _, _ = oracle.k_gate(workloads.bf16_bits(k), b, hk, sk, d, 0.0)
    stride = (sk + 2047) // 2048
    ks = k[:, ::stride].double().numpy()
    scale = np.maximum(np.abs(mu), np.abs(ks).mean(axis=1))  # the K-mean tolerance's scale
    assert np.max(np.abs(ratio - r_ref)) <= 1e-5
    clear = np.abs(r_ref - thr) > BAND
    assert np.array_equal(gate[clear], g_ref[clear])
    on = gate == 1
    assert np.all(mean[~on] == 0.0)
    assert np.all(np.abs(mean[on] - mu[on]) <= 1e-5 * scale[on])


def test_gate_long_context_k():
    """The FP8 recipe's K (b1 hk5 65536 keys d128): a stride-32 sample of 2048 rows."""
    b, hk, sk, d, thr = 1, 5, 65536, 128, 0.25
    k = k_inputs(b, hk, sk, d, seed=95, offset=0.5)
    mean, gate, ratio = b2.k_smooth_gate(k.to(DEV), thr)
    torch.cuda.synchronize()
    mean, gate, ratio = mean.cpu().numpy(), gate.cpu().numpy(), ratio.cpu().numpy()
    _, _, r_ref, g_ref = oracle.k_gate(workloads.bf16_bits(k), b, hk, sk, d, thr)
    mu, _, _, _ = oracle.k_gate(workloads.bf16_bits(k), b, hk, sk, d, 0.0)
    ks = k[:, ::32].double().numpy()
    scale = np.maximum(np.abs(mu), np.abs(ks).mean(axis=1))
    assert np.max(np.abs(ratio - r_ref)) <= 1e-5
    clear = np.abs(r_ref - thr) > BAND
    assert np.array_equal(gate[clear], g_ref[clear])
    on = gate == 1
    assert np.all(mean[~on] == 0.0)
    assert np.all(np.abs(mean[on] - mu[on]) <= 1e-5 * scale[on])


def test_gate_is_deterministic():
    k = k_inputs(1, 16, 4096, 256, seed=90, offset=1.0).to(DEV)
    a = b2.k_smooth_gate(k, 0.2)
    c = b2.k_smooth_gate(k, 0.2)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, c))


def test_gate_then_attention():
    """The gate's mean through k_smooth_sub into attention, against the oracle's own chain on
    sampled rows (the K-mean workload's shape at a smaller key count)."""
    b, hq, hk, s, d = 1, 4, 4, 1500, 128
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, d, d, seed=93, kmean=True)
    mean, gate, _ = b2.k_smooth_gate(k.to(DEV), 0.25)
    ks = b2.k_smooth_sub(k.to(DEV), mean)
    o, l = b2.attn_fwd(q.to(DEV), ks, v.to(DEV), causal=False)
    torch.cuda.synchronize()
    _, m32, _, g_ref = oracle.k_gate(workloads.bf16_bits(k), b, hk, s, d, 0.25)
    assert np.array_equal(gate.cpu().numpy(), g_ref) and g_ref.all()
    ks_ref = oracle.k_sub(workloads.bf16_bits(k), m32, b, hk, s, d)
    rows = np.array([(0, h, i) for h in range(hq) for i in (0, 1, 700, s - 1)], dtype=np.int64)
    o_ref, l_ref = oracle.attn_rows(workloads.bf16_bits(q), ks_ref, workloads.bf16_bits(v), b, hq,
                                    hk, s, s, d, d, False, 1.0 / np.sqrt(d), rows)
    o = o.float().cpu().numpy()
    l = l.cpu().numpy()
    assert np.max(np.abs(np.stack([o[0, i, h] for (_, h, i) in rows]) - o_ref)) <= 2e-2
    assert np.max(np.abs(np.array([l[0, h, i] for (_, h, i) in rows]) - l_ref)) <= 1e-3
