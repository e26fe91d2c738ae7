"""Failure detection without a GPU fault: a launch whose producer loads nothing (armed by
attn_debug_starve) makes every bounded wait give up after a short limit; the host reads
ERR_TIMEOUT, and the next, normal launch on the same context is correct."""
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


@pytest.mark.parametrize("dqk,dv", workloads.HEAD_DIMS)
def test_starved_launch_times_out_and_context_survives(dqk, dv):
    b, hq, hk, s = 1, 4, 2, 300
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, dqk, dv, seed=97)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    assert b2.attn_debug_status() == 0
    b2.attn_debug_starve(20000)  # 20 ms per wait
    b2.attn_fwd(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    assert b2.attn_debug_status() == 10  # B200ATTN_ERR_TIMEOUT, then cleared
    o, l = b2.attn_fwd(qd, kd, vd, causal=True)
    torch.cuda.synchronize()
    assert b2.attn_debug_status() == 0
    o_ref, l_ref = oracle.attn_full(workloads.bf16_bits(q), workloads.bf16_bits(k),
                                    workloads.bf16_bits(v), b, hq, hk, s, s, dqk, dv, True,
                                    1.0 / math.sqrt(dqk))
    assert np.max(np.abs(o.float().cpu().numpy() - o_ref)) <= 2e-2
    assert np.max(np.abs(l.cpu().numpy() - l_ref)) <= 1e-3
