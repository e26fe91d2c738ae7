"""GPU parity of attn_fwd_varlen (packed sequences) against the oracle, through the C-ABI."""
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


def run(q, k, v, cq, ck, max_sq, causal, scale):
    o, l = b2.attn_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cq.to(DEV), ck.to(DEV), max_sq,
                              causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert b2.attn_debug_status() == 0
    return o.float().cpu().numpy(), l.cpu().numpy()


def compare(o, l, o_ref, l_ref, rows):
    o, l, o_ref, l_ref = o[rows], l[:, rows], o_ref[rows], l_ref[:, rows]
    assert np.max(np.abs(o - o_ref)) <= TOL_O
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isneginf(l), np.isneginf(l_ref))
    if fin.any():
        assert np.max(np.abs(l[fin] - l_ref[fin])) <= TOL_LSE


@pytest.mark.parametrize("dqk,dv", workloads.HEAD_DIMS)
@pytest.mark.parametrize("causal", [False, True])
def test_mixed_lengths(dqk, dv, causal):
    # lengths across tile edges, an empty sequence, and key lengths that differ from the query
    # lengths (bottom-right causal alignment; rows with no allowed key when sq_i > sk_i)
    lq = [1, 127, 128, 129, 300, 0, 64, 200]
    lk = [5, 200, 128, 100, 300, 3, 64, 0]
    hq, hk = 4, 2
    q, k, v, cq, ck = workloads.make_varlen_inputs(lq, lk, hq, hk, dqk, dv, seed=17 + dqk)
    scale = 1.0 / math.sqrt(dqk)
    o, l = run(q, k, v, cq, ck, max(lq), causal, scale)
    o_ref, l_ref = oracle.attn_varlen(workloads.bf16_bits(q), workloads.bf16_bits(k),
                                      workloads.bf16_bits(v), cq.tolist(), ck.tolist(), hq, hk,
                                      dqk, dv, causal, scale)
    compare(o, l, o_ref, l_ref, slice(0, sum(lq)))


def test_rows_outside_sequences_are_untouched():
    hq, hk, d = 2, 1, 64
    lq = [3, 7, 10, 5]  # rows 0-2 and 20-24 belong to no sequence
    q, k, v, _, _ = workloads.make_varlen_inputs(lq, [25], hq, hk, d, d, seed=3)
    cq = torch.tensor([3, 10, 20], dtype=torch.int32)
    ck = torch.tensor([0, 12, 25], dtype=torch.int32)
    out = torch.full((25, hq, d), 7.0, dtype=torch.bfloat16, device=DEV)
    lse = torch.full((hq, 25), 7.0, dtype=torch.float32, device=DEV)
    b2.attn_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cq.to(DEV), ck.to(DEV), 10, causal=True,
                       out=out, lse=lse)
    torch.cuda.synchronize()
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(o[:3] == 7.0) and np.all(o[20:] == 7.0)
    assert np.all(l[:, :3] == 7.0) and np.all(l[:, 20:] == 7.0)
    o_ref, l_ref = oracle.attn_varlen(workloads.bf16_bits(q), workloads.bf16_bits(k),
                                      workloads.bf16_bits(v), cq.tolist(), ck.tolist(), hq, hk, d,
                                      d, True, 1.0 / 8.0)
    compare(o, l, o_ref, l_ref, slice(3, 20))


@pytest.mark.parametrize("dqk,dv", [(64, 64), (128, 128)])
def test_equal_lengths_match_dense_bitwise(dqk, dv):
    b, hq, hk, s = 3, 4, 2, 200
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, dqk, dv, seed=23)
    o_d, l_d = b2.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=True)
    cu = torch.arange(0, (b + 1) * s, s, dtype=torch.int32)
    o_v, l_v = b2.attn_fwd_varlen(q.reshape(b * s, hq, dqk).to(DEV),
                                  k.reshape(b * s, hk, dqk).to(DEV),
                                  v.reshape(b * s, hk, dv).to(DEV), cu.to(DEV), cu.to(DEV), s,
                                  causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_v.view(b, s, hq, dv), o_d)
    assert torch.equal(l_v.view(hq, b, s).permute(1, 0, 2), l_d)


@pytest.mark.parametrize("b,s,causal", [(80, 1000, True), (80, 1000, False)])
def test_many_sequences_match_dense_bitwise(b, s, causal):
    """More (sequence, rank) classes than the cost-sorted schedule takes (80 x 4 = 320 > 256): the
    weight-major (causal) and round-robin (non-causal) orders; equal lengths match the dense
    batch bit for bit."""
    hq, hk, d = 2, 1, 64
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, d, d, seed=29)
    o_d, l_d = b2.attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal)
    cu = torch.arange(0, (b + 1) * s, s, dtype=torch.int32)
    o_v, l_v = b2.attn_fwd_varlen(q.reshape(b * s, hq, d).to(DEV), k.reshape(b * s, hk, d).to(DEV),
                                  v.reshape(b * s, hk, d).to(DEV), cu.to(DEV), cu.to(DEV), s,
                                  causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o_v.view(b, s, hq, d), o_d)
    assert torch.equal(l_v.view(hq, b, s).permute(1, 0, 2), l_d)


def test_no_keys_anywhere():
    hq, hk, d = 2, 2, 128
    q, k, v, cq, ck = workloads.make_varlen_inputs([5, 9], [0, 0], hq, hk, d, d, seed=4)
    o, l = run(q, torch.empty((0, hk, d), dtype=torch.bfloat16),
               torch.empty((0, hk, d), dtype=torch.bfloat16), cq, ck, 9, False, 0.1)
    assert np.all(o == 0.0) and np.all(np.isneginf(l))


def test_packed_workload_sampled_rows():
    """The packed-sequence benchmark workload at full size, checked on sampled rows of every
    sequence (first, last and 6 seeded positions, all heads) against the dense oracle of that
    sequence."""
    c = workloads.config(6)
    q, k, v, cq, ck = workloads.config_varlen_inputs(c)
    o, l = run(q, k, v, cq, ck, c["sq"], c["causal"], c["scale"])
    g = torch.Generator().manual_seed(2006)
    cql = cq.tolist()
    for i in range(c["b"]):
        a, e = cql[i], cql[i + 1]
        n = e - a
        pos = sorted({0, n - 1, *torch.randint(0, n, (6,), generator=g).tolist()})
        rows = np.array([(0, h, p) for h in range(c["hq"]) for p in pos], dtype=np.int64)
        o_ref, l_ref = oracle.attn_rows(workloads.bf16_bits(q[a:e]), workloads.bf16_bits(k[a:e]),
                                        workloads.bf16_bits(v[a:e]), 1, c["hq"], c["hk"], n, n,
                                        c["dqk"], c["dv"], c["causal"], c["scale"], rows)
        got_o = np.stack([o[a + p, h] for (_, h, p) in rows])
        got_l = np.array([l[h, a + p] for (_, h, p) in rows])
        assert np.max(np.abs(got_o - o_ref)) <= TOL_O
        assert np.max(np.abs(got_l - l_ref)) <= TOL_LSE
