"""Pins for the packed-sequence oracle (oracle.attn_varlen) against the dense oracle it composes:
equal-length sequences are exactly a dense batch, a sequence's result does not depend on its
neighbours or on its position, empty sequences behave as the dense rules say, and rows of no
sequence are left undefined."""
import numpy as np
import pytest
import torch

import oracle
import workloads


def bits(t):
    return workloads.bf16_bits(t)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_equal_a_dense_batch(causal):
    b, hq, hk, s, d = 3, 4, 2, 37, 64
    q, k, v = workloads.make_inputs(b, hq, hk, s, s, d, d, seed=11)
    o_d, l_d = oracle.attn_full(bits(q), bits(k), bits(v), b, hq, hk, s, s, d, d, causal, 0.125)
    cu = [0, s, 2 * s, 3 * s]
    o_v, l_v = oracle.attn_varlen(bits(q.reshape(b * s, hq, d)), bits(k.reshape(b * s, hk, d)),
                                  bits(v.reshape(b * s, hk, d)), cu, cu, hq, hk, d, d, causal,
                                  0.125)
    assert np.array_equal(o_v, o_d.reshape(b * s, hq, d))
    # dense LSE is [b, hq, s]; packed is [hq, total]
    assert np.array_equal(l_v, l_d.transpose(1, 0, 2).reshape(hq, b * s))


def test_sequence_order_does_not_matter():
    lq, lk = [5, 0, 19, 8], [7, 3, 19, 0]
    hq, hk, d = 2, 1, 64
    q, k, v, cq, ck = workloads.make_varlen_inputs(lq, lk, hq, hk, d, d, seed=5)
    o, l = oracle.attn_varlen(bits(q), bits(k), bits(v), cq.tolist(), ck.tolist(), hq, hk, d, d,
                              True, 0.3)
    perm = [2, 0, 3, 1]
    cq_l, ck_l = cq.tolist(), ck.tolist()
    qs = torch.cat([q[cq_l[i]:cq_l[i + 1]] for i in perm])
    ks = torch.cat([k[ck_l[i]:ck_l[i + 1]] for i in perm])
    vs = torch.cat([v[ck_l[i]:ck_l[i + 1]] for i in perm])
    cq2 = np.cumsum([0] + [lq[i] for i in perm])
    ck2 = np.cumsum([0] + [lk[i] for i in perm])
    o2, l2 = oracle.attn_varlen(bits(qs), bits(ks), bits(vs), cq2, ck2, hq, hk, d, d, True, 0.3)
    for new, i in enumerate(perm):
        a, bnd = cq_l[i], cq_l[i + 1]
        a2 = int(cq2[new])
        assert np.array_equal(o[a:bnd], o2[a2:a2 + bnd - a])
        assert np.array_equal(l[:, a:bnd], l2[:, a2:a2 + bnd - a])


def test_empty_sequences_and_rows_outside():
    hq, hk, d = 2, 2, 64
    lq, lk = [4, 3], [0, 5]  # the first sequence has no keys
    q, k, v, cq, ck = workloads.make_varlen_inputs(lq + [2], lk + [0], hq, hk, d, d, seed=9)
    # the last 2 query rows belong to no sequence (cu stops at 7)
    o, l = oracle.attn_varlen(bits(q), bits(k), bits(v), cq.tolist()[:3], ck.tolist()[:3], hq, hk,
                              d, d, False, 0.125)
    assert np.all(o[0:4] == 0.0) and np.all(np.isneginf(l[:, 0:4]))
    assert np.all(np.isfinite(o[4:7])) and np.all(np.isfinite(l[:, 4:7]))
    assert np.all(np.isnan(o[7:])) and np.all(np.isnan(l[:, 7:]))
    # the second sequence alone, dense, gives the same rows
    o1, l1 = oracle.attn_full(bits(q[4:7]), bits(k[0:5]), bits(v[0:5]), 1, hq, hk, 3, 5, d, d,
                              False, 0.125)
    assert np.array_equal(o[4:7], o1[0]) and np.array_equal(l[:, 4:7], l1[0])
