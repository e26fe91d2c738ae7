"""No kernel writes past the end of its outputs: every output is placed at the start of a larger
byte buffer pre-filled with a canary pattern, and the bytes after the tensor must be unchanged
after the call (ragged sizes, every head-dim pair, packed sequences, the FP8 recipe and the K
mean)."""
import math

import pytest
import torch

from workloads import HEAD_DIMS, make_inputs, make_varlen_inputs

pytestmark = pytest.mark.gpu

CANARY = 0xA5
PAD = 64 * 1024  # bytes after each output


@pytest.fixture(scope="module")
def b2():
    from libutil import ensure_built
    ensure_built()
    import head_attention_forward_flash_b200 as mod
    return mod


def canaried(shape, dtype):
    """(tensor of `shape` at the start of a canary-filled buffer, the raw byte buffer, its
    byte size)."""
    nbytes = math.prod(shape) * torch.tensor([], dtype=dtype).element_size()
    raw = torch.full((nbytes + PAD,), CANARY, dtype=torch.uint8, device="cuda")
    return raw[:nbytes].view(dtype).view(shape), raw, nbytes


def intact(raw, nbytes):
    torch.cuda.synchronize()
    return bool(torch.all(raw[nbytes:] == CANARY))


@pytest.mark.parametrize("dqk,dv", HEAD_DIMS)
@pytest.mark.parametrize("causal", [True, False])
def test_attn_fwd_writes_nothing_past_outputs(b2, dqk, dv, causal):
    b, hq, hk, sq, sk = 2, 3, 1, 200, 333
    q, k, v = (t.cuda() for t in make_inputs(b, hq, hk, sq, sk, dqk, dv, seed=91))
    o, o_raw, o_n = canaried((b, sq, hq, dv), torch.bfloat16)
    lse, l_raw, l_n = canaried((b, hq, sq), torch.float32)
    b2.attn_fwd(q, k, v, causal=causal, out=o, lse=lse)
    assert intact(o_raw, o_n) and intact(l_raw, l_n)
    assert b2.attn_debug_status() == 0


def test_varlen_writes_nothing_past_outputs(b2):
    q, k, v, cu_q, cu_k = make_varlen_inputs([130, 1, 257], [130, 1, 257], 4, 2, 128, 128, seed=92)
    total = q.shape[0]
    o, o_raw, o_n = canaried((total, 4, 128), torch.bfloat16)
    lse, l_raw, l_n = canaried((4, total), torch.float32)
    b2.attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(), 257, causal=True,
                       out=o, lse=lse)
    assert intact(o_raw, o_n) and intact(l_raw, l_n)


def test_fp8_writes_nothing_past_outputs(b2):
    b, h, s, d = 1, 3, 333, 128
    q, k, v = (t.cuda() for t in make_inputs(b, h, h, s, s, d, d, seed=93))
    mean = b2.k_smooth_mean(k)
    codes = []
    for x, m in ((q, None), (k, mean), (v, None)):
        c, c_raw, c_n = canaried((b, s, h, d), torch.uint8)
        ds, d_raw, d_n = canaried((b, h), torch.float32)
        b2.fp8_quantize(x, mean=m, out=c, descale=ds)
        assert intact(c_raw, c_n) and intact(d_raw, d_n)
        codes.append((c, ds))
    (q8, dq), (k8, dk), (v8, dvs) = codes
    o, o_raw, o_n = canaried((b, s, h, d), torch.bfloat16)
    lse, l_raw, l_n = canaried((b, h, s), torch.float32)
    b2.attn_fwd_fp8(q8, k8, v8, dq, dk, dvs, causal=True, out=o, lse=lse)
    assert intact(o_raw, o_n) and intact(l_raw, l_n)
    assert b2.attn_debug_status() == 0


def test_k_mean_writes_nothing_past_output(b2):
    _, k, _ = make_inputs(2, 1, 3, 1, 77, 64, 64, seed=94, kmean=True)
    mean, m_raw, m_n = canaried((2, 3, 64), torch.float32)
    b2.k_smooth_mean(k.cuda(), mean)
    assert intact(m_raw, m_n)
