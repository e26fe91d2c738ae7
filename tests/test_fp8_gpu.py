"""FP8 (E4M3) recipe on the GPU against the oracle: the quantiser bit for bit, and the attention
on oracle-made codes within the derived bound. The bound is one E4M3 rounding of each softmax
weight (oracle.fp8.p_rounding_bound), plus O's own bf16 rounding and fp32 accumulation slack;
LSE within 1e-3, as for bf16 inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from workloads import bf16_bits, config, config_inputs, make_inputs, sample_rows

pytestmark = pytest.mark.gpu

LSE_TOL = 1e-3
ACC_SLACK = 2e-3  # fp32 accumulation order, the exp2 approximations, the V descale product


@pytest.fixture(scope="module")
def b2():
    from libutil import ensure_built
    ensure_built()
    import head_attention_forward_flash_b200 as mod
    return mod


def _u8(t):
    return t.cpu().numpy().astype(np.uint8)


@pytest.mark.parametrize("shape,with_mean", [
    ((2, 300, 3, 128), False), ((2, 300, 3, 128), True), ((1, 1000, 5, 64), True),
    ((1, 77, 2, 256), False), ((3, 1, 4, 128), True), ((1, 4096, 16, 128), True),
])
def test_quantize_bit_exact(b2, shape, with_mean):
    b, s, h, d = shape
    g = torch.Generator().manual_seed(5000 + s)
    x = (torch.randn((b, s, h, d), generator=g) * 3.0
         + torch.randn((1, 1, h, d), generator=g) * 2.0).to(torch.bfloat16)
    x[0, :, 0, :] *= 1e-3  # a head of small values (subnormal E4M3 codes)
    if h > 1:
        x[-1, :, h - 1, :] = 0  # an all-zero head
    mean32 = None
    if with_mean:
        mean32 = oracle.k_mean(bf16_bits(x), b, h, s, d)[1]
    ref_codes, ref_ds = fp8.quantize(bf16_bits(x), b, s, h, d, mean32=mean32)
    mean_t = torch.from_numpy(mean32).cuda() if with_mean else None
    codes, ds = b2.fp8_quantize(x.cuda(), mean=mean_t)
    codes2, ds2 = b2.fp8_quantize(x.cuda(), mean=mean_t)
    torch.cuda.synchronize()
    got = _u8(codes)
    assert np.array_equal(ds.cpu().numpy(), ref_ds)
    assert np.array_equal(got, ref_codes), int(np.sum(got != ref_codes))
    assert torch.equal(codes, codes2) and torch.equal(ds, ds2)


def test_quantize_empty_sequence(b2):
    x = torch.empty((2, 0, 3, 128), dtype=torch.bfloat16, device="cuda")
    codes, ds = b2.fp8_quantize(x)
    torch.cuda.synchronize()
    assert codes.shape == (2, 0, 3, 128) and torch.all(ds == 1.0)


def _quantized(b, hq, hk, sq, sk, d, seed, kmean=False):
    q, k, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=seed, kmean=kmean)
    q8, dq = fp8.quantize(bf16_bits(q), b, sq, hq, d)
    mean32 = oracle.k_mean(bf16_bits(k), b, hk, sk, d)[1] if kmean else None
    k8, dk = fp8.quantize(bf16_bits(k), b, sk, hk, d, mean32=mean32)
    v8, dv = fp8.quantize(bf16_bits(v), b, sk, hk, d)
    return q8, k8, v8, dq, dk, dv


def _run(b2, q8, k8, v8, dq, dk, dv, causal, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    o, lse = b2.attn_fwd_fp8(t(q8), t(k8), t(v8), t(dq), t(dk), t(dv), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert b2.attn_debug_status() == 0
    return o.float().cpu().double().numpy(), lse.cpu().double().numpy()


def _check(o, lse, o_ref, lse_ref, bound):
    lim = bound + np.abs(o_ref) * 2.0 ** -8 + ACC_SLACK
    err = np.abs(o - o_ref)
    assert np.all(err <= lim), (float(np.max(err - lim)), float(np.max(err)))
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.max(np.abs(lse[fin] - lse_ref[fin]), initial=0.0) <= LSE_TOL


@pytest.mark.parametrize("b,hq,hk,sq,sk,causal,scale", [
    (1, 2, 2, 128, 128, False, None),
    (2, 4, 2, 300, 300, True, None),
    (2, 4, 2, 300, 300, False, None),
    (1, 6, 2, 200, 333, True, None),    # ragged, sq < sk (bottom-right causal)
    (1, 3, 1, 333, 200, True, None),    # sq > sk: fully masked rows
    (1, 2, 1, 700, 700, True, -0.07),   # negative scale (MMA negate)
    (1, 2, 2, 513, 513, False, 0.0),    # scale 0: uniform weights
])
def test_attention_parity(b2, b, hq, hk, sq, sk, causal, scale):
    d = 128
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    q8, k8, v8, dq, dk, dv = _quantized(b, hq, hk, sq, sk, d, seed=6000 + sq + sk)
    o, lse = _run(b2, q8, k8, v8, dq, dk, dv, causal, scale)
    o_ref, lse_ref = fp8.attn_full(q8, k8, v8, dq, dk, dv, b, hq, hk, sq, sk, d, d, causal, scale)
    rows = np.array([[bi, h, i] for bi in range(b) for h in range(hq) for i in range(sq)])
    bound = fp8.p_rounding_bound(q8, k8, v8, dq, dk, dv, b, hq, hk, sq, sk, d, d, causal, scale,
                                 rows).reshape(b, hq, sq, d).transpose(0, 2, 1, 3)
    _check(o, lse, o_ref, lse_ref, bound)


def test_attention_parity_long_sampled(b2):
    """The FP8 long-context workload's shape (5 heads, 65536^2, causal) on sampled rows."""
    c = config(8)
    b, hq, hk, s, d = c["b"], c["hq"], c["hk"], c["sq"], c["dqk"]
    q, k, v = config_inputs(c)
    q8, dq = fp8.quantize(bf16_bits(q), b, s, hq, d)
    k8, dk = fp8.quantize(bf16_bits(k), b, s, hk, d)
    v8, dv = fp8.quantize(bf16_bits(v), b, s, hk, d)
    o, lse = _run(b2, q8, k8, v8, dq, dk, dv, True, c["scale"])
    rows = sample_rows(c).numpy()
    o_ref, lse_ref = fp8.attn_rows(q8, k8, v8, dq, dk, dv, b, hq, hk, s, s, d, d, True,
                                   c["scale"], rows)
    bound = fp8.p_rounding_bound(q8, k8, v8, dq, dk, dv, b, hq, hk, s, s, d, d, True, c["scale"],
                                 rows)
    got_o = o[rows[:, 0], rows[:, 2], rows[:, 1]]
    got_l = lse[rows[:, 0], rows[:, 1], rows[:, 2]]
    _check(got_o, got_l, o_ref, lse_ref, bound)


def test_recipe_on_gpu_against_bf16(b2):
    """The whole recipe on the GPU (K mean, smoothing, quantisation, FP8 attention) stays as close
    to the bf16 result as the oracle's own FP8 recipe, within the parity bound."""
    b, hq, hk, s, d = 1, 4, 2, 640, 128
    q, k, v = make_inputs(b, hq, hk, s, s, d, d, seed=6100, kmean=True)
    scale = 1.0 / math.sqrt(d)
    o_bf, _ = oracle.attn_full(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, s, s, d, d,
                               True, scale)
    q8, k8, v8, dq, dk, dv = _quantized(b, hq, hk, s, s, d, seed=6100, kmean=True)
    o_or, _ = fp8.attn_full(q8, k8, v8, dq, dk, dv, b, hq, hk, s, s, d, d, True, scale)
    kd = k.cuda()
    mean = b2.k_smooth_mean(kd)
    gq, gdq = b2.fp8_quantize(q.cuda())
    gk, gdk = b2.fp8_quantize(kd, mean=mean)
    gv, gdv = b2.fp8_quantize(v.cuda())
    og, _ = b2.attn_fwd_fp8(gq, gk, gv, gdq, gdk, gdv, causal=True, scale=scale)
    torch.cuda.synchronize()
    err_gpu = float(np.max(np.abs(og.float().cpu().double().numpy() - o_bf)))
    err_or = float(np.max(np.abs(o_or - o_bf)))
    assert err_gpu <= err_or + 2e-2, (err_gpu, err_or)


def test_attention_no_keys(b2):
    # sk = 0: every row is empty (O = 0, LSE = -inf); K and V have no rows
    q8 = torch.zeros((1, 40, 2, 128), dtype=torch.uint8, device="cuda")
    k8 = torch.empty((1, 0, 1, 128), dtype=torch.uint8, device="cuda")
    dq = torch.ones((1, 2), dtype=torch.float32, device="cuda")
    dk = torch.ones((1, 1), dtype=torch.float32, device="cuda")
    o, lse = b2.attn_fwd_fp8(q8, k8, k8, dq, dk, dk, causal=False)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
