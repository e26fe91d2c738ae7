"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded bf16
inputs.

Tolerances (fixed for this method): max |O_gpu - O_oracle| <= 2e-2 and max |LSE_gpu - LSE_oracle|
<= 1e-3 on N(0,1) inputs; the K channel mean within 1e-5 relative, read as
|mean_gpu - mean_oracle| <= 1e-5 * max(|mean_oracle|, mean over s of |K[b,s,g,c]|); K' = K - mean
within one bf16 step (the GPU subtracts in fp32 and rounds once more than the oracle's fp64 path).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from libutil import ensure_built
from workloads import (HEAD_DIMS, bf16_bits, config, config_inputs, make_inputs, sample_rows,
                       tile_edge_rows)

pytestmark = pytest.mark.gpu

TOL_O = 2e-2
TOL_LSE = 1e-3


@pytest.fixture(scope="module")
def b2():
    ensure_built()
    import head_attention_forward_flash_b200 as mod
    assert mod.attn_debug_status() == 0
    yield mod
    assert mod.attn_debug_status() == 0, "a kernel reported a bounded-wait timeout"


def gpu_attn(b2, q, k, v, causal, scale):
    dev = torch.device("cuda:0")
    o, lse = b2.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale)
    torch.cuda.synchronize()
    return o.float().cpu().double().numpy(), lse.cpu().double().numpy()


def lse_err(a, b):
    both_inf = np.isneginf(a) & np.isneginf(b)
    d = np.abs(np.subtract(a, b, out=np.zeros_like(a, dtype=np.float64), where=~both_inf))
    return float(np.max(d)) if d.size else 0.0


def check_full(b2, b, hq, hk, sq, sk, dqk, dv, causal, scale, seed):
    q, k, v = make_inputs(b, hq, hk, sq, sk, dqk, dv, seed)
    o, lse = gpu_attn(b2, q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attn_full(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, sq, sk,
                                      dqk, dv, causal, scale)
    err_o = float(np.max(np.abs(o - o_ref))) if o.size else 0.0
    err_l = lse_err(lse, lse_ref)
    assert err_o <= TOL_O, f"max|dO| = {err_o}"
    assert err_l <= TOL_LSE, f"max|dLSE| = {err_l}"
    return o, lse


# Several tiles and ragged tails on both axes, every head-dim pair, causal and not, MHA and GQA.
SMALL = []
for (dqk, dv) in HEAD_DIMS:
    SMALL += [(2, 4, 2, 300, 300, dqk, dv, True), (1, 6, 2, 300, 300, dqk, dv, False),
              (1, 2, 2, 129, 1000, dqk, dv, True), (1, 2, 1, 257, 190, dqk, dv, False)]
SMALL += [(1, 8, 1, 1000, 127, 64, 64, True),   # sq > sk: fully masked rows at the top
          (1, 2, 2, 1, 1, 128, 128, False), (1, 2, 2, 1, 1, 128, 128, True),
          (3, 2, 2, 127, 1, 64, 64, False), (1, 3, 3, 64, 513, 192, 128, True),
          (2, 16, 2, 130, 130, 256, 256, True), (1, 1, 1, 384, 384, 64, 64, True)]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "b{}_hq{}_hk{}_sq{}_sk{}_d{}x{}_c{}".format(*c))
def test_small_shapes_match_oracle(b2, case):
    b, hq, hk, sq, sk, dqk, dv, causal = case
    check_full(b2, b, hq, hk, sq, sk, dqk, dv, causal, 1.0 / math.sqrt(dqk),
               seed=hash(case) % 100000)


# More work tiles than SMs, so each persistent CTA walks several tiles (and, with sq > sk, a mix
# of tiles with and without keys).
MULTI = [(1, 40, 8, 1000, 1000, dqk, dv, causal) for (dqk, dv) in HEAD_DIMS for causal in (True, False)]
MULTI += [(1, 64, 4, 1000, 200, 128, 128, True), (2, 24, 24, 700, 900, 64, 64, True)]


@pytest.mark.parametrize("case", MULTI, ids=lambda c: "b{}_hq{}_hk{}_sq{}_sk{}_d{}x{}_c{}".format(*c))
def test_many_tiles_per_cta_match_oracle(b2, case):
    b, hq, hk, sq, sk, dqk, dv, causal = case
    check_full(b2, b, hq, hk, sq, sk, dqk, dv, causal, 1.0 / math.sqrt(dqk),
               seed=hash(case) % 100000)


# d256 non-causal shapes whose units leave a partly filled last round on 148 SMs (158, 640 and
# 160 query tiles), with 3, 16 and 13 key blocks (ragged key tails), MHA and GQA; run twice,
# bitwise equal.
PARTIAL_ROUND = [(1, 1, 1, 128 * 158, 130, 256, 256), (2, 40, 4, 1000, 1000, 256, 256),
                 (1, 20, 5, 900, 777, 256, 256)]


@pytest.mark.parametrize("case", PARTIAL_ROUND,
                         ids=lambda c: "b{}_hq{}_hk{}_sq{}_sk{}_d{}x{}".format(*c))
def test_partial_last_round_matches_oracle(b2, case):
    b, hq, hk, sq, sk, dqk, dv = case
    o, lse = check_full(b2, b, hq, hk, sq, sk, dqk, dv, False, 1.0 / math.sqrt(dqk),
                        seed=hash(case) % 100000)
    q, k, v = make_inputs(b, hq, hk, sq, sk, dqk, dv, hash(case) % 100000)
    o2, lse2 = gpu_attn(b2, q, k, v, False, 1.0 / math.sqrt(dqk))
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2), "results must be deterministic"


@pytest.mark.parametrize("scale", [0.0, -0.08, 0.5])
def test_unusual_scales(b2, scale):
    check_full(b2, 1, 2, 1, 200, 200, 128, 128, True, scale, seed=31)


def test_config1_full(b2):
    c = config(1)
    check_full(b2, c["b"], c["hq"], c["hk"], c["sq"], c["sk"], c["dqk"], c["dv"], c["causal"],
               c["scale"], c["seed"])


def test_config1_matches_stored_oracle_values(b2):
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "mha_b1_h2_s128_d64_rows.json")))
    c = config(1)
    q, k, v = config_inputs(c)
    o, lse = gpu_attn(b2, q, k, v, c["causal"], c["scale"])
    for n, (bi, h, i) in enumerate(g["rows"]):
        assert np.max(np.abs(o[bi, i, h, g["channels"]] - np.array(g["o"][n]))) <= TOL_O
        assert abs(lse[bi, h, i] - g["lse"][n]) <= TOL_LSE


def _sampled(b2, n, n_pos, edges=False):
    """Workload n at full size on the GPU; the oracle on n_pos sampled query positions of every
    (batch, head), plus (edges) the first and last row of every 128-row query tile, so that a
    work unit the scheduler dropped or misplaced cannot escape."""
    c = config(n)
    q, k, v = config_inputs(c)
    kk = k
    if c["kmean"]:
        m64, m32 = oracle.k_mean(bf16_bits(k), c["b"], c["hk"], c["sk"], c["dqk"])
        kbits = oracle.k_sub(bf16_bits(k), m32, c["b"], c["hk"], c["sk"], c["dqk"])
        kk_ref = kbits
        dev = torch.device("cuda:0")
        kd = k.to(dev)
        mean = b2.k_smooth_mean(kd)
        kd2 = b2.k_smooth_sub(kd, mean)
        o, lse = b2.attn_fwd(q.to(dev), kd2, v.to(dev), causal=c["causal"], scale=c["scale"])
    else:
        kk_ref = bf16_bits(kk)
        dev = torch.device("cuda:0")
        o, lse = b2.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=c["causal"], scale=c["scale"])
    torch.cuda.synchronize()
    rows = sample_rows(c, n_pos).numpy()
    if edges:
        rows = np.unique(np.concatenate([rows, tile_edge_rows(c).numpy()]), axis=0)
    o_ref, lse_ref = oracle.attn_rows(bf16_bits(q), kk_ref, bf16_bits(v), c["b"], c["hq"], c["hk"],
                                      c["sq"], c["sk"], c["dqk"], c["dv"], c["causal"], c["scale"],
                                      rows)
    bi, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    o_g = o[torch.from_numpy(bi), torch.from_numpy(i), torch.from_numpy(h)].float().cpu().double()
    lse_g = lse[torch.from_numpy(bi), torch.from_numpy(h), torch.from_numpy(i)].cpu().double()
    err_o = float(np.max(np.abs(o_g.numpy() - o_ref)))
    err_l = lse_err(lse_g.numpy(), lse_ref)
    assert err_o <= TOL_O, f"config {n}: max|dO| = {err_o}"
    assert err_l <= TOL_LSE, f"config {n}: max|dLSE| = {err_l}"
    # properties that hold at any size: finite, and each channel within [min V, max V]
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("n,n_pos", [(2, 16), (3, 12), (4, 48), (5, 256)])
def test_full_size_configs_sampled_rows(b2, n, n_pos):
    _sampled(b2, n, n_pos)


@pytest.mark.parametrize("n", [3, 4, 5])
def test_full_size_every_query_tile(b2, n):
    """Full-size workloads with the first and last row of every query tile of every head checked
    against the oracle (the scheduler's unit orders at the real geometry: head-major for the
    many-head workload, weight-major for the five-head one)."""
    _sampled(b2, n, 8, edges=True)


def test_config2_every_row(b2):
    """The b8 hq48:hk8 2048^2 d64 causal workload compared with the oracle on every output row."""
    c = config(2)
    check_full(b2, c["b"], c["hq"], c["hk"], c["sq"], c["sk"], c["dqk"], c["dv"], c["causal"],
               c["scale"], c["seed"])


def test_k_mean_and_sub_match_oracle(b2):
    c = config(4)
    _, k, _ = config_inputs(c)
    b, hk, sk, d = c["b"], c["hk"], c["sk"], c["dqk"]
    m64, m32 = oracle.k_mean(bf16_bits(k), b, hk, sk, d)
    kd = k.cuda()
    mean = b2.k_smooth_mean(kd)
    mean2 = b2.k_smooth_mean(kd)
    torch.cuda.synchronize()
    assert torch.equal(mean, mean2), "k_smooth_mean must be deterministic"
    mg = mean.cpu().double().numpy()
    scale = np.maximum(np.abs(m64), np.abs(k.double().numpy()).mean(axis=1))
    assert np.all(np.abs(mg - m64) <= 1e-5 * scale), float(np.max(np.abs(mg - m64) / scale))
    ks = b2.k_smooth_sub(kd, mean)
    ref = oracle.k_sub(bf16_bits(k), m32, b, hk, sk, d)
    got = ks.cpu().view(torch.int16).numpy().view(np.uint16)
    gv = oracle.bf16_to_f64(got)
    rv = oracle.bf16_to_f64(ref)
    # One bf16 step of K', plus the (separately bounded) difference of the two means: where
    # K is close to its mean the subtraction cancels and the mean's own rounding shows through.
    dmean = np.abs(mg - m32.astype(np.float64))[:, None]  # [b, 1, hk, d]
    step = np.abs(rv) * 2.0 ** -7 + 2.0 ** -133 + dmean
    assert np.all(np.abs(gv - rv) <= step)
    assert np.mean(got == ref) > 0.99


@pytest.mark.parametrize("shape", [(2, 3, 100, 64), (1, 1, 1, 128), (3, 5, 17, 256)])
def test_k_mean_small_shapes(b2, shape):
    b, hk, sk, d = shape
    _, k, _ = make_inputs(b, 1, hk, 1, sk, d, d, seed=77, kmean=True)
    m64, _ = oracle.k_mean(bf16_bits(k), b, hk, sk, d)
    mg = b2.k_smooth_mean(k.cuda()).cpu().double().numpy()
    scale = np.maximum(np.abs(m64), np.abs(k.double().numpy()).mean(axis=1))
    assert np.all(np.abs(mg - m64) <= 1e-5 * scale)


@pytest.mark.parametrize("shape", [None, (2, 3, 100, 64), (1, 1, 1, 128), (3, 5, 17, 256),
                                   (1, 8, 4099, 128), (2, 40, 300, 256), (1, 5, 65536, 128)])
def test_k_mean_sub_fused_equals_two_calls(b2, shape):
    """The one-launch mean and subtraction gives the bits of k_smooth_mean then k_smooth_sub, at
    the K-mean workload's size (b1 hk16 4096 keys d256), at the long-context K (b1 hk5 65536
    keys d128: the bulk-copy row-chunk launch at full size) and at small and ragged shapes."""
    if shape is None:
        c = config(4)
        _, k, _ = config_inputs(c)
        b, hk, sk, d = c["b"], c["hk"], c["sk"], c["dqk"]
    else:
        b, hk, sk, d = shape
        _, k, _ = make_inputs(b, 1, hk, 1, sk, d, d, seed=78, kmean=True)
    kd = k.cuda()
    mean, ks = b2.k_smooth_mean_sub(kd)
    mean_ref = b2.k_smooth_mean(kd)
    ks_ref = b2.k_smooth_sub(kd, mean_ref)
    torch.cuda.synchronize()
    assert torch.equal(mean, mean_ref)
    assert torch.equal(ks.view(torch.int16), ks_ref.view(torch.int16))
    m64, m32 = oracle.k_mean(bf16_bits(k), b, hk, sk, d)
    mg = mean.cpu().double().numpy()
    scale = np.maximum(np.abs(m64), np.abs(k.double().numpy()).mean(axis=1))
    assert np.all(np.abs(mg - m64) <= 1e-5 * scale)
    if b * sk * hk * d <= 1 << 21:
        # the oracle's subtraction (exact, one rounding to bf16) with the GPU's mean; the kernel
        # rounds the fp32 difference to bf16, so a rare double rounding may move one unit
        ref = oracle.k_sub(bf16_bits(k), mean.cpu().numpy().astype(np.float32), b, hk, sk, d)
        got = ks.cpu().view(torch.int16).numpy().view(np.uint16)
        gv, rv = oracle.bf16_to_f64(got), oracle.bf16_to_f64(ref)
        assert np.all(np.abs(gv - rv) <= np.abs(rv) * 2.0 ** -7 + 2.0 ** -133)
        assert np.mean(got == ref) > 0.999


def test_kmean_leaves_output_invariant(b2):
    """Subtracting the K channel mean changes O only by rounding and shifts LSE by scale*q.mean."""
    c = config(4)
    b, hq, hk, s, d = 1, 4, 4, 512, 256
    q, k, v = make_inputs(b, hq, hk, s, s, d, d, seed=91, kmean=True)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o1, l1 = b2.attn_fwd(qd, kd, vd, scale=c["scale"])
    mean = b2.k_smooth_mean(kd)
    o2, l2 = b2.attn_fwd(qd, b2.k_smooth_sub(kd, mean), vd, scale=c["scale"])
    shift = c["scale"] * torch.einsum("bihc,bhc->bhi", qd.float(), mean)
    assert (o1.float() - o2.float()).abs().max().item() <= TOL_O
    assert (l1 - shift - l2).abs().max().item() <= 5e-2  # bf16 rounding of K' moves scores


def test_gqa_bitwise_equals_replicated_heads(b2):
    b, hq, hk, s, dqk, dv = 2, 6, 2, 333, 192, 128
    q, k, v = make_inputs(b, hq, hk, s, s, dqk, dv, seed=5)
    dev = torch.device("cuda:0")
    o1, l1 = b2.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    kr = k.repeat_interleave(hq // hk, dim=2).contiguous()
    vr = v.repeat_interleave(hq // hk, dim=2).contiguous()
    o2, l2 = b2.attn_fwd(q.to(dev), kr.to(dev), vr.to(dev), causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_deterministic_across_launches(b2):
    q, k, v = make_inputs(2, 8, 2, 700, 700, 128, 128, seed=6)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    outs = [b2.attn_fwd(qd, kd, vd, causal=True) for _ in range(3)]
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


def test_outputs_stay_inside_their_buffers(b2):
    """Canary bytes right after O and LSE are never written."""
    b, hq, hk, sq, sk, d = 1, 3, 1, 200, 260, 64
    q, k, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=8)
    dev = torch.device("cuda:0")
    n_o, n_l = b * sq * hq * d, b * hq * sq
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device=dev)
    l_buf = torch.full((n_l + 1024,), 7.0, dtype=torch.float32, device=dev)
    o = o_buf[:n_o].view(b, sq, hq, d)
    l = l_buf[:n_l].view(b, hq, sq)
    b2.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=True, out=o, lse=l)
    torch.cuda.synchronize()
    assert (o_buf[n_o:] == 7.0).all() and (l_buf[n_l:] == 7.0).all()
    o_ref, lse_ref = oracle.attn_full(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, sq, sk,
                                      d, d, True, 0.125)
    assert np.max(np.abs(o.float().cpu().double().numpy() - o_ref)) <= TOL_O


def test_empty_inputs(b2):
    dev = torch.device("cuda:0")
    # sk == 0: every row is empty -> O = 0, LSE = -inf
    q = torch.randn(1, 5, 2, 64, device=dev).to(torch.bfloat16)
    k = torch.empty(1, 0, 2, 64, device=dev, dtype=torch.bfloat16)
    v = torch.empty(1, 0, 2, 64, device=dev, dtype=torch.bfloat16)
    o = torch.full((1, 5, 2, 64), 3.0, device=dev, dtype=torch.bfloat16)
    o, l = b2.attn_fwd(q, k, v, out=o)
    torch.cuda.synchronize()
    assert (o == 0).all() and torch.isneginf(l).all()
    # sq == 0 and b == 0: nothing to do
    q0 = torch.empty(1, 0, 2, 64, device=dev, dtype=torch.bfloat16)
    k1 = torch.randn(1, 4, 2, 64, device=dev).to(torch.bfloat16)
    o0, l0 = b2.attn_fwd(q0, k1, k1)
    assert o0.shape == (1, 0, 2, 64) and l0.shape == (1, 2, 0)


def test_misaligned_view_is_refused(b2):
    dev = torch.device("cuda:0")
    buf = torch.zeros(64 * 16 * 2 + 1, device=dev, dtype=torch.bfloat16)
    qm = buf[1:].view(1, 16, 2, 64)  # 2-byte offset
    k = torch.zeros(1, 16, 2, 64, device=dev, dtype=torch.bfloat16)
    with pytest.raises(b2.B200AttnError) as e:
        b2.attn_fwd(qm, k, k)
    assert e.value.status == 5
