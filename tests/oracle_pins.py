"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes a loaded oracle library (the real one, or a deliberately broken
build used by the mutation tests) and raises AssertionError when the oracle disagrees with

* torch's fp64 scaled-dot-product attention and ``torch.logsumexp`` (library routines),
* closed forms (uniform scores, causal row 0, one key, two keys),
* invariants (GQA equals explicit head replication, joint key permutation, convexity,
  batch/head independence, the K-mean shift identity), and
* numpy's fp64 mean and torch's fp32 -> bf16 round-to-nearest-even cast.

The attention the oracle implements is the standard scaled-dot-product attention that the
"Tune MHA config & small-head pipeline pathology" page benchmarks (shape notation in its
"Source of shapes" paragraph: sq, sk, d_head_qk, d_v, HQ/HK, causal c0/c1); the K mean is the
per-(batch, head) channel statistic of "[HIP] Mha v4: run the K-smoothing gate as one HIP
call" (Summary, commit message).
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from workloads import HEAD_DIMS, bf16_bits, make_inputs

TOL = 1e-12


def _run(lib, q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale):
    return oracle.attn_full(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, sq, sk, dqk, dv,
                            causal, scale, nthreads=4, lib=lib)


def _causal_keep(sq, sk):
    i = torch.arange(sq)[:, None]
    j = torch.arange(sk)[None, :]
    return j <= i + (sk - sq)


def _torch_reference(q, k, v, hq, hk, sq, sk, causal, scale):
    """torch fp64 SDPA (math path) and logsumexp, in BSHD / [b,hq,sq]."""
    Q = q.double().permute(0, 2, 1, 3)
    K = k.double().permute(0, 2, 1, 3)
    V = v.double().permute(0, 2, 1, 3)
    mask = _causal_keep(sq, sk) if causal else None
    with torch.no_grad():
        O = F.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=scale,
                                           enable_gqa=(hq != hk))
        Kr = K.repeat_interleave(hq // hk, dim=1)
        S = torch.matmul(Q, Kr.transpose(-1, -2)) * scale
        if causal:
            S = S.masked_fill(~mask, float("-inf"))
        L = torch.logsumexp(S, dim=-1)
    return O.permute(0, 2, 1, 3).numpy(), L.numpy()


def pin_sdpa(lib):
    """Oracle == torch fp64 SDPA on every head-dim pair, causal and not, MHA and GQA,
    square and non-square (bottom-right causal) shapes."""
    cases = []
    for (dqk, dv) in HEAD_DIMS:
        cases.append((2, 4, 2, 37, 37, dqk, dv, True))
        cases.append((1, 6, 2, 19, 41, dqk, dv, False))
    cases += [(2, 6, 3, 23, 50, 64, 64, True), (1, 2, 1, 33, 33, 192, 128, False),
              (1, 8, 8, 5, 70, 128, 128, True), (1, 3, 1, 64, 64, 64, 64, True)]
    for n, (b, hq, hk, sq, sk, dqk, dv, causal) in enumerate(cases):
        q, k, v = make_inputs(b, hq, hk, sq, sk, dqk, dv, seed=500 + n)
        scale = 1.0 / math.sqrt(dqk)
        o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale)
        o_ref, lse_ref = _torch_reference(q, k, v, hq, hk, sq, sk, causal, scale)
        err_o = np.max(np.abs(o - o_ref))
        err_l = np.max(np.abs(lse - lse_ref))
        assert err_o <= TOL, f"O vs torch SDPA: {err_o} on case {n}"
        if err_l > TOL:  # report where, and both values, before failing
            at = np.unravel_index(np.argmax(np.abs(lse - lse_ref)), lse.shape)
            raise AssertionError(f"LSE vs torch logsumexp: {err_l} on case {n} at {at}: oracle "
                                 f"{lse[at]!r}, torch {lse_ref[at]!r}")


def pin_uniform_scores(lib):
    """Q = 0 makes every allowed score equal: O is the mean of V over the allowed keys and
    LSE = ln(number of allowed keys)."""
    b, hq, hk, sq, sk, dqk, dv = 1, 2, 1, 9, 13, 64, 64
    _, k, v = make_inputs(b, hq, hk, sq, sk, dqk, dv, seed=7)
    q = torch.zeros((b, sq, hq, dqk), dtype=torch.bfloat16)
    vd = v.double().numpy()
    for causal in (False, True):
        o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, 0.125)
        for i in range(sq):
            n = min(sk, i + sk - sq + 1) if causal else sk
            want = vd[0, :n, 0, :].mean(axis=0)
            for h in range(hq):
                assert np.max(np.abs(o[0, i, h] - want)) <= TOL, "uniform-score mean of V"
                assert abs(lse[0, h, i] - math.log(n)) <= TOL, "uniform-score LSE"
    # scale = 0 is the same situation with nonzero Q
    q, k, v = make_inputs(b, hq, hk, sq, sk, dqk, dv, seed=8)
    o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, dqk, dv, False, 0.0)
    want = v.double().numpy()[0, :, 0, :].mean(axis=0)
    assert np.max(np.abs(o[0, :, 0] - want)) <= TOL
    assert np.max(np.abs(lse - math.log(sk))) <= TOL


def pin_causal_row0_and_single_key(lib):
    """Causal, sq = sk: row 0 sees key 0 only, so O = V[0] and LSE = scale * q0.k0.
    With sk = 1 (non-causal) every row returns V[0] and LSE = scale * q_i.k0."""
    b, hq, hk, s, dqk, dv = 2, 4, 2, 17, 128, 128
    q, k, v = make_inputs(b, hq, hk, s, s, dqk, dv, seed=9)
    scale = 0.37
    o, lse = _run(lib, q, k, v, b, hq, hk, s, s, dqk, dv, True, scale)
    qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
    for bi in range(b):
        for h in range(hq):
            g = h // (hq // hk)
            assert np.max(np.abs(o[bi, 0, h] - vd[bi, 0, g])) <= TOL, "causal row 0"
            want = scale * float(np.dot(qd[bi, 0, h], kd[bi, 0, g]))
            assert abs(lse[bi, h, 0] - want) <= TOL, "causal row 0 LSE"
    q, k, v = make_inputs(b, hq, hk, 5, 1, dqk, dv, seed=10)
    o, lse = _run(lib, q, k, v, b, hq, hk, 5, 1, dqk, dv, False, scale)
    qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
    for bi in range(b):
        for h in range(hq):
            g = h // (hq // hk)
            for i in range(5):
                assert np.max(np.abs(o[bi, i, h] - vd[bi, 0, g])) <= TOL, "single key"
                want = scale * float(np.dot(qd[bi, i, h], kd[bi, 0, g]))
                assert abs(lse[bi, h, i] - want) <= TOL, "single key LSE"


def pin_two_keys(lib):
    """Two keys: O = sigmoid(s0 - s1) * v0 + sigmoid(s1 - s0) * v1 and
    LSE = max(s0, s1) + log1p(exp(-|s0 - s1|))."""
    b, hq, hk, sq, sk, d = 1, 1, 1, 6, 2, 64
    q, k, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=11)
    scale = 0.5
    o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, d, d, False, scale)
    qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
    for i in range(sq):
        s0 = scale * float(np.dot(qd[0, i, 0], kd[0, 0, 0]))
        s1 = scale * float(np.dot(qd[0, i, 0], kd[0, 1, 0]))
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))
        w1 = 1.0 / (1.0 + math.exp(s0 - s1))
        assert np.max(np.abs(o[0, i, 0] - (w0 * vd[0, 0, 0] + w1 * vd[0, 1, 0]))) <= TOL
        assert abs(lse[0, 0, i] - (max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))))) <= TOL


def pin_large_scores(lib):
    """Scores of several hundred (exp would overflow without the max shift): the two-key
    closed form still holds, and LSE = max(s0, s1) + log1p(exp(-|s0 - s1|)) stays finite."""
    b, hq, hk, sq, sk, d = 1, 1, 1, 4, 2, 64
    q = torch.zeros((b, sq, hq, d), dtype=torch.bfloat16)
    k = torch.zeros((b, sk, hk, d), dtype=torch.bfloat16)
    v = torch.zeros((b, sk, hk, d), dtype=torch.bfloat16)
    q[0, :, 0, 0] = torch.tensor([8.0, -8.0, 4.0, 6.0])
    k[0, 0, 0, 0], k[0, 1, 0, 0] = 100.0, 99.5
    v[0, 0, 0, :], v[0, 1, 0, :] = 1.0, -2.0
    o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, d, d, False, 1.0)
    for i, qi in enumerate([8.0, -8.0, 4.0, 6.0]):
        s0, s1 = qi * 100.0, qi * 99.5
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))
        w1 = 1.0 / (1.0 + math.exp(s0 - s1))
        assert np.max(np.abs(o[0, i, 0] - (w0 * 1.0 + w1 * -2.0))) <= TOL, "large scores"
        assert abs(lse[0, 0, i] - (max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))))) <= 1e-10


def pin_gqa_replication(lib):
    """hq = 6 query heads over hk = 2 kv heads equals hq = hk = 6 with each kv head repeated
    for its group of 3 consecutive query heads."""
    b, hq, hk, sq, sk, dqk, dv = 2, 6, 2, 21, 29, 192, 128
    q, k, v = make_inputs(b, hq, hk, sq, sk, dqk, dv, seed=12)
    for causal in (False, True):
        o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, 0.07)
        kr = k.repeat_interleave(hq // hk, dim=2).contiguous()
        vr = v.repeat_interleave(hq // hk, dim=2).contiguous()
        o2, lse2 = _run(lib, q, kr, vr, b, hq, hq, sq, sk, dqk, dv, causal, 0.07)
        assert np.array_equal(o, o2) and np.array_equal(lse, lse2), "GQA head map"


def pin_permutation_and_independence(lib):
    """Non-causal O is invariant to a joint permutation of K/V rows; batch and head slices
    do not influence one another."""
    b, hq, hk, sq, sk, d = 2, 4, 4, 11, 40, 64
    q, k, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=13)
    o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, d, d, False, 0.125)
    perm = torch.randperm(sk, generator=torch.Generator().manual_seed(3))
    o2, lse2 = _run(lib, q, k[:, perm].contiguous(), v[:, perm].contiguous(), b, hq, hk, sq, sk,
                    d, d, False, 0.125)
    assert np.max(np.abs(o - o2)) <= TOL and np.max(np.abs(lse - lse2)) <= TOL, "permutation"
    q3, k3, v3 = q.clone(), k.clone(), v.clone()
    q3[1], k3[1], v3[1] = -q3[1], k3[1] * 2, v3[1] + 1  # change batch 1 only
    q3[0, :, 3] = 0                                     # and head 3 of batch 0
    k3[0, :, 3] = 1
    o3, lse3 = _run(lib, q3, k3, v3, b, hq, hk, sq, sk, d, d, False, 0.125)
    assert np.array_equal(o3[0, :, :3], o[0, :, :3]), "batch/head independence"
    assert np.array_equal(lse3[0, :3], lse[0, :3])


def pin_convexity(lib):
    """Each output channel lies between the min and max of V over the allowed keys."""
    b, hq, hk, sq, sk, d = 1, 3, 1, 30, 30, 128
    q, k, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=14)
    o, _ = _run(lib, q, k, v, b, hq, hk, sq, sk, d, d, True, 0.2)
    vd = v.double().numpy()
    for i in range(sq):
        lo = vd[0, :i + 1, 0].min(axis=0) - TOL
        hi = vd[0, :i + 1, 0].max(axis=0) + TOL
        assert np.all(o[0, i] >= lo) and np.all(o[0, i] <= hi), "convexity"


def pin_fully_masked_rows(lib):
    """Causal with sq > sk: rows i < sq - sk see no key, giving O = 0 and LSE = -inf; the
    remaining rows still match torch SDPA on the same (bottom-right) mask."""
    b, hq, hk, sq, sk, d = 1, 2, 2, 12, 5, 64
    q, k, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=15)
    o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, d, d, True, 0.125)
    assert np.all(o[0, :sq - sk] == 0.0) and np.all(np.isneginf(lse[0, :, :sq - sk]))
    o_ref, lse_ref = _torch_reference(q[:, sq - sk:].contiguous(), k, v, hq, hk, sk, sk, True,
                                      0.125)
    assert np.max(np.abs(o[:, sq - sk:] - o_ref)) <= TOL
    assert np.max(np.abs(lse[:, :, sq - sk:] - lse_ref)) <= TOL


def pin_kmean_shift_identity(lib):
    """Subtracting a per-channel constant c from every key leaves O unchanged and lowers LSE by
    scale * q.c (exact here: K and K - c are both exactly representable in bf16)."""
    b, hq, hk, sq, sk, d = 1, 2, 1, 16, 24, 64
    g = torch.Generator().manual_seed(16)
    kq = torch.randint(-16, 17, (b, sk, hk, d), generator=g).double() / 4.0
    c = torch.randint(-3, 4, (d,), generator=g).double()
    k = (kq + c).to(torch.bfloat16)
    k2 = kq.to(torch.bfloat16)
    assert torch.equal(k.double() - c, k2.double())
    q, _, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=17)
    for causal in (False, True):
        o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, d, d, causal, 0.125)
        o2, lse2 = _run(lib, q, k2, v, b, hq, hk, sq, sk, d, d, causal, 0.125)
        shift = 0.125 * np.einsum("bihc,c->bhi", q.double().numpy(), c.numpy())
        assert np.max(np.abs(o - o2)) <= 1e-12, "K-mean: O invariant"
        assert np.max(np.abs((lse - shift) - lse2)) <= 1e-12, "K-mean: LSE shift"


def pin_k_mean(lib):
    """Channel mean == numpy's fp64 mean of the bf16 values; a K whose rows are all equal
    returns that row exactly; K' = K - mean matches torch's fp32 subtract + bf16 cast
    wherever the fp32 difference is exact."""
    b, hk, sk, d = 2, 3, 77, 128
    _, k, _ = make_inputs(b, 1, hk, 1, sk, d, d, seed=18, kmean=True)
    m64, m32 = oracle.k_mean(bf16_bits(k), b, hk, sk, d, lib=lib)
    want = k.double().numpy().mean(axis=1)  # [b, hk, d]
    assert np.max(np.abs(m64 - want)) <= 1e-13 * max(1.0, np.max(np.abs(want))), "k mean"
    assert np.array_equal(m32, m64.astype(np.float32)), "k mean fp32 rounding"
    row = k[:, :1].expand(b, sk, hk, d).contiguous()
    r64, _ = oracle.k_mean(bf16_bits(row), b, hk, sk, d, lib=lib)
    assert np.array_equal(r64, row[:, 0].double().numpy()), "constant K rows"
    kout = oracle.k_sub(bf16_bits(k), m32, b, hk, sk, d, lib=lib)
    ref = (k.float() - torch.from_numpy(m32)[:, None]).to(torch.bfloat16)
    exact = ((k.double() - torch.from_numpy(m32).double()[:, None]) ==
             (k.float() - torch.from_numpy(m32)[:, None]).double())
    got = torch.from_numpy(kout.view(np.int16)).view(torch.bfloat16)
    assert torch.equal(got[exact], ref[exact]), "K' rounding"
    assert exact.float().mean() > 0.5


def pin_bf16_rne(lib):
    """Round-to-nearest-even to bf16 == torch's fp32 -> bf16 cast on fp32 inputs (one
    rounding), plus ties, subnormals, overflow and a case where rounding through fp32 first
    would give the wrong answer."""
    g = torch.Generator().manual_seed(19)
    x = torch.cat([torch.randn(4000, generator=g) * 10.0 ** torch.randint(-40, 38, (4000,),
                                                                        generator=g).float(),
                   torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 2.0 ** -134,
                                 3 * 2.0 ** -134, 3.3963e38, -3.3963e38, 1e-45, 0.0, -0.0])])
    got = oracle.bf16_rne(x.double().numpy(), lib=lib)
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want), "bf16 RNE vs torch"
    assert int(oracle.bf16_rne(np.array([1.0 + 2 ** -8]), lib=lib)[0]) == 0x3F80
    assert int(oracle.bf16_rne(np.array([1.0 + 3 * 2 ** -8]), lib=lib)[0]) == 0x3F82
    # 1 + 2^-8 + 2^-30 lies above the midpoint between 1 and 1 + 2^-7: the answer is 0x3F81,
    # while rounding to fp32 first would land exactly on the midpoint and give 0x3F80.
    assert int(oracle.bf16_rne(np.array([1.0 + 2 ** -8 + 2 ** -30]), lib=lib)[0]) == 0x3F81


def pin_rows_api(lib):
    """The row-sampling entry point returns the same values as the full one."""
    b, hq, hk, sq, sk, dqk, dv = 2, 4, 2, 20, 33, 256, 256
    q, k, v = make_inputs(b, hq, hk, sq, sk, dqk, dv, seed=20)
    o, lse = _run(lib, q, k, v, b, hq, hk, sq, sk, dqk, dv, True, 0.0625)
    rows = np.array([[0, 0, 0], [1, 3, 19], [0, 2, 7], [1, 1, 13]], dtype=np.int64)
    o_r, lse_r = oracle.attn_rows(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, sq, sk,
                                  dqk, dv, True, 0.0625, rows, nthreads=2, lib=lib)
    for n, (bi, h, i) in enumerate(rows):
        assert np.array_equal(o_r[n], o[bi, i, h]) and lse_r[n] == lse[bi, h, i]


def _band_keep(sq, sk, causal, window):
    """Allowed (i, j): j <= i + sk - sq when causal, j >= i + sk - sq - window when window >= 0."""
    i = torch.arange(sq)[:, None]
    j = torch.arange(sk)[None, :]
    keep = torch.ones(sq, sk, dtype=torch.bool)
    if causal:
        keep &= j <= i + (sk - sq)
    if window >= 0:
        keep &= j >= i + (sk - sq) - window
    return keep


def _brute_force_window_sink(q, k, v, hq, hk, sq, sk, causal, scale, window, sinks):
    """fp64 full-matrix softmax with a band mask and an extra sink column per head (numpy),
    written independently of the oracle: O [b,sq,hq,dv], LSE [b,hq,sq]."""
    Q = q.double().permute(0, 2, 1, 3).numpy()
    K = k.double().permute(0, 2, 1, 3).repeat_interleave(hq // hk, dim=1).numpy()
    V = v.double().permute(0, 2, 1, 3).repeat_interleave(hq // hk, dim=1).numpy()
    S = np.einsum("bhid,bhjd->bhij", Q, K) * scale
    keep = _band_keep(sq, sk, causal, window).numpy()
    S = np.where(keep[None, None], S, -np.inf)
    if sinks is not None:
        col = np.broadcast_to(np.asarray(sinks, np.float64)[None, :, None, None],
                              S.shape[:3] + (1,))
        S = np.concatenate([S, col], axis=-1)
        V = np.concatenate([V, np.zeros(V.shape[:2] + (1, V.shape[3]))], axis=2)
    m = np.max(S, axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(S - m)
    l = np.sum(w, axis=-1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        O = np.where(l > 0, np.einsum("bhij,bhjd->bhid", w, V) / np.where(l > 0, l, 1.0), 0.0)
        L = np.where(l[..., 0] > 0, m[..., 0] + np.log(np.where(l[..., 0] > 0, l[..., 0], 1.0)),
                     -np.inf)
    return O.transpose(0, 2, 1, 3), L


def pin_window_brute_force(lib):
    """Sliding window (with and without the causal bound, windows 0 .. past sk) == the numpy
    band-masked full softmax; sq != sk exercises the diagonal offset."""
    b, hq, hk, sq, sk, d = 1, 4, 2, 9, 13, 64
    q, k, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=41)
    for causal in (False, True):
        for window in (0, 1, 3, 7, 20):
            o, l = oracle.attn_full(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, sq, sk,
                                    d, d, causal, 0.2, nthreads=2, lib=lib, window=window)
            o_ref, l_ref = _brute_force_window_sink(q, k, v, hq, hk, sq, sk, causal, 0.2, window,
                                                    None)
            assert np.max(np.abs(o - o_ref)) < 1e-12
            assert np.array_equal(np.isneginf(l), np.isneginf(l_ref))
            fin = np.isfinite(l_ref)
            assert np.max(np.abs(l[fin] - l_ref[fin])) < 1e-12


def pin_window_zero_is_the_diagonal(lib):
    """Causal with window 0: every row sees only its diagonal key, so O is that key's V row
    exactly and LSE is that key's scaled score."""
    b, hq, hk, s, d = 1, 2, 2, 6, 64
    q, k, v = make_inputs(b, hq, hk, s, s, d, d, seed=43)
    o, l = oracle.attn_full(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, s, s, d, d, True,
                            0.3, nthreads=2, lib=lib, window=0)
    vd, qd, kd = v.double().numpy(), q.double().numpy(), k.double().numpy()
    for h in range(hq):
        for i in range(s):
            assert np.array_equal(o[0, i, h], vd[0, i, h])
            assert abs(l[0, h, i] - 0.3 * float(np.dot(qd[0, i, h], kd[0, i, h]))) < 1e-12


def pin_sink_closed_form(lib):
    """A sink logit sigma joins the denominator: LSE_sink = logaddexp(LSE, sigma) and
    O_sink = O * exp(LSE - LSE_sink), exactly; rows with no allowed key give O = 0 and
    LSE = sigma; the numpy brute force with a sink column agrees."""
    b, hq, hk, sq, sk, d = 2, 4, 2, 11, 7, 64  # sq > sk: causal rows 0..3 have no key
    q, k, v = make_inputs(b, hq, hk, sq, sk, d, d, seed=47)
    sinks = np.array([-1.5, 0.0, 2.25, 30.0])
    for causal in (False, True):
        o0, l0 = oracle.attn_full(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, sq, sk, d,
                                  d, causal, 0.125, nthreads=2, lib=lib)
        o1, l1 = oracle.attn_full(bf16_bits(q), bf16_bits(k), bf16_bits(v), b, hq, hk, sq, sk, d,
                                  d, causal, 0.125, nthreads=2, lib=lib, sinks=sinks)
        expect_l = np.logaddexp(l0, sinks[None, :, None])
        assert np.max(np.abs(l1 - expect_l)) < 1e-12
        scale_o = np.exp(l0 - expect_l).transpose(0, 2, 1)[..., None]  # [b, sq, hq, 1]
        assert np.max(np.abs(o1 - o0 * np.where(np.isfinite(scale_o), scale_o, 0.0))) < 1e-12
        o_ref, l_ref = _brute_force_window_sink(q, k, v, hq, hk, sq, sk, causal, 0.125, -1, sinks)
        assert np.max(np.abs(o1 - o_ref)) < 1e-12 and np.max(np.abs(l1 - l_ref)) < 1e-12
        if causal:
            assert np.all(o1[:, :4] == 0.0)
            assert np.array_equal(l1[:, :, :4], np.broadcast_to(sinks[None, :, None], (b, hq, 4)))


def pin_k_gate(lib):
    """K-smoothing gate: constant key rows put all of K's energy in the mean (ratio 1, gate on
    at a threshold of exactly 1, output = that row); rows in +/- pairs have zero mean (ratio 0,
    output 0); two alternating values a, b in one channel give the closed form
    r = (a + b)^2 / (2 (a^2 + b^2)); at 4096 keys every 2nd key is sampled (changing an
    unsampled key changes nothing, a sampled one changes the mean); with threshold 0 the output
    is numpy's fp64 mean over all keys (sk <= 2048)."""
    b, hk, d = 1, 2, 64
    g = torch.Generator().manual_seed(51)
    row = torch.randn(hk, d, generator=g).to(torch.bfloat16)
    const = row.expand(b, 100, hk, d).contiguous()
    m64, m32, r, gate = oracle.k_gate(bf16_bits(const), b, hk, 100, d, 1.0, lib=lib)
    assert np.all(r == 1.0) and np.all(gate == 1)
    assert np.array_equal(m32, row.float().numpy()[None])
    _, _, _, gate = oracle.k_gate(bf16_bits(const), b, hk, 100, d, 1.0 + 1e-12, lib=lib)
    assert np.all(gate == 0)
    pm = torch.stack([row, -row], dim=0).repeat(50, 1, 1)[None].contiguous()  # [1,100,hk,d]
    m64, m32, r, gate = oracle.k_gate(bf16_bits(pm), b, hk, 100, d, 1e-9, lib=lib)
    assert np.all(r == 0.0) and np.all(gate == 0) and np.all(m64 == 0.0)
    a_, b_ = 3.0, -0.5
    two = torch.zeros(b, 64, hk, d)
    two[:, 0::2, :, 0] = a_
    two[:, 1::2, :, 0] = b_
    _, _, r, _ = oracle.k_gate(bf16_bits(two.to(torch.bfloat16)), b, hk, 64, d, 0.5, lib=lib)
    assert np.allclose(r, (a_ + b_) ** 2 / (2 * (a_ ** 2 + b_ ** 2)), rtol=0, atol=1e-15)
    sk = 4096
    big = torch.randn(b, sk, hk, d, generator=g).to(torch.bfloat16)
    m_ref, _, r_ref, _ = oracle.k_gate(bf16_bits(big), b, hk, sk, d, 0.0, lib=lib)
    unsampled = big.clone()
    unsampled[:, 3] += 5.0
    m_u, _, r_u, _ = oracle.k_gate(bf16_bits(unsampled), b, hk, sk, d, 0.0, lib=lib)
    assert np.array_equal(m_u, m_ref) and np.array_equal(r_u, r_ref)
    sampled = big.clone()
    sampled[:, 2] += 5.0
    m_s, _, _, _ = oracle.k_gate(bf16_bits(sampled), b, hk, sk, d, 0.0, lib=lib)
    assert not np.array_equal(m_s, m_ref)
    assert np.allclose(m_ref, big[:, 0::2].double().numpy().mean(axis=1), rtol=0, atol=1e-14)
    small = big[:, :1500].contiguous()
    m_a, _, _, gate = oracle.k_gate(bf16_bits(small), b, hk, 1500, d, 0.0, lib=lib)
    assert np.all(gate == 1)
    assert np.allclose(m_a, small.double().numpy().mean(axis=1), rtol=0, atol=1e-14)


ALL_PINS = [pin_sdpa, pin_uniform_scores, pin_causal_row0_and_single_key, pin_two_keys, pin_large_scores,
            pin_gqa_replication, pin_permutation_and_independence, pin_convexity,
            pin_fully_masked_rows, pin_kmean_shift_identity, pin_k_mean, pin_bf16_rne,
            pin_rows_api, pin_window_brute_force, pin_window_zero_is_the_diagonal,
            pin_sink_closed_form, pin_k_gate]
