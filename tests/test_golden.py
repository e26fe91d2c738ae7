"""The stored oracle fixture still matches the oracle (guards the oracle against drift)."""
import json
import os

import numpy as np

import oracle
from workloads import bf16_bits, config, config_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mha_b1_h2_s128_d64_rows.json")


def test_golden_rows_match_oracle():
    g = json.load(open(GOLDEN))
    c = config(1)
    q, k, v = config_inputs(c)
    o, lse = oracle.attn_rows(bf16_bits(q), bf16_bits(k), bf16_bits(v), c["b"], c["hq"], c["hk"],
                              c["sq"], c["sk"], c["dqk"], c["dv"], c["causal"], c["scale"],
                              g["rows"], nthreads=2)
    assert np.allclose(o[:, g["channels"]], np.array(g["o"]), rtol=0, atol=1e-13)
    assert np.allclose(lse, np.array(g["lse"]), rtol=0, atol=1e-13)


GOLDEN_FP8 = os.path.join(os.path.dirname(__file__), "golden", "fp8_b1_h2_s128_d128.json")


def test_golden_fp8_matches_oracle():
    """The FP8 recipe fixture (descales, code digests, sampled attention values) still matches
    the oracle."""
    import hashlib

    from oracle import fp8
    from workloads import make_inputs

    g = json.load(open(GOLDEN_FP8))
    b, h, s, d = g["shape"]
    q, k, v = make_inputs(b, h, h, s, s, d, d, seed=g["seed"], kmean=True)
    m32 = oracle.k_mean(bf16_bits(k), b, h, s, d)[1]
    q8, dq = fp8.quantize(bf16_bits(q), b, s, h, d)
    k8, dk = fp8.quantize(bf16_bits(k), b, s, h, d, mean32=m32)
    v8, dv = fp8.quantize(bf16_bits(v), b, s, h, d)
    for name, codes, ds in (("q", q8, dq), ("k", k8, dk), ("v", v8, dv)):
        assert hashlib.sha256(codes.tobytes()).hexdigest() == g["codes_sha256"][name]
        assert ds.ravel().tolist() == g["descale"][name]
    assert k8[0, 0, 0, :16].tolist() == g["k_codes_row0_head0"]
    o, lse = fp8.attn_rows(q8, k8, v8, dq, dk, dv, b, h, h, s, s, d, d, g["causal"], g["scale"],
                           g["rows"], nthreads=2)
    assert np.allclose(o[:, g["channels"]], np.array(g["o"]), rtol=0, atol=1e-13)
    assert np.allclose(lse, np.array(g["lse"]), rtol=0, atol=1e-13)
