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
