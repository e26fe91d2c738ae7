"""Writes tests/golden/mha_b1_h2_s128_d64_rows.json from the CPU oracle alone.

The workload is the smallest benchmark shape (b=1, hq=hk=2, sq=sk=128, dqk=dv=64,
non-causal, scale 1/sqrt(64), inputs iid N(0,1) cast to bf16 from seed 1001), the
correctness-only case beside the shapes of "Tune MHA config & small-head pipeline pathology"
(Test Plan). The pages print no output values for any shape, so the stored values are the
oracle's; they guard the oracle against drift and give the GPU tests a fixed expectation.
Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from workloads import bf16_bits, config, config_inputs  # noqa: E402

ROWS = [(0, 0, 0), (0, 1, 0), (0, 0, 1), (0, 1, 63), (0, 0, 64), (0, 1, 127), (0, 0, 127)]
CHANNELS = [0, 1, 31, 32, 63]


def main():
    c = config(1)
    q, k, v = config_inputs(c)
    o, lse = oracle.attn_rows(bf16_bits(q), bf16_bits(k), bf16_bits(v), c["b"], c["hq"], c["hk"],
                              c["sq"], c["sk"], c["dqk"], c["dv"], c["causal"], c["scale"], ROWS,
                              nthreads=1)
    out = {
        "workload": c["workload"], "seed": c["seed"], "scale": c["scale"],
        "source": "CPU oracle (oracle/attn_oracle.c), written by tests/golden/make_golden.py",
        "rows": [list(r) for r in ROWS], "channels": CHANNELS,
        "o": [[float(o[n, ch]) for ch in CHANNELS] for n in range(len(ROWS))],
        "lse": [float(x) for x in lse],
    }
    with open(os.path.join(HERE, "mha_b1_h2_s128_d64_rows.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
