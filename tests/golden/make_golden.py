"""Writes tests/golden/mha_b1_h2_s128_d64_rows.json and tests/golden/fp8_b1_h2_s128_d128.json
from the CPU oracle alone.

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


FP8_SEED = 1801
FP8_ROWS = [(0, 0, 0), (0, 1, 5), (0, 0, 64), (0, 1, 127)]
FP8_CHANNELS = [0, 7, 64, 127]


def main_fp8():
    """The FP8 recipe on a small causal shape (b=1, hq=hk=2, sq=sk=128, d=128, seed 1801, the
    K-mean recipe's K with per-channel offsets, smoothed by the oracle's own mean): descales,
    a digest and a sample of the E4M3 codes, and sampled O / LSE values of the attention on them.
    The format (E4M3) and the recipe (smoothing before K is quantised) follow "[HIP] Mha v4: run
    the K-smoothing gate as one HIP call" (Summary, Performance); the scale layout is this
    build's reading. The pages print no values."""
    import hashlib
    from oracle import fp8
    from workloads import make_inputs

    b, h, s, d = 1, 2, 128, 128
    q, k, v = make_inputs(b, h, h, s, s, d, d, seed=FP8_SEED, kmean=True)
    m32 = oracle.k_mean(bf16_bits(k), b, h, s, d)[1]
    q8, dq = fp8.quantize(bf16_bits(q), b, s, h, d)
    k8, dk = fp8.quantize(bf16_bits(k), b, s, h, d, mean32=m32)
    v8, dv = fp8.quantize(bf16_bits(v), b, s, h, d)
    scale = 1.0 / d ** 0.5
    o, lse = fp8.attn_rows(q8, k8, v8, dq, dk, dv, b, h, h, s, s, d, d, True, scale, FP8_ROWS,
                           nthreads=1)
    out = {
        "shape": [b, h, s, d], "seed": FP8_SEED, "causal": True, "scale": scale,
        "source": "CPU oracle (oracle/fp8.py on oracle/attn_oracle.c), written by "
                  "tests/golden/make_golden.py",
        "descale": {"q": dq.ravel().tolist(), "k": dk.ravel().tolist(), "v": dv.ravel().tolist()},
        "codes_sha256": {n: hashlib.sha256(a.tobytes()).hexdigest()
                         for n, a in (("q", q8), ("k", k8), ("v", v8))},
        "k_codes_row0_head0": k8[0, 0, 0, :16].tolist(),
        "rows": [list(r) for r in FP8_ROWS], "channels": FP8_CHANNELS,
        "o": [[float(o[n, ch]) for ch in FP8_CHANNELS] for n in range(len(FP8_ROWS))],
        "lse": [float(x) for x in lse],
    }
    with open(os.path.join(HERE, "fp8_b1_h2_s128_d128.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
    main_fp8()
