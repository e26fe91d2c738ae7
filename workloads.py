"""Seeded synthetic inputs for the attention forward pass and the K channel-mean pre-pass.

This module only draws random numbers and names shapes. It holds none of the arithmetic of
the method: both the CPU oracle (through the tests) and the CUDA path (through the tests and
the benchmark) receive the same bf16 bits from here, and neither side imports the other.

Workloads follow the shapes the pages benchmark ("Tune MHA config & small-head pipeline
pathology", Test Plan and Profiles 1/2: b8 hq48:hk8 2048^2 d64 causal and b1 hq128 8192^2
dqk192/dv128 causal; "[HIP] Mha v4: run the K-smoothing gate as one HIP call", Performance
table: hd256 b1 h16 s4096 and hd128 b1 h5 s65536). Values are iid N(0,1) cast to bf16 by
round-to-nearest-even; the K-mean workload adds a per-(head, channel) offset drawn N(0, 2^2)
so that the channel mean of K is far from zero.
"""
from __future__ import annotations

import math

import torch

# The workloads (sizes as the pages' benchmarks and the quantised-attention table give them).
WORKLOADS = {
    1: dict(workload="mha_b1_h2_s128_d64", b=1, hq=2, hk=2, sq=128, sk=128, dqk=64, dv=64,
            causal=False, kmean=False),
    2: dict(workload="gqa_b8_hq48_hk8_s2048_d64_causal", b=8, hq=48, hk=8, sq=2048, sk=2048,
            dqk=64, dv=64, causal=True, kmean=False),
    3: dict(workload="mla_prefill_b1_h128_s8192_dqk192_dv128_causal", b=1, hq=128, hk=128,
            sq=8192, sk=8192, dqk=192, dv=128, causal=True, kmean=False),
    4: dict(workload="mha_kmean_b1_h16_s4096_d256", b=1, hq=16, hk=16, sq=4096, sk=4096,
            dqk=256, dv=256, causal=False, kmean=True),
    5: dict(workload="long_b1_h5_s65536_d128_causal", b=1, hq=5, hk=5, sq=65536, sk=65536,
            dqk=128, dv=128, causal=True, kmean=False),
    # Packed sequences (the "varlen" layout of the pages' shape tables, e.g. 2048^2 d64 48/8
    # varlen): b sequences whose lengths are drawn uniformly from [min_s, sq] (seed 3000 + id),
    # each sequence's query and key lengths equal; sq / sk hold the longest possible length.
    6: dict(workload="varlen_b8_hq48_hk8_s1024to2048_d64_causal", b=8, hq=48, hk=8, sq=2048,
            sk=2048, min_s=1024, dqk=64, dv=64, causal=True, kmean=False, varlen=True),
    # Sliding window + attention sinks (the "GPT-OSS sink+sliding-window" shapes of the pages'
    # shape sources): 64:8 heads of d64, a 128-key window, one sink logit per head drawn
    # 1.5 * N(0,1) with seed 4000 + id.
    7: dict(workload="swa_sink_b1_hq64_hk8_s8192_d64_causal_w128", b=1, hq=64, hk=8, sq=8192,
            sk=8192, dqk=64, dv=64, causal=True, kmean=False, window=128, sinks=True),
    # The FP8 recipe on the pages' long FP8 shape (hd128, b1 h5 s65536; causal as the bf16 one):
    # the same N(0,1) draws, quantised to E4M3 with one scale per (batch, head) after the
    # K-smoothing gate.
    8: dict(workload="fp8_long_b1_h5_s65536_d128_causal", b=1, hq=5, hk=5, sq=65536, sk=65536,
            dqk=128, dv=128, causal=True, kmean=False, fp8=True),
}

HEAD_DIMS = ((64, 64), (128, 128), (192, 128), (256, 256))


def config(n: int) -> dict:
    """Copy of workload ``n`` with its seed and softmax scale filled in."""
    c = dict(WORKLOADS[n])
    c["id"] = n
    c["seed"] = 1000 + n
    c["scale"] = 1.0 / math.sqrt(c["dqk"])
    return c


def with_heads(c: dict, hq: int) -> dict:
    """Workload ``c`` with ``hq`` query heads and the kv heads scaled by the same factor (the
    group size stays), named after the new head count; ``hq`` = 0 leaves it unchanged."""
    if not hq or hq == c["hq"]:
        return c
    group = c["hq"] // c["hk"]
    if hq % group != 0:
        raise ValueError(f"{hq} query heads do not form groups of {group}")
    c = dict(c)
    c["hq"], c["hk"] = hq, hq // group
    c["workload"] = f"{c['workload']}_heads{hq}"
    return c


def flops(c: dict) -> float:
    """Algorithmic FLOPs of one forward pass: 2*b*hq*sq*sk*(dqk+dv), halved when causal (for
    packed sequences, the sum of that over the sequences; with a sliding window, 2*b*hq*(dqk+dv)
    times the exact number of allowed (query, key) pairs)."""
    if c.get("window") is not None:
        return 2.0 * c["b"] * c["hq"] * (c["dqk"] + c["dv"]) * allowed_pairs(c)
    if c.get("varlen"):
        lengths = varlen_lengths(c)
        f = sum(2.0 * c["hq"] * n * n * (c["dqk"] + c["dv"]) for n in lengths)
    else:
        f = 2.0 * c["b"] * c["hq"] * c["sq"] * c["sk"] * (c["dqk"] + c["dv"])
    return f / 2.0 if c["causal"] else f


def allowed_pairs(c: dict) -> int:
    """Allowed (query, key) pairs of one (batch, head): key j <= i + sk - sq when causal and
    j >= i + sk - sq - window."""
    total = 0
    for i in range(c["sq"]):
        d = i + c["sk"] - c["sq"]
        hi = min(c["sk"] - 1, d) if c["causal"] else c["sk"] - 1
        lo = max(0, d - c["window"]) if c.get("window") is not None else 0
        total += max(0, hi - lo + 1)
    return total


def sinks(c: dict):
    """The per-head sink logits of a workload with sinks (fp32 [hq]), else None."""
    if not c.get("sinks"):
        return None
    g = torch.Generator(device="cpu").manual_seed(4000 + int(c.get("id", 0)))
    return (1.5 * torch.randn(c["hq"], generator=g)).float()


def varlen_lengths(c: dict) -> list:
    """The sequence lengths of a packed-sequence workload (query length = key length)."""
    g = torch.Generator(device="cpu").manual_seed(3000 + int(c.get("id", 0)))
    return [int(x) for x in torch.randint(c["min_s"], c["sq"] + 1, (c["b"],), generator=g)]


def make_varlen_inputs(lengths_q, lengths_k, hq, hk, dqk, dv, seed):
    """Packed Q [sum lengths_q, hq, dqk], K, V [sum lengths_k, hk, d] (bf16, CPU) drawn from
    ``seed`` in the order Q, K, V, and the int32 offsets cu_q, cu_k (b + 1 entries each)."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    f32 = torch.float32
    tq, tk = int(sum(lengths_q)), int(sum(lengths_k))
    q = torch.randn((tq, hq, dqk), generator=g, dtype=f32).to(torch.bfloat16)
    k = torch.randn((tk, hk, dqk), generator=g, dtype=f32).to(torch.bfloat16)
    v = torch.randn((tk, hk, dv), generator=g, dtype=f32).to(torch.bfloat16)
    cu_q = torch.tensor([0] + list(lengths_q), dtype=torch.int64).cumsum(0).to(torch.int32)
    cu_k = torch.tensor([0] + list(lengths_k), dtype=torch.int64).cumsum(0).to(torch.int32)
    return q, k, v, cu_q, cu_k


def config_varlen_inputs(c: dict):
    lengths = varlen_lengths(c)
    return make_varlen_inputs(lengths, lengths, c["hq"], c["hk"], c["dqk"], c["dv"], c["seed"])


def make_inputs(b, hq, hk, sq, sk, dqk, dv, seed, kmean=False):
    """Draw Q, K, V (bf16, BSHD, contiguous, on the CPU) from ``seed``.

    Draw order is Q, K, V; with ``kmean`` it is Q, K noise, the per-(head, channel) offset
    (2 * N(0,1), broadcast over batch and sequence), then V.
    """
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    f32 = torch.float32
    q = torch.randn((b, sq, hq, dqk), generator=g, dtype=f32).to(torch.bfloat16)
    if kmean:
        noise = torch.randn((b, sk, hk, dqk), generator=g, dtype=f32)
        offset = 2.0 * torch.randn((hk, dqk), generator=g, dtype=f32)
        k = (noise + offset).to(torch.bfloat16)
        del noise
    else:
        k = torch.randn((b, sk, hk, dqk), generator=g, dtype=f32).to(torch.bfloat16)
    v = torch.randn((b, sk, hk, dv), generator=g, dtype=f32).to(torch.bfloat16)
    return q, k, v


def config_inputs(c: dict):
    return make_inputs(c["b"], c["hq"], c["hk"], c["sq"], c["sk"], c["dqk"], c["dv"],
                       c["seed"], c["kmean"])


def sample_rows(c: dict, n_pos: int = 256) -> torch.Tensor:
    """Seeded sample of output rows as int64 (batch, head, query) triples.

    ``n_pos`` query positions are drawn from a permutation seeded with 2000 + the workload
    number; positions 0 and sq-1 are always included. Every (batch, head) pair is sampled at
    those positions.
    """
    sq = c["sq"]
    g = torch.Generator(device="cpu").manual_seed(2000 + int(c.get("id", 0)))
    perm = torch.randperm(sq, generator=g)
    pos = [0, sq - 1] + [int(p) for p in perm.tolist() if p not in (0, sq - 1)]
    pos = sorted(set(pos[:max(2, min(n_pos, sq))]))
    rows = [(bi, h, i) for bi in range(c["b"]) for h in range(c["hq"]) for i in pos]
    return torch.tensor(rows, dtype=torch.int64)


def tile_edge_rows(c: dict, tile: int = 128) -> torch.Tensor:
    """Every (batch, head) pair at the first and the last query row of every ``tile``-row query
    tile, as int64 (batch, head, query) triples: each work unit of the attention kernel (one or
    two 128-row tiles of one (batch, head)) then contributes its first and last row."""
    sq = c["sq"]
    pos = sorted({p for t in range(0, sq, tile) for p in (t, min(t + tile - 1, sq - 1))})
    rows = [(bi, h, i) for bi in range(c["b"]) for h in range(c["hq"]) for i in pos]
    return torch.tensor(rows, dtype=torch.int64)


def bf16_bits(t: torch.Tensor):
    """The raw bf16 bit patterns of ``t`` as a contiguous numpy uint16 array."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
