"""The FP8 quantiser's work split (csrc/fp8_quant.cu), transcribed and checked on the CPU: the
host's chunk count and rows per chunk, and each CTA thread's walk over its chunk, convert every
(row, 16-byte group) of every (batch, head) slice exactly once; the grid stays within launch
limits; and chunk 0, which writes the descale, always exists."""
import random

import pytest

THREADS = 256
TARGET_CTAS = 4 * 148


def host_split(b, s, h, d):
    """fp8_quantize's chunking: (chunks per slice, rows per chunk)."""
    nbh = b * h
    R = THREADS // (d // 8)
    nch = (TARGET_CTAS + nbh - 1) // nbh
    max_ch = (s + R - 1) // R
    nch = min(nch, max_ch, 1024)
    nch = max(nch, 1)
    rpc = (s + nch - 1) // nch
    rpc = (rpc + R - 1) // R * R
    rpc = max(rpc, R)
    nch = (s + rpc - 1) // rpc if s > 0 else 1
    return nch, rpc


def covered(s, d, nch, rpc):
    """(row, group) pairs one slice's CTAs visit, with multiplicity."""
    G = d // 8
    R = THREADS // G
    seen = {}
    for chunk in range(nch):
        s0 = chunk * rpc
        s1 = min(s0 + rpc, s)
        for t in range(THREADS):
            gi = t % G
            r = s0 + t // G
            while r < s1:
                seen[(r, gi)] = seen.get((r, gi), 0) + 1
                r += R
    return seen


@pytest.mark.parametrize("d", [64, 128, 256])
def test_every_group_once(d):
    rnd = random.Random(d)
    cases = [(1, 0, 2), (1, 1, 1), (3, 1, 4), (1, 4096, 16), (1, 65536, 5), (2, 300, 3),
             (8, 2048, 8), (1, 77, 2), (1, 1000, 5)]
    cases += [(rnd.randint(1, 4), rnd.randint(0, 3000), rnd.randint(1, 20)) for _ in range(40)]
    for b, s, h in cases:
        nch, rpc = host_split(b, s, h, d)
        assert 1 <= nch <= 1024 and b * h < 2 ** 31
        assert rpc % (THREADS // (d // 8)) == 0
        seen = covered(s, d, nch, rpc)
        assert len(seen) == s * (d // 8), (b, s, h, d, nch, rpc)
        assert all(v == 1 for v in seen.values()), (b, s, h, d)
        assert all(0 <= r < s for r, _ in seen)
