"""The FP8 quantiser's work split (csrc/fp8_quant.cu: fp8_quantize and fp8_quant_onepass),
transcribed and checked on the CPU:
  - the host's chunk count and rows per chunk, and each thread's walk over its chunk (in the
    amax pass and in the convert pass), cover every (row, 16-byte group) of every (batch, head)
    slice exactly once;
  - with several chunks per slice every CTA holds at most one item (the grid-wide wait needs
    every CTA resident and each pass 2 to find its own item), and the chunk count fits the fold
    (one partial per thread);
  - with one chunk per slice the CTAs' strided loop takes every slice once;
  - chunk 0, which writes the descale, always exists."""
import random

import pytest

THREADS = 512
MAX_CHUNKS = 64
SMS = 148


def host_split(b, s, h, d, grid_max=SMS):
    """fp8_quantize's split: (chunks per slice, rows per chunk, items, grid)."""
    nbh = b * h
    R = THREADS // (d // 8)
    nch = grid_max // nbh if nbh < grid_max else 1
    max_ch = (s + R - 1) // R
    nch = min(nch, max_ch, MAX_CHUNKS)
    nch = max(nch, 1)
    rpc = (s + nch - 1) // nch if s > 0 else 0
    if s > 0:
        nch = (s + rpc - 1) // rpc
    n_items = nbh * nch
    return nch, rpc, n_items, min(n_items, grid_max)


def walks(s, d, nch, rpc):
    """(row, group) pairs one slice's chunks visit in the amax pass and in the convert pass."""
    G = d // 8
    R = THREADS // G
    amax, conv = {}, {}
    for chunk in range(nch):
        s0 = chunk * rpc
        s1 = min(s0 + rpc, s) if nch > 1 else s
        for t in range(THREADS):
            gi = t % G
            r = s0 + t // G
            while r + 11 * R < s1:  # twelve loads in flight, then the tail
                for e in range(12):
                    amax[(r + e * R, gi)] = amax.get((r + e * R, gi), 0) + 1
                r += 12 * R
            while r < s1:
                amax[(r, gi)] = amax.get((r, gi), 0) + 1
                r += R
            r = s0 + t // G
            while r < s1:  # eight groups in flight
                for e in range(8):
                    if r + e * R < s1:
                        conv[(r + e * R, gi)] = conv.get((r + e * R, gi), 0) + 1
                r += 8 * R
    return amax, conv


@pytest.mark.parametrize("d", [64, 128, 256])
def test_every_group_once(d):
    rnd = random.Random(d)
    cases = [(1, 0, 2), (1, 1, 1), (3, 1, 4), (1, 4096, 16), (1, 65536, 5), (2, 300, 3),
             (8, 2048, 8), (1, 77, 2), (1, 1000, 5), (8, 2048, 48), (1, 8192, 200)]
    cases += [(rnd.randint(1, 4), rnd.randint(0, 3000), rnd.randint(1, 80)) for _ in range(40)]
    for b, s, h in cases:
        nch, rpc, n_items, grid = host_split(b, s, h, d)
        assert 1 <= nch <= MAX_CHUNKS and b * h < 2 ** 31
        if nch > 1:
            assert n_items <= grid, (b, s, h, d)  # one item per CTA at most
        else:  # CTA c takes slices c, c + grid, ...: every slice once
            taken = sorted(bh for c in range(grid) for bh in range(c, n_items, grid))
            assert taken == list(range(b * h))
        amax, conv = walks(s, d, nch, rpc)
        for seen in (amax, conv):
            assert len(seen) == s * (d // 8), (b, s, h, d, nch, rpc)
            assert all(v == 1 for v in seen.values()), (b, s, h, d)
            assert all(0 <= r < s for r, _ in seen)


def test_fp8_workload_split():
    # b1 h5 65536 rows d128: 29 chunks per head, 145 CTAs of one item each
    nch, rpc, n_items, grid = host_split(1, 65536, 5, 128)
    assert (nch, n_items, grid) == (29, 145, 145)
