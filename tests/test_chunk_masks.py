"""The softmax's per-chunk masking in the attention kernel (csrc/attn_fwd_kernel.cuh), transcribed
and checked against brute force on random shapes (CPU only).

Inside a block that needs the per-key mask, each warp (32 consecutive rows of a query tile)
computes per row `rel` (the last allowed key, relative to the block, clamped to [-1, BN]) and
`lor` (the first allowed key, clamped to [0, BN]; 0 without a window). It reduces them over the
warp and takes one of three paths per 32-key chunk:
  - skip (P = 0 without exp2) when no row of the warp allows any key of the chunk;
  - no masking when every row allows every key of the chunk;
  - otherwise keep key c of the block iff lor <= c <= rel.
Checked for every real row (i < sq): skipped chunks hold no allowed key, unmasked chunks hold
only allowed keys, and the per-key rule equals the definition (j < sk, j <= i + sk - sq when
causal, j >= i + sk - sq - window with a window).
"""
import random

import numpy as np
import pytest

from test_unit_ranges import unit_ranges


def row_bounds(i, sq, sk, causal, window):
    """lim (last allowed key) and lol (first allowed key) of row i, as the kernel sets them."""
    lim_row = i + sk - sq if causal else sk - 1
    lim = min(lim_row, sk - 1)
    lol = i + sk - sq - window if window >= 0 else -(1 << 40)
    return lim, lol


def chunk_paths(j, BN, rows, sq, sk, causal, window):
    """Per chunk of block j: 'skip', 'none' or 'mask', and per row the kernel's kept keys."""
    rel, lor = [], []
    for i in rows:
        lim, lol = row_bounds(i, sq, sk, causal, window)
        rel.append(min(max(lim - j * BN, -1), BN))
        lor.append(min(max(lol - j * BN, 0), BN) if window >= 0 else 0)
    rel_lo, rel_hi, lor_lo, lor_hi = min(rel), max(rel), min(lor), max(lor)
    paths = []
    for ch in range(BN // 32):
        if ch * 32 > rel_hi or ch * 32 + 31 < lor_lo:
            paths.append("skip")
        elif ch * 32 + 31 <= rel_lo and ch * 32 >= lor_hi:
            paths.append("none")
        else:
            paths.append("mask")
    keep = np.array([[lor[r] <= c <= rel[r] for c in range(BN)] for r in range(len(rows))])
    return paths, keep


def check(sq, sk, NT, BN, causal, window):
    for q0 in range(0, sq, NT * 128):
        jb, nb, mlo, mfrom = unit_ranges(q0, sq, sk, NT, BN, causal, window)
        for j in range(jb, nb):
            if not ((window >= 0 and j < mlo) or j >= mfrom):
                continue  # an unmasked block (checked by test_unit_ranges)
            for tile in range(NT):
                for w in range(4):
                    rows = list(range(q0 + tile * 128 + w * 32, q0 + tile * 128 + w * 32 + 32))
                    paths, keep = chunk_paths(j, BN, rows, sq, sk, causal, window)
                    keys = j * BN + np.arange(BN)
                    for r, i in enumerate(rows):
                        if i >= sq:
                            continue  # rows past the end are computed but never stored
                        ok = keys < sk
                        if causal:
                            ok &= keys <= i + sk - sq
                        if window >= 0:
                            ok &= keys >= i + sk - sq - window
                        ctx = (sq, sk, NT, BN, causal, window, q0, j, tile, w, i)
                        assert np.array_equal(keep[r], ok), f"per-key rule differs {ctx}"
                        for ch, path in enumerate(paths):
                            seg = ok[ch * 32:(ch + 1) * 32]
                            if path == "skip":
                                assert not seg.any(), f"skipped chunk {ch} has a key {ctx}"
                            elif path == "none":
                                assert seg.all(), f"unmasked chunk {ch} has a masked key {ctx}"


@pytest.mark.parametrize("seed", range(4))
def test_chunk_masks_random(seed):
    rnd = random.Random(100 + seed)
    for _ in range(60):
        sq = rnd.choice([1, 31, 32, 33, 127, 128, 129]) if rnd.random() < 0.3 else rnd.randint(1, 600)
        sk = rnd.choice([1, 31, 32, 33, 64, 65, 128, 129]) if rnd.random() < 0.3 else rnd.randint(1, 600)
        window = rnd.choice([-1, -1, 0, 1, 31, 32, 33, 64, 127, 128, 300])
        check(sq, sk, rnd.choice([1, 2]), rnd.choice([64, 128]), rnd.random() < 0.75, window)
