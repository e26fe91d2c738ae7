"""The attention kernel's per-unit key-block ranges (unit_info in csrc/attn_fwd_kernel.cuh),
transcribed line by line and checked against brute force on random shapes (CPU only).

For a unit of NT query tiles starting at row q0, the kernel visits key blocks
j_begin .. n_blocks-1, and applies the per-key mask only to blocks < mask_lo (window) or
>= mask_from (causal diagonal, ragged key tail). The brute force builds the allowed-key matrix of
the unit's rows (key j allowed for row i iff j < sk, j <= i + sk - sq when causal, and
j >= i + sk - sq - window with a window) and checks:
  - no allowed key lies in a block the unit skips;
  - the first and last visited blocks each hold an allowed key of some row (no wasted block at
    either end);
  - every block the kernel leaves unmasked is allowed for every key and every real row;
  - a unit with no visited block has no allowed key at all.
"""
import random

import numpy as np
import pytest


def unit_ranges(q0, sq, sk, NT, BN, causal, window):
    """unit_info's range arithmetic (dense problem; window < 0: none). The operands of every
    division are non-negative, so floor division equals the kernel's truncating division."""
    if q0 >= sq:
        return 0, 0, 0, 0
    n_kv = (sk + BN - 1) // BN
    if causal:
        last_row = min(q0 + NT * 128 - 1, sq - 1)
        last_key = last_row + sk - sq
        nb = 0 if last_key < 0 else last_key // BN + 1
        nb = min(nb, n_kv)
        first_lim = q0 + sk - sq + 1
        full = 0 if first_lim <= 0 else first_lim // BN
        full = min(full, sk // BN)
        n_blocks, mask_from = nb, min(full, nb)
    else:
        n_blocks, mask_from = n_kv, sk // BN
    j_begin, mask_lo = 0, 0
    if window >= 0:
        last_row = min(q0 + NT * 128 - 1, sq - 1)
        lo_first = q0 + sk - sq - window
        lo_last = last_row + sk - sq - window
        jb = 0 if lo_first <= 0 else lo_first // BN
        j_begin = min(jb, n_blocks)
        mask_lo = 0 if lo_last <= 0 else (lo_last + BN - 1) // BN
    return j_begin, n_blocks, mask_lo, mask_from


def allowed(q0, sq, sk, NT, causal, window):
    rows = np.arange(q0, min(q0 + NT * 128, sq))[:, None]
    keys = np.arange(sk)[None, :]
    ok = np.ones((rows.shape[0], sk), dtype=bool)
    if causal:
        ok &= keys <= rows + sk - sq
    if window >= 0:
        ok &= keys >= rows + sk - sq - window
    return ok


def check_shape(sq, sk, NT, BN, causal, window):
    for q0 in range(0, sq, NT * 128):
        jb, nb, mlo, mfrom = unit_ranges(q0, sq, sk, NT, BN, causal, window)
        ok = allowed(q0, sq, sk, NT, causal, window)
        any_key = ok.any(axis=0)  # key allowed for some row of the unit
        blocks = np.nonzero(any_key)[0] // BN
        ctx = (sq, sk, NT, BN, causal, window, q0, (jb, nb, mlo, mfrom))
        if blocks.size == 0:
            assert nb <= jb, f"unit with no allowed key visits blocks {ctx}"
            continue
        assert jb <= blocks.min() and blocks.max() < nb, f"allowed key outside the range {ctx}"
        assert blocks.min() == jb and blocks.max() == nb - 1, f"wasted block at an end {ctx}"
        for b in range(jb, nb):
            masked = (window >= 0 and b < mlo) or b >= mfrom
            if masked:
                continue
            lo, hi = b * BN, (b + 1) * BN
            assert hi <= sk and ok[:, lo:hi].all(), f"unmasked block {b} is not all allowed {ctx}"


@pytest.mark.parametrize("seed", range(6))
def test_unit_ranges_random(seed):
    rnd = random.Random(seed)
    for _ in range(250):
        sq = rnd.choice([1, 2, 127, 128, 129, 255, 256, 257]) if rnd.random() < 0.3 else rnd.randint(1, 1200)
        sk = rnd.choice([1, 63, 64, 65, 128, 129]) if rnd.random() < 0.3 else rnd.randint(1, 1200)
        window = rnd.choice([-1, -1, 0, 1, 5, 63, 64, 127, 128, 129, 300, 2000])
        check_shape(sq, sk, rnd.choice([1, 2]), rnd.choice([64, 128]), rnd.random() < 0.7, window)


def test_unit_ranges_workload_shapes():
    # the benchmark shapes' geometry (per head): 2048^2, 8192^2 (and its window), 4096^2, 65536^2
    for sq, NT, BN, causal, window in [(2048, 2, 64, True, -1), (8192, 2, 128, True, -1),
                                       (8192, 2, 64, True, 128), (4096, 1, 64, False, -1),
                                       (65536, 2, 128, True, -1)]:
        check_shape(sq, sq, NT, BN, causal, window)
