"""The work split of the one-pass K-mean and K-smoothing-gate kernels (csrc/kmean.cu: make_split,
sum_chunks, sum_chunks_bulk and the two folds), transcribed and checked on the CPU:
  - phase 1 sums every (key row, 8-channel group) of every batch exactly once (the gate: exactly
    the strided sample 0, stride, 2*stride, ... < sk, every key up to 2048 keys, at most 2048
    samples beyond), and every partial it writes lies inside the scratch sized for the split;
  - the mean's bulk-copy phase 1 (rows of at most 4096 channels): every copy is a whole number
    of 16-byte units inside K and inside one ring buffer, and each row lane reads its own rows in
    order;
  - the fold covers every (batch, column) of the mean once (the gate: every (batch, kv head)),
    and its chunk ranges (per warp, per channel group) cover every chunk exactly once;
  - the allocation-free entry point's split never needs more partials than its fixed array holds.
"""
import random

import pytest

THREADS = 512
COLS_PER_CTA = THREADS * 8
FOLD_WARPS = THREADS // 32
SMS = 148
NOALLOC_FLOATS = 1 << 20
STAGES, STAGE_BYTES = 4, 32768  # the bulk-copy ring
COLS_MIN_G = 2


def lanes_of(cols, lanes_ok):
    """Row lanes of the mean's bulk-copy phase 1 (0: the register path)."""
    colgroups = (cols + COLS_PER_CTA - 1) // COLS_PER_CTA
    return THREADS // (cols // 8) if lanes_ok and colgroups == 1 else 0


def make_split(b, cols, n_rows, max_chunks, grid_max, lanes_ok=False):
    colgroups = (cols + COLS_PER_CTA - 1) // COLS_PER_CTA
    per = 16 * max(lanes_of(cols, lanes_ok), 1)
    nch = (grid_max + b * colgroups - 1) // (b * colgroups)
    nch = min(nch, (n_rows + per - 1) // per, max_chunks, 1024)
    nch = max(nch, 1)
    rpc = (n_rows + nch - 1) // nch
    nchunks = (n_rows + rpc - 1) // rpc
    n_items = b * colgroups * nchunks
    return colgroups, rpc, nchunks, n_items, min(n_items, grid_max)


def phase1_bulk(b, cols, sk, split):
    """(bi, row, 8-channel group) -> times summed by the bulk-copy phase 1; checks every copy
    and every shared-memory read on the way."""
    colgroups, rpc, nchunks, n_items, grid = split
    assert colgroups == 1
    c8 = cols // 8
    R = THREADS // c8
    row_bytes = c8 * 16
    rps = STAGE_BYTES // row_bytes
    assert rps >= 1
    seen = {}
    for cta in range(grid):
        fills = 0
        for it in range(cta, n_items, grid):
            chunk, bi = it % nchunks, it // nchunks
            t0 = chunk * rpc
            t1 = min(t0 + rpc, sk)
            nst = (t1 - t0 + rps - 1) // rps
            src = (bi * sk + t0) * row_bytes
            last = [-1] * (R * c8)
            for st in range(nst):
                r0 = st * rps
                n = min(rps, t1 - t0 - r0)
                nbytes = n * row_bytes
                assert nbytes % 16 == 0 and 0 < nbytes <= STAGE_BYTES and src % 16 == 0
                assert src + r0 * row_bytes + nbytes <= b * sk * row_bytes
                slot = (fills + st) % STAGES
                assert (slot + 1) * STAGE_BYTES <= STAGES * STAGE_BYTES
                for tid in range(R * c8):
                    lane, g8 = divmod(tid, c8)
                    r = (lane - r0 % R + R) % R
                    while r < n:
                        assert (r * c8 + g8 + 1) * 16 <= STAGE_BYTES
                        row = t0 + r0 + r
                        assert (row - t0) % R == lane and row > last[tid]
                        last[tid] = row
                        seen[(bi, row, g8)] = seen.get((bi, row, g8), 0) + 1
                        r += R
            fills += nst
    return seen


def phase1(b, cols, n_rows, stride, split, planes):
    """(bi, row, 8-channel group) -> times summed, and the largest partial index written."""
    colgroups, rpc, nchunks, n_items, grid = split
    c8 = cols // 8
    seen = {}
    top = -1
    for cta in range(grid):
        for it in range(cta, n_items, grid):
            chunk = it % nchunks
            bcg = it // nchunks
            cg, bi = bcg % colgroups, bcg // colgroups
            for tid in range(THREADS):
                g8 = cg * THREADS + tid
                if g8 >= c8:
                    continue
                for t in range(chunk * rpc, min(chunk * rpc + rpc, n_rows)):
                    key = (bi, t * stride, g8)
                    seen[key] = seen.get(key, 0) + 1
                base = ((bi * nchunks + chunk) * planes) * cols + g8 * 8
                top = max(top, base + (planes - 1) * cols + 7)
    return seen, top


CASES = [(1, 16, 4096, 256), (1, 5, 65536, 128), (8, 8, 2048, 64), (2, 3, 100, 64),
         (1, 1, 1, 128), (3, 5, 17, 256), (1, 4, 2049, 64), (1, 2, 5000, 128), (2, 40, 300, 256)]


def random_cases(rnd, max_sk):
    return [(rnd.randint(1, 6), rnd.randint(1, 24), rnd.randint(1, max_sk),
             rnd.choice([64, 128, 256])) for _ in range(12)]


@pytest.mark.parametrize("seed", range(2))
def test_mean_sums_every_row_once_inside_its_scratch(seed):
    rnd = random.Random(seed)
    for b, hk, sk, d in CASES + random_cases(rnd, 3000):
        cols = hk * d
        split = make_split(b, cols, sk, 1024, SMS, lanes_ok=True)
        colgroups, rpc, nchunks, n_items, grid = split
        assert 1 <= nchunks <= 1024 and 1 <= grid <= SMS
        if sk * b * cols > 4_000_000:  # the full transcription is slow: check the row split only
            rows = [t for ch in range(nchunks) for t in range(ch * rpc, min(ch * rpc + rpc, sk))]
            assert sorted(rows) == list(range(sk))
            continue
        if lanes_of(cols, True):
            seen = phase1_bulk(b, cols, sk, split)
            top = (b * nchunks - 1) * cols + cols - 1  # thread t < c8 writes chunk row t*8..t*8+7
        else:
            seen, top = phase1(b, cols, sk, 1, split, 1)
        assert set(seen.values()) == {1}
        assert len(seen) == b * sk * (cols // 8), (b, hk, sk, d)
        assert top < b * nchunks * cols  # the partials the host allocates


@pytest.mark.parametrize("seed", range(2))
def test_gate_reads_the_strided_sample_once(seed):
    rnd = random.Random(10 + seed)
    for b, hk, sk, d in CASES + random_cases(rnd, 70000):
        cols = hk * d
        stride = (sk + 2047) // 2048
        n_samp = (sk + stride - 1) // stride
        if sk <= 2048:
            assert stride == 1 and n_samp == sk
        else:
            assert n_samp <= 2048
        split = make_split(b, cols, n_samp, 1024, SMS)
        colgroups, rpc, nchunks, n_items, grid = split
        ts = [t for ch in range(nchunks) for t in range(ch * rpc, min(ch * rpc + rpc, n_samp))]
        assert sorted(ts) == list(range(n_samp))
        assert sorted(t * stride for t in ts) == list(range(0, sk, stride)), (b, hk, sk, d)
        if n_samp * b * cols <= 4_000_000:
            seen, top = phase1(b, cols, n_samp, stride, split, 2)
            assert set(seen.values()) == {1} and len(seen) == b * n_samp * (cols // 8)
            assert top < b * nchunks * 2 * cols


def test_fold_covers_every_column_and_chunk_once():
    for b, hk, sk, d in CASES:
        cols = hk * d
        _, _, nchunks, _, grid = make_split(b, cols, sk, 1024, SMS, lanes_ok=True)
        nblk = (cols + 31) // 32
        outs = [(f // nblk, (f % nblk) * 32 + lane) for cta in range(grid)
                for f in range(cta, b * nblk, grid) for lane in range(32)
                if (f % nblk) * 32 + lane < cols]
        assert sorted(outs) == [(bi, c) for bi in range(b) for c in range(cols)]
        ranges = [c for w in range(FOLD_WARPS)
                  for c in range(w * nchunks // FOLD_WARPS, (w + 1) * nchunks // FOLD_WARPS)]
        assert ranges == list(range(nchunks))
        # gate fold: (batch, kv head) items; the head's 2d partial columns as d/2 float4 columns
        # (d/4 of channel sums, then d/4 of sums of squares), 1024/d chunk groups
        c4s = d // 2
        groups = THREADS // c4s
        assert groups * c4s == THREADS
        heads = [f for cta in range(grid) for f in range(cta, b * hk, grid)]
        assert sorted(heads) == list(range(b * hk))
        for grp in range(groups):
            got = []
            for t in range(grp * c4s, (grp + 1) * c4s):
                c4 = t % c4s
                plane = 0 if c4 < d // 4 else 1
                ch = 4 * (c4 - plane * (d // 4))
                got += [(plane, ch + k) for k in range(4)]
                # the float index of the column in the group's shared row: d sums, then d squares
                assert [4 * c4 + k for k in range(4)] == [plane * d + ch + k for k in range(4)]
            assert sorted(got) == [(pl, c) for pl in range(2) for c in range(d)]
        ranges = [c for g in range(groups)
                  for c in range(g * nchunks // groups, (g + 1) * nchunks // groups)]
        assert ranges == list(range(nchunks))


def test_noalloc_split_fits_the_fixed_scratch():
    for b, hk, sk, d in CASES + [(4, 1024, 40, 256), (1, 4096, 300, 256), (64, 64, 5000, 256)]:
        cols = hk * d
        if b * cols > NOALLOC_FLOATS:
            continue  # refused with ERR_SCRATCH
        _, _, nchunks, _, grid = make_split(b, cols, sk, NOALLOC_FLOATS // (b * cols), SMS,
                                            lanes_ok=True)
        assert b * nchunks * cols <= NOALLOC_FLOATS and grid <= 1024


def cols_group(pairs, n_sm):
    """The column-partitioned split's pairs per CTA (0: the row-chunk kernel is used)."""
    G = 1
    while G < THREADS and (pairs + G - 1) // G > n_sm:
        G <<= 1
    grid = (pairs + G - 1) // G
    return G if grid <= n_sm and 2 * grid >= n_sm and G >= COLS_MIN_G else 0


@pytest.mark.parametrize("seed", range(2))
def test_column_path_sums_every_row_once(seed):
    """k_mean_cols: CTA c owns (batch, 8-channel group) pairs [c*G, c*G + G); thread t takes pair
    slot t % G at rows t // G, + L, ... (L = 512 / G); the tree over lanes folds every lane into
    lane 0 exactly once. The K-mean workload (16 x 256 channels) takes it with G = 4 on 128 CTAs;
    narrow K falls back to the row-chunk kernel, and so does K whose pairs would need G = 1
    (16 bytes of a row per CTA: the 5 x 128-channel K of the long-context workload)."""
    assert cols_group(1 * 16 * 256 // 8, SMS) == 4
    assert (512 + 3) // 4 == 128
    assert cols_group(2 * 3 * 64 // 8, SMS) == 0  # 48 pairs: too few CTAs
    assert cols_group(1 * 5 * 128 // 8, SMS) == 0  # 80 pairs: G = 1
    rnd = random.Random(20 + seed)
    cases = [(1, 16, 4096, 256), (2, 40, 300, 256), (1, 64, 77, 128), (4, 20, 33, 64), (1, 148, 9, 64)]
    cases += [(rnd.randint(1, 4), rnd.randint(1, 200), rnd.randint(1, 300),
               rnd.choice([64, 128, 256])) for _ in range(30)]
    for b, hk, sk, d in cases:
        pairs = b * hk * d // 8
        G = cols_group(pairs, SMS)
        if G == 0:
            continue
        assert G & (G - 1) == 0 and 1 <= G <= THREADS
        grid = (pairs + G - 1) // G
        assert SMS / 2 <= grid <= SMS
        L = THREADS // G
        if pairs * sk <= 2_000_000:
            seen = {}
            for cta in range(grid):
                for t in range(THREADS):
                    pair = cta * G + t % G
                    if pair >= pairs:
                        continue
                    for r in range(t // G, sk, L):
                        seen[(pair, r)] = seen.get((pair, r), 0) + 1
            assert len(seen) == pairs * sk and set(seen.values()) == {1}
        held = [{ln} for ln in range(L)]  # the tree: lane ln absorbs lane ln + w
        w = L // 2
        while w > 0:
            for ln in range(w):
                assert not (held[ln] & held[ln + w])
                held[ln] |= held[ln + w]
            w //= 2
        assert held[0] == set(range(L))
