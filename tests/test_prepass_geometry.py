"""The work split of the K-mean and K-smoothing-gate pre-passes (csrc/kmean.cu), transcribed and
checked on the CPU: k_mean_partial sums every (key row, 8-channel group) exactly once, and
k_gate_partial reads exactly the strided sample 0, stride, 2*stride, ... < sk (every key up to
2048 keys, at most 2048 samples beyond), each sampled row in exactly one chunk."""
import random

import pytest

THREADS = 256
COLS_PER_CTA = THREADS * 8
TARGET_CTAS = 4 * 148
MIN_ROWS_PER_CHUNK = 16


def mean_split(b, hk, sk, d):
    cols = hk * d
    col_ctas = (cols + COLS_PER_CTA - 1) // COLS_PER_CTA
    nchunks = (TARGET_CTAS + col_ctas * b - 1) // (col_ctas * b)
    nchunks = min(nchunks, (sk + MIN_ROWS_PER_CHUNK - 1) // MIN_ROWS_PER_CHUNK, 1024)
    nchunks = max(nchunks, 1)
    rpc = (sk + nchunks - 1) // nchunks
    nchunks = (sk + rpc - 1) // rpc
    return cols, col_ctas, nchunks, rpc


def gate_split(b, hk, sk, d):
    cols = hk * d
    stride = (sk + 2047) // 2048
    n_samp = (sk + stride - 1) // stride
    col_ctas = (cols + COLS_PER_CTA - 1) // COLS_PER_CTA
    nchunks = (TARGET_CTAS + col_ctas * b - 1) // (col_ctas * b)
    nchunks = min(nchunks, (n_samp + 31) // 32, 1024)
    nchunks = max(nchunks, 1)
    per_chunk = (n_samp + nchunks - 1) // nchunks
    nchunks = (n_samp + per_chunk - 1) // per_chunk
    return cols, col_ctas, stride, n_samp, nchunks, per_chunk


CASES = [(1, 16, 4096, 256), (1, 5, 65536, 128), (8, 8, 2048, 64), (2, 3, 100, 64),
         (1, 1, 1, 128), (3, 5, 17, 256), (1, 4, 2049, 64), (1, 2, 5000, 128)]


@pytest.mark.parametrize("seed", range(3))
def test_mean_covers_every_row_once(seed):
    rnd = random.Random(seed)
    cases = CASES + [(rnd.randint(1, 8), rnd.randint(1, 40), rnd.randint(1, 9000),
                      rnd.choice([64, 128, 256])) for _ in range(25)]
    for b, hk, sk, d in cases:
        cols, col_ctas, nchunks, rpc = mean_split(b, hk, sk, d)
        assert 1 <= nchunks <= 1024
        c8 = cols // 8
        groups = {g8 for x in range(col_ctas) for g8 in range(x * THREADS, (x + 1) * THREADS)
                  if g8 < c8}
        assert groups == set(range(c8))  # every 8-channel group has one thread per chunk
        rows = [s for chunk in range(nchunks) for s in range(chunk * rpc, min(chunk * rpc + rpc, sk))]
        assert sorted(rows) == list(range(sk)), (b, hk, sk, d)


@pytest.mark.parametrize("seed", range(3))
def test_gate_reads_the_strided_sample_once(seed):
    rnd = random.Random(10 + seed)
    cases = CASES + [(rnd.randint(1, 8), rnd.randint(1, 40), rnd.randint(1, 70000),
                      rnd.choice([64, 128, 256])) for _ in range(25)]
    for b, hk, sk, d in cases:
        cols, col_ctas, stride, n_samp, nchunks, per_chunk = gate_split(b, hk, sk, d)
        assert 1 <= nchunks <= 1024
        if sk <= 2048:
            assert stride == 1 and n_samp == sk
        else:
            assert n_samp <= 2048
        ts = [t for chunk in range(nchunks)
              for t in range(chunk * per_chunk, min(chunk * per_chunk + per_chunk, n_samp))]
        assert sorted(ts) == list(range(n_samp))
        keys = [t * stride for t in ts]
        assert sorted(keys) == list(range(0, sk, stride)), (b, hk, sk, d)
