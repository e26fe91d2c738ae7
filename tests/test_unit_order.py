"""The persistent kernel's unit schedule (unit_of in csrc/attn_fwd_kernel.cuh and the grid size
of csrc/attn_api.cu), transcribed and checked on the CPU: in every order (0 round robin,
1 snake, 2 weight-major snake) each unit is taken by exactly one (CTA, round); a CTA's positions
grow with the round, so once a round is past the last unit every later one is too (the kernel's
loops stop at the first such round); and order 2 takes, per round, the most expensive units that
are left (the k-th heaviest unit of every (batch, head) before any (k+1)-th)."""
import random

import pytest


def unit_of(r, c, grid, n_units, order, bh_count, n_qu):
    pos = r * grid + (grid - 1 - c if (order != 0 and (r & 1)) else c)
    if pos >= n_units:
        return -1
    if order == 2:
        k = pos // bh_count  # rank within its head (0 = the unit that sees the most keys)
        bh = pos - k * bh_count
        return bh * n_qu + k
    return pos


def schedule(bh_count, n_qu, n_sm, order):
    n_units = bh_count * n_qu
    grid = min(n_units, n_sm)
    taken = {}
    for c in range(grid):
        r, last_pos = 0, -1
        while True:
            u = unit_of(r, c, grid, n_units, order, bh_count, n_qu)
            if u < 0:
                # every later round of this CTA is past the end as well
                for r2 in range(r + 1, r + 4):
                    assert unit_of(r2, c, grid, n_units, order, bh_count, n_qu) < 0
                break
            pos = r * grid + (grid - 1 - c if (order != 0 and (r & 1)) else c)
            assert pos > last_pos
            last_pos = pos
            assert u not in taken, f"unit {u} taken twice"
            taken[u] = (c, r)
            r += 1
    assert sorted(taken) == list(range(n_units)), "some unit never taken"
    return taken, grid


@pytest.mark.parametrize("order", [0, 1, 2])
def test_every_unit_once(order):
    rnd = random.Random(order)
    cases = [(384, 8, 148), (128, 32, 148), (5, 256, 148), (16, 16, 148), (1, 1, 148), (3, 1, 148),
             (1, 300, 148), (148, 1, 148), (149, 2, 148)]
    cases += [(rnd.randint(1, 400), rnd.randint(1, 64), rnd.choice([1, 7, 132, 148])) for _ in range(60)]
    for bh_count, n_qu, n_sm in cases:
        schedule(bh_count, n_qu, n_sm, order)


def test_weight_major_takes_heaviest_first():
    # within a head, unit index k covers the query rows that see the most keys first (causal);
    # order 2 hands out all heads' rank-k units before any rank-(k+1) unit
    bh_count, n_qu, n_sm = 5, 256, 148
    taken, grid = schedule(bh_count, n_qu, n_sm, 2)
    ranks_by_round = {}
    for u, (c, r) in taken.items():
        ranks_by_round.setdefault(r, []).append(u % n_qu)
    for r in sorted(ranks_by_round)[:-1]:
        assert max(ranks_by_round[r]) <= min(ranks_by_round[r + 1])


def per_cta_balance(b, hq, sq, NT, order, n_sm=148):
    """max / mean of the per-CTA key-block totals of a causal square problem (cost of a unit =
    its visited key blocks x its tiles)."""
    from test_unit_ranges import unit_ranges
    n_qu = (sq + NT * 128 - 1) // (NT * 128)
    bh_count = b * hq
    taken, grid = schedule(bh_count, n_qu, n_sm, order)
    cost = {}
    for u in taken:
        qu = n_qu - 1 - (u % n_qu)  # within a head: most keys first
        jb, nb, _, _ = unit_ranges(qu * NT * 128, sq, sq, NT, 128, True, -1)
        cost[u] = (nb - jb) * NT
    load = [0] * grid
    for u, (c, _) in taken.items():
        load[c] += cost[u]
    return max(load) / (sum(load) / grid)


def test_causal_balance_by_order():
    # the causal workloads' geometry: 8 x 48 heads 2048^2, 128 heads 8192^2, 5 heads 65536^2
    for b, hq, sq in [(8, 48, 2048), (1, 128, 8192), (1, 5, 65536)]:
        rr = per_cta_balance(b, hq, sq, 2, 0)
        wm = per_cta_balance(b, hq, sq, 2, 2)
        assert wm <= 1.02 < 1.1 < rr, (b, hq, sq, rr, wm)


def test_packed_sequence_ranks():
    """Packed sequences: rank k of a (sequence, head) is its query unit nqu_seq - 1 - k (the k-th
    most expensive under a causal mask); ranks past the sequence's units are empty. Every unit
    of every sequence gets exactly one rank."""
    rnd = random.Random(3)
    for _ in range(200):
        NT = rnd.choice([1, 2])
        lens = [rnd.randint(0, 3000) for _ in range(rnd.randint(1, 9))]
        nqu = max(1, (max(lens) + NT * 128 - 1) // (NT * 128))
        for sq in lens:
            nqu_seq = (sq + NT * 128 - 1) // (NT * 128)
            q0s = [(nqu_seq - 1 - k) * NT * 128 if k < nqu_seq else sq for k in range(nqu)]
            busy = [q for q in q0s if q < sq]
            assert sorted(busy) == list(range(0, sq, NT * 128))
            assert busy == sorted(busy, reverse=True)  # most keys first
