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


# ---- order 3 (packed sequences): cost-sorted (sequence, rank) classes ----
from test_unit_ranges import unit_ranges  # noqa: E402

MAX_CLASSES = 256


def class_costs(lengths_q, lengths_k, n_qu, NT, BN, causal):
    """The kernel's class cost: key blocks the class's units visit (unit_info with its rank counted
    from the sequence's own last query tile), plus 2 when it visits any."""
    costs = []
    for sq, sk in zip(lengths_q, lengths_k):
        nqu_seq = (sq + NT * 128 - 1) // (NT * 128)
        for k in range(n_qu):
            q0 = (nqu_seq - 1 - k) * NT * 128 if k < nqu_seq else sq
            jb, nb, _, _ = unit_ranges(q0, sq, sk, NT, BN, causal, -1)
            w = nb - jb
            costs.append(min(w + 2, 65535) if w > 0 else 0)
    return costs


def order3_units(costs, b, hq, n_qu, grid):
    """(CTA, round) -> unit of order 3: classes ranked by (cost desc, class asc), all hq heads of
    a class in turn, positions handed out in snake order."""
    ncls = b * n_qu
    assert ncls <= MAX_CLASSES
    vcls = [None] * ncls
    for c in range(ncls):
        rank = sum(1 for c2 in range(ncls)
                   if costs[c2] > costs[c] or (costs[c2] == costs[c] and c2 < c))
        vcls[rank] = c
    taken = {}
    n_units = b * hq * n_qu
    for cta in range(grid):
        r = 0
        while True:
            pos = r * grid + (grid - 1 - cta if r & 1 else cta)
            if pos >= n_units:
                break
            cr, h = divmod(pos, hq)
            bi, k = divmod(vcls[cr], n_qu)
            u = (bi * hq + h) * n_qu + k
            assert u not in taken
            taken[u] = (cta, r, costs[vcls[cr]])
            r += 1
    return vcls, taken


@pytest.mark.parametrize("seed", range(3))
def test_order3_sorted_classes_cover_every_unit_once(seed):
    rnd = random.Random(100 + seed)
    for _ in range(20):
        b = rnd.randint(1, 16)
        hq = rnd.choice([1, 3, 8, 48])
        NT, BN = rnd.choice([(2, 64), (2, 128), (1, 64)])
        causal = rnd.random() < 0.7
        lq = [rnd.randint(0, 2100) for _ in range(b)]
        lk = [x if rnd.random() < 0.7 else rnd.randint(0, 2100) for x in lq]
        max_sq = max(max(lq), 1)
        n_qu = (max_sq + NT * 128 - 1) // (NT * 128)
        if b * n_qu > MAX_CLASSES:
            continue
        costs = class_costs(lq, lk, n_qu, NT, BN, causal)
        vcls, taken = order3_units(costs, b, hq, n_qu, rnd.choice([1, 7, 148]))
        assert sorted(vcls) == list(range(b * n_qu))          # a permutation of the classes
        ranked = [costs[c] for c in vcls]
        assert ranked == sorted(ranked, reverse=True)         # most expensive classes first
        assert sorted(taken) == list(range(b * hq * n_qu))    # every unit exactly once


def test_order3_balances_the_packed_workload():
    """The packed-sequence workload's lengths (8 sequences of 1024-2048, hq48, d64 pipelined
    layout: two 128-row tiles, 64-key blocks): per-CTA work peaks within 2 % of the mean with
    order 3, against 10 % with weight-major order."""
    import workloads
    c = workloads.config(6)
    L = workloads.varlen_lengths(c)
    b, hq, NT, BN, grid = len(L), c["hq"], 2, 64, 148
    n_qu = (max(L) + 255) // 256
    costs = class_costs(L, L, n_qu, NT, BN, True)
    _, taken = order3_units(costs, b, hq, n_qu, grid)
    loads = [0] * grid
    for cta, _, w in taken.values():
        loads[cta] += w
    assert max(loads) / (sum(loads) / grid) < 1.02
    loads2 = [0] * grid
    bh = b * hq
    for pos in range(bh * n_qu):
        r, cp = divmod(pos, grid)
        cta = cp if r % 2 == 0 else grid - 1 - cp
        k, bhi = divmod(pos, bh)
        loads2[cta] += costs[(bhi // hq) * n_qu + k]
    assert max(loads2) / (sum(loads2) / grid) > 1.05
