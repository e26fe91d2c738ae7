"""Executable model of the mbarrier protocol of the attention kernel (csrc/attn_fwd_kernel.cuh).

TEST INFRASTRUCTURE: a model of the kernel's design, not of the method; it shares no code with
the CUDA library and the library never uses it.

Roles (as in the kernel): one TMA producer, one MMA issuer and one softmax warpgroup per
query tile (one or two tiles per work unit).
The tensor core runs each issuer's MMAs and commits in its issue order, interleaving issuers at
random. TMA loads land at random later times.
A random scheduler interleaves everything. mbarriers count arrivals and transaction bytes and
complete phases; a wait on parity p passes once the phase with that parity has completed, as
on the hardware.

Checked on every schedule:
  - each Q K^T reads the K tile and the Q of its own (unit, block, tile), and never overwrites a
    score buffer whose P is still unconsumed;
  - each P V reads its own V tile and the P of its own item, and accumulates into an O that
    holds exactly the unit's previous blocks;
  - an O rescale (softmax) sees all earlier blocks of its tile accumulated;
  - the epilogue reads a complete O, and O is not overwritten before it has been read;
  - the staged Q copied into tensor memory is the unit the copy expects;
  - no deadlock: whenever no load or MMA is in flight, some role can still make progress.

`run(..., mutant=name)` plants one protocol mistake (see MUTANTS) so that the tests can check
that the model catches it.
"""
from __future__ import annotations

import random

MUTANTS = {
    "k_slot_reused_without_wait": "the producer refills a K slot without waiting for kempty",
    "kempty_after_first_tile": "a K slot is freed by the first MMA issuer's commit alone",
    "no_o_free_wait": "the MMA warp starts a unit's first P V without waiting for o_free",
    "no_pv_done_wait": "where S(j+1) can land before P V(j) (one tile, or the pipelined two-tile "
                       "layout), the softmax rescales O without waiting for its bar_pv_done",
    "q_refill_without_wait": "the producer refills the Q staging buffer without waiting q_empty",
    "s_full_wrong_parity": "the softmax waits for the wrong phase of its score buffer",
    "p_full_early": "the softmax hands over P before writing it",
    "kempty_wrong_parity": "the producer waits for the wrong phase of a free K slot",
}


class Violation(AssertionError):
    pass


class Deadlock(RuntimeError):
    pass


def check(cond, msg):
    if not cond:
        raise Violation(msg)


class Bar:
    """mbarrier: `count` arrivals plus the expected transaction bytes complete a phase. `clock`
    (shared by a run's barriers) counts every arrival and transaction, i.e. every change of
    barrier state."""

    def __init__(self, count, name, clock):
        self.count, self.pending, self.tx, self.completed, self.name = count, count, 0, 0, name
        self.clock = clock

    def arrive(self, n=1):
        self.clock[0] += 1
        self.pending -= n
        check(self.pending >= 0, f"too many arrivals on {self.name}")
        self._complete()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive(1)

    def complete_tx(self, nbytes):
        self.clock[0] += 1
        self.tx -= nbytes
        check(self.tx >= 0, f"transaction underflow on {self.name}")
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def passed(self, parity):
        """A wait on `parity` passes once the phase with that parity has completed."""
        return (self.completed & 1) != parity


def run(units, NT, NSM, q_tmem, NK, NV, seed, mutant=None, pipe=False, late_turn=False):
    """One random schedule over `units` (dicts with 'id' and 'n' = key blocks, 0 = skipped).
    late_turn: the two tiles' softmax take their turn after waiting for (and loading) their own
    S, as the E4M3 layout does, instead of before."""
    rnd = random.Random(seed)
    clock = [0]
    kfull = [Bar(1, f"kfull{i}", clock) for i in range(NK)]
    # one commit per MMA issuer (the planted mistake counts one)
    kempty = [Bar(1 if mutant == "kempty_after_first_tile" else NT, f"kempty{i}", clock)
              for i in range(NK)]
    vfull = [Bar(1, f"vfull{i}", clock) for i in range(NV)]
    vempty = [Bar(NT, f"vempty{i}", clock) for i in range(NV)]
    # pipe (two tiles): each tile owns two score buffers and pipelines its own MMAs (Q K^T of
    # block j+1 before P V of block j); otherwise two tiles own one buffer each and take turns,
    # and one tile alternates between the two buffers
    nsbuf = 2 * NT if pipe else 2
    s_full = [Bar(1, f"s_full{i}", clock) for i in range(nsbuf)]
    p_full = [Bar(128, f"p_full{i}", clock) for i in range(nsbuf)]
    pv_done = [Bar(1, f"pv_done{t}", clock) for t in range(NT)]

    def sbuf_of(jg, tt):
        return tt * 2 + (jg & 1) if pipe else (tt if NT == 2 else jg & 1)

    def sphase_of(jg):
        return (jg >> 1) & 1 if (pipe or NT == 1) else jg & 1
    q_full = Bar(1, "q_full", clock)
    q_empty = Bar(128 * NT if q_tmem else NT, "q_empty", clock)
    q_tmem_bar = [Bar(128, f"q_tmem{t}", clock) for t in range(NT)]
    o_full = [Bar(1, f"o_full{t}", clock) for t in range(NT)]
    o_free = [Bar(128, f"o_free{t}", clock) for t in range(NT)]

    mma_done = Bar(NT, "mma_done", clock)

    kslot = [None] * NK
    vslot = [None] * NV
    qstage = [None]
    qtm = {}            # tile -> unit whose Q is in tensor memory
    # score buffer -> per half ("lo": the columns P overwrites, "hi": the rest) the item and
    # its state: 'S' (scores landed), 'read' (in the softmax's registers), 'P' (P written),
    # 'consumed' (read by P V)
    sbuf = [{"lo": None, "hi": None} for _ in range(nsbuf)]
    obuf = {}           # tile -> [unit, blocks accumulated, 'acc' | 'read']
    landings = []       # TMA loads in flight
    tensor = []         # issued MMAs and commits: (issuer, kind, x); in order per issuer
    busy = [u for u in units if u["n"] > 0]
    current = [None]  # the role being stepped
    waits = {}        # role -> (barrier, parity, completed phases) it last blocked on

    def wait(bar, parity):
        while not bar.passed(parity):
            waits[current[0]] = (bar.name, parity, bar.completed)
            yield False

    # ------------------------------ TMA producer ------------------------------
    def producer():
        cnt = {"k": 0, "v": 0, "q": 0}

        def load_q(u):
            if mutant != "q_refill_without_wait":
                yield from wait(q_empty, (cnt["q"] & 1) ^ 1)
            q_full.expect_tx(1)

            def land(uid=u["id"]):
                qstage[0] = uid
                q_full.complete_tx(1)
            landings.append(land)
            cnt["q"] += 1
            yield True

        def load_kv(kind, u, j):
            slots, full, empty, nslot = ((kslot, kfull, kempty, NK) if kind == "k"
                                         else (vslot, vfull, vempty, NV))
            c = cnt[kind]
            s = c % nslot
            if not (kind == "k" and mutant == "k_slot_reused_without_wait"):
                flip = 0 if (kind == "k" and mutant == "kempty_wrong_parity") else 1
                yield from wait(empty[s], ((c // nslot) & 1) ^ flip)
            full[s].expect_tx(1)

            def land(s=s, item=(u["id"], j)):
                slots[s] = item
                full[s].complete_tx(1)
            landings.append(land)
            cnt[kind] += 1
            yield True

        pend = None
        if busy:
            yield from load_q(busy[0])
        for ui, u in enumerate(busy):
            nxt = busy[ui + 1] if ui + 1 < len(busy) else None
            for j in range(u["n"]):
                for tt in range(1 if pipe else NT):
                    if tt == 0:
                        yield from load_kv("k", u, j)
                    if q_tmem and j == 0 and tt == 0 and nxt:
                        yield from load_q(nxt)
                    if pend and pend[2] == 0:
                        yield from load_kv("v", pend[0], pend[1])
                    pend = (u, j, tt)
            if not q_tmem and nxt:
                yield from load_q(nxt)
        if pend and pend[2] == 0:
            yield from load_kv("v", pend[0], pend[1])

    # ------------------------------ MMA issuers ------------------------------
    # NT = 2: one issuer per query tile; its tile's chain is Q K^T(j), P V(j) once P(j) is out,
    # then Q K^T(j+1) (one score buffer per tile). NT = 1: one issuer; the tile alternates
    # between the two score buffers, so Q K^T(g+1) goes before P V(g).
    def mma(tiles):
        st = {"k": 0, "v": 0, "units": 0, "kslot": None}
        me = tiles[0]

        class Q:  # this issuer's view of the tensor queue
            @staticmethod
            def append(x):
                tensor.append((me,) + x)

        def take_k():
            s = st["k"] % NK
            ph = (st["k"] // NK) & 1
            st["k"] += 1
            yield from wait(kfull[s], ph)
            st["kslot"] = s

        def qk_op(s, item, sb, halves):
            def op():
                check(kslot[s] == item[:2], f"Q K^T {item} reads K {kslot[s]}")
                q = qtm.get(item[2]) if q_tmem else qstage[0]
                check(q == item[0], f"Q K^T {item} reads the Q of unit {q}")
                b = sbuf[sb]
                for h in halves:
                    free = ("consumed",) if h == "lo" else ("read", "consumed")
                    check(b[h] is None or b[h][1] in free, f"Q K^T {item} overwrites {h} {b[h]}")
                    b[h] = (item, "S")
            return op

        def qk(u, j, tt, sb, last):  # a whole Q K^T (both key halves) into score buffer sb
            if q_tmem and j == 0:
                yield from wait(q_tmem_bar[tt], st["units"] & 1)
            yield from take_k()
            s = st["kslot"]
            Q.append(("op", qk_op(s, (u["id"], j, tt), sb, ("lo", "hi"))))
            Q.append(("commit", s_full[sb]))
            Q.append(("commit", kempty[s]))
            if not q_tmem and last:
                Q.append(("commit", q_empty))
            yield True

        def pv(sb, ph, u, j, tt, last_block, uidx):
            item = (u["id"], j, tt)
            yield from wait(p_full[sb], ph)
            if j == 0 and uidx > 0 and mutant != "no_o_free_wait":
                yield from wait(o_free[tt], (uidx - 1) & 1)
            s = st["v"] % NV
            ph = (st["v"] // NV) & 1
            st["v"] += 1
            yield from wait(vfull[s], ph)

            def op(s=s, item=item, sb=sb):
                check(vslot[s] == item[:2], f"P V {item} reads V {vslot[s]}")
                lo = sbuf[sb]["lo"]
                check(lo == (item, "P"), f"P V {item} reads {lo}")
                sbuf[sb]["lo"] = (item, "consumed")
                o = obuf.get(item[2])
                if item[1] == 0:
                    check(o is None or o[2] == "read", f"P V {item} overwrites unread O {o}")
                    obuf[item[2]] = [item[0], 1, "acc"]
                else:
                    check(o[0] == item[0] and o[1] == item[1], f"P V {item} finds O {o}")
                    o[1] += 1
            Q.append(("op", op))
            if NT == 1 or pipe:
                Q.append(("commit", pv_done[tt]))
            Q.append(("commit", vempty[s]))
            if last_block:
                Q.append(("commit", o_full[tt]))
            yield True

        pend = None
        jg = 0
        for u in busy:
            if not q_tmem:
                yield from wait(q_full, st["units"] & 1)
            for j in range(u["n"]):
                last = j == u["n"] - 1
                for tt in tiles:
                    sb = sbuf_of(jg, tt)
                    if NT == 2 and not pipe:
                        yield from qk(u, j, tt, sb, last)
                        yield from pv(sb, sphase_of(jg), u, j, tt, last, st["units"])
                    else:
                        yield from qk(u, j, tt, sb, last)
                        if pend:
                            yield from pv(*pend)
                        pend = (sb, sphase_of(jg), u, j, tt, last, st["units"])
                jg += 1
            st["units"] += 1
        if pend:
            yield from pv(*pend)
        Q.append(("commit", mma_done))
        yield True

    # ------------------------ softmax + epilogue warpgroups ------------------------
    def softmax(tiles):
        """One warpgroup handling the query tiles in `tiles` (all of them when NSM = 1)."""
        def copy_q(qidx, tt, expect):
            yield from wait(q_full, qidx & 1)
            check(qstage[0] == expect, f"Q copy for tile {tt} finds unit {qstage[0]}, "
                                       f"expected {expect}")
            qtm[tt] = qstage[0]
            q_tmem_bar[tt].arrive(128)
            q_empty.arrive(128)
            yield True

        def epilogue(u, tt, uidx):
            yield from wait(o_full[tt], uidx & 1)
            o = obuf[tt]
            check(o[0] == u["id"] and o[1] == u["n"] and o[2] == "acc",
                  f"epilogue of unit {u['id']} tile {tt} finds O {o}")
            o[2] = "read"
            o_free[tt].arrive(128)
            yield True

        if q_tmem and busy:
            for tt in tiles:
                yield from copy_q(0, tt, busy[0]["id"])
        jg = 0
        pend = None
        for ui, u in enumerate(busy):
            nxt = busy[ui + 1] if ui + 1 < len(busy) else None
            for j in range(u["n"]):
                for tt in tiles:
                    sb = sbuf_of(jg, tt)
                    item = (u["id"], j, tt)
                    def take_turn():  # the two tiles' softmax take turns, block by block
                        if tt == 1:
                            yield from wait(p_full[0], jg & 1)
                        elif jg > 0:
                            yield from wait(p_full[1], (jg - 1) & 1)
                    if NT == 2 and not pipe and not late_turn:
                        yield from take_turn()
                    parity = sphase_of(jg) ^ (1 if mutant == "s_full_wrong_parity" else 0)
                    yield from wait(s_full[sb], parity)
                    if q_tmem and j == u["n"] - 1 and nxt:
                        yield from copy_q(ui + 1, tt, nxt["id"])
                    b = sbuf[sb]
                    check(b["lo"] == (item, "S") and b["hi"] == (item, "S"),
                          f"softmax of {item} reads {b}")
                    b["lo"], b["hi"] = (item, "read"), (item, "read")
                    if NT == 2 and not pipe and late_turn:
                        yield from take_turn()
                    if j > 0 and rnd.random() < 0.3:  # the running max grew: rescale O
                        if (NT == 1 or pipe) and mutant != "no_pv_done_wait":
                            yield from wait(pv_done[tt], (jg - 1) & 1)
                        o = obuf.get(tt)
                        check(o is not None and o[0] == u["id"] and o[1] == j,
                              f"rescale of {item} finds O {o}")
                    if mutant == "p_full_early":
                        p_full[sb].arrive(128)
                        yield True
                        b["lo"] = (item, "P")
                    else:
                        yield True
                        b["lo"] = (item, "P")
                        p_full[sb].arrive(128)
                    if j == 0 and pend:
                        yield from epilogue(pend[0], tt, pend[1])
                jg += 1
            pend = (u, ui)
        if pend:
            for tt in tiles:
                yield from epilogue(pend[0], tt, pend[1])

    roles = {"tma": producer()}
    for t in range(NT):  # one MMA issuer per query tile
        roles[f"mma{t}"] = mma([t])
    if NSM == 1:
        roles["softmax"] = softmax(list(range(NT)))
    else:
        for t in range(NT):
            roles[f"softmax{t}"] = softmax([t])
    blocked = set()
    steps = 0
    while roles or landings or tensor:
        steps += 1
        if steps > 5_000_000:
            raise Deadlock("step limit")
        if not landings and not tensor and roles and blocked >= set(roles):
            raise Deadlock(f"every role waits: {[(r, waits.get(r)) for r in sorted(roles)]}")
        choices = list(roles) + ["land"] * (2 if landings else 0) + ["tensor"] * (2 if tensor else 0)
        c = rnd.choice(choices)
        if c == "land":
            landings.pop(rnd.randrange(len(landings)) if rnd.random() < 0.3 else 0)()
            blocked.clear()
        elif c == "tensor":
            # the next operation of a random issuer (in issue order within each issuer)
            issuer = rnd.choice(sorted({e[0] for e in tensor}))
            idx = next(i for i, e in enumerate(tensor) if e[0] == issuer)
            _, kind, x = tensor.pop(idx)
            x() if kind == "op" else x.arrive(1)
            blocked.clear()
        else:
            current[0] = c
            before = (clock[0], len(landings), len(tensor))
            try:
                progressed = next(roles[c])
            except StopIteration:
                del roles[c]
                blocked.discard(c)
                continue
            # a step that changed any barrier or issued any load or MMA made progress, even if
            # it then blocked on its next wait
            if progressed or before != (clock[0], len(landings), len(tensor)):
                blocked.clear()
            else:
                blocked.add(c)
    check(mma_done.completed == 1, "MMAs not drained")  # every issuer committed once
    return steps


# The kernel's layouts: (NT, NSM, Q in tensor memory, K slots, V slots, pipelined two-tile), from
# the traits table of csrc/attn_api.cu (d64, d128, d192/128, d256, E4M3 d128) plus ring-depth
# edge cases (a single slot) and layouts the kernel supports but does not dispatch.
LAYOUTS = [(2, 2, True, 8, 8, True), (2, 2, False, 3, 2, False), (2, 2, False, 2, 1, False),
           (1, 1, True, 2, 2, False), (2, 2, False, 4, 4, False), (1, 1, True, 6, 6, False),
           (2, 2, True, 1, 1, True), (1, 1, False, 1, 1, False), (2, 2, False, 1, 1, False),
           (2, 2, False, 2, 2, True), (2, 2, True, 5, 5, False), (2, 2, False, 5, 3, False)]


def random_units(rnd):
    n = rnd.randint(1, 6)
    return [{"id": i, "n": rnd.choice([0, 1, 1, 2, 3, 5]) if rnd.random() < 0.5
             else rnd.randint(1, 4)} for i in range(n)]
