"""CPU model of the prefill kernel's barrier protocol (exact_attention_139_b200/csrc/prefill2.cuh).

The kernel's roles are transcribed as generators that yield the barrier waits they make:
  * the TMA producer (the Q slots of a unit's two query tiles, and a ring of NS stages, stage t
    holding K and V of key tile t under one barrier);
  * the MMA issuer (S = Q.K^T and O += P.V products, commits to the barriers);
  * the two softmax warpgroups (S -> P in TMEM, handed over in two halves: keys 0-63 under a
    half barrier, then all of P; a warpgroup that rescales O hands both over after the rescale; at
    the end of a unit they leave the row statistics in one of two shared-memory buffers per tile
    and move on);
  * the epilogue warpgroup (per output tile: waits for the last P.V and the statistics, reads O
    out of TMEM and releases it).
Tensor-core work runs in issue order on a FIFO "pipe"; TMA loads complete in random order. Every
product checks, when it executes, that the buffers it reads hold the content it expects (the right
Q tile, K or V tile, P of the right step, O accumulated up to the previous step), so a slot that
is refilled or overwritten too early fails the run; a state in which no role, product or load can
move is a deadlock and fails the run too. The scheduler picks among runnable actions at random.

This checks the ordering logic only (which barrier guards which buffer), not the arithmetic.
"""
from __future__ import annotations

import random


class Fail(Exception):
    pass


class Bar:
    """An mbarrier: `count` arrivals plus a transaction count complete a phase."""

    def __init__(self, name, count=1):
        self.name, self.count = name, count
        self.pending, self.tx, self.phase = count, 0, 0  # phase = phases completed so far

    def arrive(self):
        self.pending -= 1
        if self.pending < 0:
            raise Fail(f"{self.name}: too many arrivals")
        self._check()

    def expect_tx(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        # the phase with this parity has completed once the current phase's parity differs
        return (self.phase & 1) != parity


def kv_tiles(Lq, Lk, causal, r0):
    """Key tiles a 128-row query tile starting at row r0 needs (0 past the last row)."""
    if r0 >= Lq:
        return 0
    n = (Lk + 127) // 128
    if causal:
        last = min(r0 + 127, Lq - 1)
        n = min(n, (last + (Lk - Lq)) // 128 + 1)
    return n


def unit_lists(units, geom, sparse_rng=None):
    """Per unit, the sorted key-tile list of tile A and of tile B. Dense: 0 .. n-1. Sparse: a
    random subset of the dense range (possibly empty), as a caller-given block list."""
    Lq, Lk, causal = geom
    out = []
    for rows in units:
        lists = []
        for r0 in rows:
            n = kv_tiles(Lq, Lk, causal, r0)
            if sparse_rng is None:
                lists.append(list(range(n)))
            else:
                lists.append(sorted(t for t in range(n) if sparse_rng.random() < 0.6))
        out.append(lists)
    return out


def union_walk(la, lb):
    """(block, in_a, in_b) over the union of two sorted lists, as the kernel's UnionWalk."""
    ia = ib = 0
    while ia < len(la) or ib < len(lb):
        ka = la[ia] if ia < len(la) else None
        kc = lb[ib] if ib < len(lb) else None
        kb = min(k for k in (ka, kc) if k is not None)
        in_a, in_b = ka == kb, kc == kb
        ia += in_a
        ib += in_b
        yield kb, in_a, in_b


def run(lists, NS, seed, mut=0):
    """Run one CTA's units (lists[u] = [blocks of tile A, blocks of tile B]) to completion.
    `mut` plants one protocol slip (see mutation_check)."""
    rng = random.Random(seed)
    B = {}
    for name in ["q_full", "q_empty"] + [f"kv_{k}{i}" for i in range(NS) for k in ("full", "empty")]:
        B[name] = Bar(name)
    for x in range(2):
        B[f"s_full{x}"] = Bar(f"s_full{x}")
        B[f"p_full{x}"] = Bar(f"p_full{x}")
        B[f"p_half{x}"] = Bar(f"p_half{x}")
        B[f"o_ready{x}"] = Bar(f"o_ready{x}")
        B[f"o_free{x}"] = Bar(f"o_free{x}")
        for b in range(2):
            B[f"stats_ready{x}{b}"] = Bar(f"stats_ready{x}{b}")

    qslot = [None, None]       # ("Q", unit) per slot
    stage = [None] * NS        # ("KV", tile seq) per stage (K and V of one key tile)
    scol = [None, None]        # TMEM S_x columns: ("S" | "Ph" (first half of P) | "P", unit, step)
    ocol = [None, None]        # TMEM O_x: (unit, steps accumulated, first half of the next step in)
    epi_done = [set(), set()]  # units whose epilogue has read O_x
    stats = [[None, None], [None, None]]  # per tile, two buffers: the unit whose statistics they hold
    pipe = []                  # FIFO of ("mma", fn) / ("commit", bar)
    tma = []                   # pending loads: (bar, land fn)
    active = [u for u, (la, lb) in enumerate(lists) if la or lb]

    # ---------------- TMA producer ----------------
    def producer():
        kv_t = qc = 0
        for u in active:
            la, lb = lists[u]
            if qc > 0 and mut != 5:
                yield ("wait", "q_empty", (qc - 1) & 1)
            B["q_full"].expect_tx(1)

            def land_q(u=u):
                qslot[0] = qslot[1] = ("Q", u)
            tma.append(("q_full", land_q))
            qc += 1
            for _ in union_walk(la, lb):
                s = kv_t % NS
                if kv_t >= NS:
                    yield ("wait", f"kv_empty{s}", ((kv_t // NS) & 1) ^ 1)
                B[f"kv_full{s}"].expect_tx(1)

                def land(s=s, tag=("KV", kv_t)):
                    stage[s] = tag
                tma.append((f"kv_full{s}", land))
                kv_t += 1

    # ---------------- MMA issuer ----------------
    def issuer():
        p_cnt = [0, 0]
        units_done = [0, 0]
        qc = 0
        kv_t = 0

        def wait_stage(idx):
            yield ("wait", f"kv_full{idx % NS}", (idx // NS) & 1)

        def issue_s(x, sidx, u, j):
            def ex(x=x, sidx=sidx, u=u, j=j):
                if qslot[x] != ("Q", u):
                    raise Fail(f"S{x}({u},{j}) reads Q slot holding {qslot[x]}")
                if stage[sidx % NS] != ("KV", sidx):
                    raise Fail(f"S{x}({u},{j}) reads stage holding {stage[sidx % NS]}, wants tile {sidx}")
                if scol[x] is not None and scol[x][0] == "S":
                    raise Fail(f"S{x}({u},{j}) overwrites unread {scol[x]}")
                if scol[x] is not None and scol[x][0] == "P" and not consumed[x]:
                    raise Fail(f"S{x}({u},{j}) overwrites P {scol[x]} before its P.V")
                scol[x] = ("S", u, j)
                consumed[x] = False
            pipe.append(("mma", ex))
            pipe.append(("commit", f"s_full{x}"))

        def issue_pv(x, sidx, u, jx, half):
            def ex(x=x, sidx=sidx, u=u, jx=jx, half=half):
                ready = ("Ph", "P") if half == 0 else ("P",)
                if scol[x] is None or scol[x][0] not in ready or scol[x][1] != u:
                    raise Fail(f"PV{x}({u},{jx}) half {half} reads S columns holding {scol[x]}")
                if stage[sidx % NS] != ("KV", sidx):
                    raise Fail(f"PV{x}({u},{jx}) reads stage holding {stage[sidx % NS]}, wants tile {sidx}")
                if half == 1:
                    if ocol[x] != (u, jx, 1):
                        raise Fail(f"PV{x}({u},{jx}) second half accumulates onto {ocol[x]}")
                    ocol[x] = (u, jx + 1, 0)
                    consumed[x] = True
                elif jx == 0:
                    prev = [w for w in active if w < u and lists[w][x]]
                    if prev and prev[-1] not in epi_done[x]:
                        raise Fail(f"PV{x}({u},0) overwrites O before the epilogue of unit {prev[-1]}")
                    ocol[x] = (u, 0, 1)
                else:
                    if ocol[x] != (u, jx, 0):
                        raise Fail(f"PV{x}({u},{jx}) accumulates onto {ocol[x]}")
                    ocol[x] = (u, jx, 1)
            pipe.append(("mma", ex))

        for u in active:
            lx = lists[u]
            steps = list(union_walk(*lx))
            n = len(steps)
            yield ("wait", "q_full", qc & 1)
            qc += 1
            _, a0, b0 = steps[0]
            inn = [a0, b0]
            if mut != 4:
                yield from wait_stage(kv_t)
            for x in range(2):
                if inn[x]:
                    issue_s(x, kv_t, u, 0)
            if n == 1:
                pipe.append(("commit", "q_empty"))
            jx = [0, 0]
            for j in range(n):
                si = kv_t + j
                in_next = [steps[j + 1][1], steps[j + 1][2]] if j + 1 < n else [False, False]
                x_last = 1 if inn[1] else 0  # last tile whose P.V reads this stage
                if mut == 2:
                    x_last = 0 if inn[0] else 1
                next_ready = False
                for x in range(2):
                    if inn[x]:
                        if jx[x] == 0 and units_done[x] > 0 and mut != 8:
                            yield ("wait", f"o_free{x}", (units_done[x] - 1) & 1)
                        yield ("wait", f"p_half{x}", p_cnt[x] & 1)
                        issue_pv(x, si, u, jx[x], 0)
                        if mut != 10:
                            yield ("wait", f"p_full{x}", p_cnt[x] & 1)
                        p_cnt[x] += 1
                        issue_pv(x, si, u, jx[x], 1)
                        if x == x_last and mut != 1:
                            pipe.append(("commit", f"kv_empty{si % NS}"))
                    if in_next[x]:
                        if not next_ready:
                            if mut != 3:
                                yield from wait_stage(si + 1)
                            next_ready = True
                        issue_s(x, si + 1, u, j + 1)
                    if inn[x]:
                        if jx[x] == len(lx[x]) - 1:
                            pipe.append(("commit", f"o_ready{x}"))
                            units_done[x] += 1
                        jx[x] += 1
                if j == n - 2:
                    pipe.append(("commit", "q_empty"))
                inn = in_next
            kv_t += n

    # ---------------- softmax warpgroups ----------------
    def softmax(x):
        s_cnt = e_cnt = 0
        for u in active:
            nt = len(lists[u][x])
            for j in range(nt):
                yield ("wait", f"s_full{x}", s_cnt & 1)
                s_cnt += 1
                if scol[x] is None or scol[x][:2] != ("S", u):
                    raise Fail(f"softmax{x}({u},{j}) reads {scol[x]}")
                tag = scol[x][1:]
                if j > 0 and rng.random() < 0.3:
                    # rescale O after all of P is written, then hand both halves over
                    scol[x] = ("P",) + tag
                    if mut == 11:  # the first half handed over before the rescale
                        B[f"p_half{x}"].arrive()
                    yield ("step",)
                    if ocol[x] != (u, j, 0):
                        raise Fail(f"softmax{x}({u},{j}) rescales O holding {ocol[x]}")
                    if mut != 11:
                        B[f"p_half{x}"].arrive()
                    B[f"p_full{x}"].arrive()
                else:
                    scol[x] = ("Ph",) + tag
                    B[f"p_half{x}"].arrive()
                    yield ("step",)
                    scol[x] = ("P",) + tag
                    B[f"p_full{x}"].arrive()
            if nt == 0:
                continue
            b = e_cnt & 1 if mut != 6 else 0
            if stats[x][b] is not None:
                raise Fail(f"softmax{x}({u}) overwrites the statistics of unit {stats[x][b]} before the epilogue read them")
            stats[x][b] = u
            e_cnt += 1
            B[f"stats_ready{x}{b if mut != 9 else 0}"].arrive()

    # ---------------- epilogue warpgroup ----------------
    def epilogue():
        ecnt = [0, 0]
        for u in active:
            for x in range(2):
                nt = len(lists[u][x])
                if nt == 0:
                    continue
                par = ecnt[x] & 1
                if mut != 7:
                    yield ("wait", f"o_ready{x}", par)
                if mut != 9:
                    yield ("wait", f"stats_ready{x}{par}", (ecnt[x] >> 1) & 1)
                else:  # one barrier for both buffers: its phases can run two ahead of this wait
                    yield ("wait", f"stats_ready{x}0", par)
                ecnt[x] += 1
                if stats[x][par] != u:
                    raise Fail(f"epilogue{x}({u}) reads statistics of unit {stats[x][par]}")
                stats[x][par] = None
                if ocol[x] != (u, nt, 0):
                    raise Fail(f"epilogue{x}({u}) reads O holding {ocol[x]}")
                epi_done[x].add(u)
                B[f"o_free{x}"].arrive()

    consumed = [True, True]
    roles = {"producer": producer(), "issuer": issuer(), "smA": softmax(0), "smB": softmax(1),
             "epilogue": epilogue()}
    waiting = {name: None for name in roles}
    alive = set(roles)
    steps = 0
    while alive or pipe or tma:
        steps += 1
        choices = [("role", r) for r in sorted(alive)
                   if waiting[r] is None or waiting[r][0] == "step" or B[waiting[r][1]].done(waiting[r][2])]
        if pipe:
            choices.append(("pipe", None))
        if tma:
            choices.append(("tma", None))
        if not choices:
            raise Fail("deadlock: " + str({n: waiting[n][1:] for n in alive}))
        kind, name = rng.choice(choices)
        if kind == "role":
            try:
                waiting[name] = next(roles[name])
            except StopIteration:
                alive.discard(name)
                waiting[name] = None
        elif kind == "pipe":
            op, arg = pipe.pop(0)
            if op == "mma":
                arg()
            else:
                B[arg].arrive()
        else:
            b, land = tma.pop(rng.randrange(len(tma)))
            land()
            B[b].complete_tx(1)
    return steps


def cta_units(Lq, Hq, batch, grid, cta, sib=False):
    """One CTA's units in the kernel's order (one scheduling group), as (row0_A, row0_B): pairs of
    adjacent 128-row tiles of one head, or (sib) the same 128 rows of two sibling heads; heaviest
    level first, dealt boustrophedon over `grid` CTAs."""
    n_qt = (Lq + 127) // 128
    n_lvl = n_qt if sib else (n_qt + 1) // 2
    hpl = Hq // 2 if sib else Hq
    n_units = n_lvl * batch * hpl
    out = []
    k, u = 0, cta
    while u < n_units:
        lvl = u // (batch * hpl)
        if sib:
            q0 = (n_lvl - 1 - lvl) * 128
            out.append((q0, q0))
        else:
            q0 = (n_lvl - 1 - lvl) * 256
            out.append((q0, q0 + 128))
        k += 1
        u = k * grid + ((grid - 1 - cta) if (k & 1) else cta)
    return out


GEOMS = [(128, 128, True), (256, 256, True), (384, 384, True), (1024, 1024, True), (300, 1000, True),
         (1000, 1000, False), (129, 129, True), (640, 640, False), (100, 100, True)]
# the kernel uses NS = 2 (d = 128) and 3 (d = 64); one stage deadlocks (the issuer needs the next
# tile's stage for its S before the P.V that releases the current one), which the model finds
RINGS = [2, 3]


def check(trials=20, geoms=GEOMS, rings=RINGS, mut=0):
    """First failure over dense and sparse runs of the given ring depths and shapes, or None."""
    for NS in rings:
        for geom in geoms:
            for grid, sib in ((1, False), (3, False), (1, True), (3, True)):
                units = cta_units(geom[0], 2, 2, grid, 0, sib)
                for t in range(trials):
                    for sparse in ((False,) if sib else (False, True)):
                        lists = unit_lists(units, geom, random.Random(1000 + t) if sparse else None)
                        try:
                            run(lists, NS, seed=t, mut=mut)
                        except Fail as e:
                            return dict(NS=NS, geom=geom, grid=grid, sib=sib, seed=t, sparse=sparse, error=str(e))
    return None


# planted slips: 1 a stage never released; 2 a stage released after the first instead of the last
# P.V of its key tile; 3 the next key tile's S issued without waiting for its stage; 4 a unit's
# first S issued without waiting for its stage; 5 Q reloaded without waiting for its slot; 6 one
# statistics buffer per tile instead of two; 7 the epilogue reads O without waiting for the last
# P.V; 8 the first P.V of a unit issued without waiting for the previous epilogue to release O;
# 9 one statistics-ready barrier for both buffers of a tile (a tile whose units have a single key
# tile can then complete two phases before the epilogue waits for the first: a parity wait
# cannot tell them apart); 10 the second half of a key tile's P.V issued without waiting for all
# of P; 11 a warpgroup that rescales O hands the first half of P over before the rescale
MUTANTS = (1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11)


def mutation_check(trials=20):
    return {m: check(trials=trials, rings=[2, 3], geoms=GEOMS[:6], mut=m) for m in MUTANTS}


if __name__ == "__main__":
    print("clean:", check(trials=60))
    for m, r in mutation_check().items():
        print("mutant", m, "caught" if r else "NOT caught", r)
