"""CPU model checks of the kernels' barrier protocols (no GPU).

Each model restates, role by role, the waits, arrivals, commits, tensor-core products and
copies of one kernel as written in csrc/flex_fwd_sm100.cuh (flex_fwd_kernel: TMA producer,
one MMA-issuing thread per query tile, two softmax warpgroups) and csrc/flex_bwd_sm100.cuh (bwd_dq_kernel
with its separate K and V rings; bwd_dkdv_kernel with its query-half pipelining).
tests/protocol_model.py runs them under many random schedules with the hardware's
phase-parity rule for mbarrier waits and checks that no schedule deadlocks and that every
product and every element-wise pass reads the tile it expects (a slot or tensor-memory
region overwritten too early shows up as a stale tag).  Planted mistakes (a K slot
released before dQ has read it, a Q/dO slot released after the first query half, a
second issuer releasing skipped slots without waiting, slots released by the first of two
issuers) must be caught, which pins the checker.  The models check ordering only, not memory visibility between proxies.
"""
import random

import pytest

from protocol_model import Bar, Deadlock, Hazard, run

TB = 32768


class _Model:
    def __init__(self):
        self.bars = {}

    def bar(self, name, count=1):
        self.bars[name] = Bar(name, count)
        return self.bars[name]


# ----------------------------------------------------------------------------- forward

def fwd_roles(sets, NS, issuers="two"):
    """Two query tiles with key-tile sets `sets` (descending), an NS-slot K/V ring.
    issuers: "two" (the kernel: one MMA-issuing thread per query tile, each waiting for
    every use of a slot before releasing it, even on steps its tile skips), "one" (the
    earlier single issuer), or the planted mistakes "two_naive" (a skipped step's slots
    released without waiting for them) and "two_count1" (slots released by whichever
    issuer finishes first: empty barriers expecting one arrival)."""
    m = _Model()
    two = issuers != "one"
    bar_q = m.bar("q")
    full = [m.bar(f"full{s}") for s in range(NS)]
    empty = [m.bar(f"empty{s}", 2 if two and issuers != "two_count1" else 1) for s in range(NS)]
    bar_s = [m.bar("s0"), m.bar("s1")]
    bar_p = [[m.bar(f"p{k}{h}") for h in range(2)] for k in range(2)]
    bar_o = [m.bar("o0"), m.bar("o1")]
    drain = [m.bar("drain0"), m.bar("drain1")]
    steps = sorted(set(sets[0]) | set(sets[1]), reverse=True)

    def rec(t):  # the step record: per visiting tile, "pre", "last" or "later"
        j, jn = steps[t], (steps[t + 1] if t + 1 < len(steps) else None)
        r = {}
        for k in range(2):
            if j in sets[k]:
                i = sets[k].index(j)
                nxt = sets[k][i + 1] if i + 1 < len(sets[k]) else None
                r[k] = "last" if nxt is None else ("pre" if nxt == jn else "later")
        return r

    def producer():
        yield ("write", {("rec", NS): ("rec", 0)})  # the first step's record, with Q
        yield ("expect", bar_q, TB)
        yield ("tma", ("Q",), "Q", bar_q, TB)
        r = 0
        for t, j in enumerate(steps):
            for which in ("K", "V"):
                s = r % NS
                yield ("wait", empty[s], ((r // NS) & 1) ^ 1)
                if which == "V":  # the next step's record travels with V of this step
                    yield ("write", {("rec", s): ("rec", t + 1)})
                yield ("expect", full[s], TB)
                yield ("tma", ("slot", s), (which, j), full[s], TB)
                r += 1
        for e in range(max(0, r - NS), r):
            yield ("wait", full[e % NS], (e // NS) & 1)

    def S(k, j, slot):  # P aliases the first columns of S
        return ("mma", [(("Q",), "Q"), (("slot", slot), ("K", j))],
                {("S", k): ("S", j), ("P", k, 0): ("Sx", j), ("P", k, 1): ("Sx", j)})

    def PV(k, j, half, slot, count):
        reads = [(("P", k, half), ("P", j, half)), (("slot", slot), ("V", j))]
        if count > 0:
            reads.append((("O", k), count))
        return ("mma", reads, {("O", k): count + 1})

    def issuer_one():
        yield ("wait", bar_q, 0)
        yield ("read", [(("rec", NS), ("rec", 0))])
        s_ready, np_ = [False, False], [0, 0]
        for t, j in enumerate(steps):
            rK, rV = 2 * t, 2 * t + 1
            sK, sV = rK % NS, rV % NS
            r = rec(t)
            need = [k in r and not s_ready[k] for k in range(2)]
            if any(need):
                yield ("wait", full[sK], (rK // NS) & 1)
                for k in range(2):
                    if need[k]:
                        yield S(k, j, sK)
                        yield ("commit", bar_s[k])
            yield ("commit", empty[sK])
            yield ("wait", full[sV], (rV // NS) & 1)
            yield ("read", [(("rec", sV), ("rec", t + 1))])
            next_k_ready = False
            for k in range(2):
                if k not in r:
                    continue
                s_ready[k] = False
                for half in range(2):
                    yield ("wait", bar_p[k][half], np_[k] & 1)
                    yield PV(k, j, half, sV, 2 * np_[k] + half)
                np_[k] += 1
                if r[k] == "pre":
                    rK2 = rK + 2
                    if not next_k_ready:
                        yield ("wait", full[rK2 % NS], (rK2 // NS) & 1)
                        next_k_ready = True
                    yield S(k, steps[t + 1], rK2 % NS)
                    yield ("commit", bar_s[k])
                    s_ready[k] = True
                elif r[k] == "last":
                    yield ("commit", bar_o[k])
            yield ("commit", empty[sV])
        yield ("commit", drain[0])
        yield ("wait", drain[0], 0)

    def issuer_two(k):
        """One issuer per query tile.  On a step its tile skips it still waits for the fill of
        both slots (and reads the record) before arriving on their empty barriers, so it can
        never arrive for a slot's next use before the other issuer has arrived for this one."""
        yield ("wait", bar_q, 0)
        yield ("read", [(("rec", NS), ("rec", 0))])
        s_ready, k_ready, np_ = False, False, 0
        for t, j in enumerate(steps):
            rK, rV = 2 * t, 2 * t + 1
            sK, sV = rK % NS, rV % NS
            r = rec(t)
            visit = k in r
            if not k_ready:
                yield ("wait", full[sK], (rK // NS) & 1)
            k_ready = False
            if visit:
                if not s_ready:
                    yield S(k, j, sK)
                    yield ("commit", bar_s[k])
                s_ready = False
                yield ("commit", empty[sK])
            else:
                yield ("arrive", empty[sK])
            yield ("wait", full[sV], (rV // NS) & 1)
            yield ("read", [(("rec", sV), ("rec", t + 1))])
            if not visit:
                yield ("arrive", empty[sV])
                continue
            for half in range(2):
                yield ("wait", bar_p[k][half], np_ & 1)
                yield PV(k, j, half, sV, 2 * np_ + half)
            np_ += 1
            if r[k] == "pre":
                yield ("wait", full[(rK + 2) % NS], ((rK + 2) // NS) & 1)
                k_ready = True
                yield S(k, steps[t + 1], (rK + 2) % NS)
                yield ("commit", bar_s[k])
                s_ready = True
            elif r[k] == "last":
                yield ("commit", bar_o[k])
            yield ("commit", empty[sV])
        yield ("commit", drain[k])
        yield ("wait", drain[k], 0)

    def issuer_naive(k):
        yield ("wait", bar_q, 0)
        s_ready, np_ = False, 0
        for t, j in enumerate(steps):
            rK, rV = 2 * t, 2 * t + 1
            sK, sV = rK % NS, rV % NS
            r = rec(t)
            if k not in r:
                yield ("arrive", empty[sK])  # the mistake: no wait for this use of the slots
                yield ("arrive", empty[sV])
                continue
            if not s_ready:
                yield ("wait", full[sK], (rK // NS) & 1)
                yield S(k, j, sK)
                yield ("commit", bar_s[k])
            yield ("commit", empty[sK])
            yield ("wait", full[sV], (rV // NS) & 1)
            for half in range(2):
                yield ("wait", bar_p[k][half], np_ & 1)
                yield PV(k, j, half, sV, 2 * np_ + half)
            np_ += 1
            s_ready = False
            if r[k] == "pre":
                yield ("wait", full[(rK + 2) % NS], ((rK + 2) // NS) & 1)
                yield S(k, steps[t + 1], (rK + 2) % NS)
                yield ("commit", bar_s[k])
                s_ready = True
            elif r[k] == "last":
                yield ("commit", bar_o[k])
            yield ("commit", empty[sV])
        yield ("commit", drain[k])
        yield ("wait", drain[k], 0)

    def softmax(k):
        for v, j in enumerate(sets[k]):
            yield ("wait", bar_s[k], v & 1)
            yield ("read", [(("S", k), ("S", j))])
            if v > 0:  # a lazy rescale of O needs every earlier P.V product in
                yield ("read", [(("O", k), 2 * v)])
            for half in range(2):
                yield ("write", {("P", k, half): ("P", j, half)})
                yield ("arrive", bar_p[k][half])
        if sets[k]:
            yield ("wait", bar_o[k], 0)
            yield ("read", [(("O", k), 2 * len(sets[k]))])

    roles = {"producer": producer(), "sm0": softmax(0), "sm1": softmax(1)}
    if issuers == "two_naive":
        roles["I0"], roles["I1"] = issuer_naive(0), issuer_naive(1)
    elif two:
        roles["I0"], roles["I1"] = issuer_two(0), issuer_two(1)
    else:
        roles["I"] = issuer_one()
    return roles, m.bars


def fwd_persistent_roles(units, NS, wait_q_free=True, q_free_at="last_step"):
    """The persistent forward: one CTA runs the units (each a pair of key-tile sets) in
    order with one MMA issuer.  The K/V ring and every barrier's phases run on across
    units, and so does the issuer's step loop: the record carried with V of a unit's last
    step is the next unit's first record (flagged as a new unit), at which the issuer
    waits for the next phase of the Q barrier.  The producer loads a unit's Q tiles once
    the S products of the previous unit have completed (Q free), which the issuer commits
    at the unit's last step, after reading the chained record and before that step's P.V
    products.  The first P.V of a tile in a unit overwrites its O accumulator; it needs
    no barrier of its own, since it waits for that tile's first P of the unit, which its
    warpgroup writes only after its epilogue has read O of the previous unit.  Planted
    mistakes: wait_q_free=False (Q loaded without waiting) and q_free_at="first_step" (Q
    released at the unit's first step, before the S products of the later steps)."""
    m = _Model()
    bar_q, q_free = m.bar("q"), m.bar("q_free")
    full = [m.bar(f"full{s}") for s in range(NS)]
    empty = [m.bar(f"empty{s}") for s in range(NS)]
    bar_s = [m.bar("s0"), m.bar("s1")]
    bar_p = [[m.bar(f"p{k}{h}") for h in range(2)] for k in range(2)]
    bar_o = [m.bar("o0"), m.bar("o1")]
    drain = m.bar("drain")
    work = [u for u in units if u[0] or u[1]]
    steps_of = [sorted(set(u[0]) | set(u[1]), reverse=True) for u in work]

    def rec(ui, t):
        sets, steps = work[ui], steps_of[ui]
        j, jn = steps[t], (steps[t + 1] if t + 1 < len(steps) else None)
        r = {}
        for k in range(2):
            if j in sets[k]:
                i = sets[k].index(j)
                nxt = sets[k][i + 1] if i + 1 < len(sets[k]) else None
                r[k] = "last" if nxt is None else ("pre" if nxt == jn else "later")
        return r

    def after(ui, t):  # the record carried with V of step t of unit ui
        if t + 1 < len(steps_of[ui]):
            return ("rec", ui, t + 1)
        return ("rec", ui + 1, 0) if ui + 1 < len(work) else ("end",)

    def producer():
        r = 0
        for ui in range(len(work)):
            if ui == 0:
                yield ("write", {("rec", NS): ("rec", 0, 0)})  # later units' come chained
            elif wait_q_free:
                yield ("wait", q_free, (ui - 1) & 1)
            yield ("expect", bar_q, TB)
            yield ("tma", ("Q",), ("Q", ui), bar_q, TB)
            for t, j in enumerate(steps_of[ui]):
                for which in ("K", "V"):
                    s = r % NS
                    yield ("wait", empty[s], ((r // NS) & 1) ^ 1)
                    if which == "V":
                        yield ("write", {("rec", s): after(ui, t)})
                    yield ("expect", full[s], TB)
                    yield ("tma", ("slot", s), (which, ui, j), full[s], TB)
                    r += 1
        for e in range(max(0, r - NS), r):
            yield ("wait", full[e % NS], (e // NS) & 1)

    def S(ui, k, j, slot):
        return ("mma", [(("Q",), ("Q", ui)), (("slot", slot), ("K", ui, j))],
                {("S", k): ("S", ui, j), ("P", k, 0): ("Sx",), ("P", k, 1): ("Sx",)})

    def PV(ui, k, j, half, slot, first):
        reads = [(("P", k, half), ("P", ui, j, half)), (("slot", slot), ("V", ui, j))]
        if not first:
            reads.append((("O", k), ("O", ui)))
        return ("mma", reads, {("O", k): ("O", ui)})

    def issuer():
        r = 0
        np_, n_o = [0, 0], [0, 0]
        for ui in range(len(work)):
            yield ("wait", bar_q, ui & 1)  # unit 0: before the loop; later: at the chained record
            if ui == 0:
                yield ("read", [(("rec", NS), ("rec", 0, 0))])
            s_ready, started = [False, False], [False, False]
            fin = [not work[ui][0], not work[ui][1]]  # tile k has no key tile left
            released = False
            for t, j in enumerate(steps_of[ui]):
                rK, rV = r, r + 1
                r += 2
                sK, sV = rK % NS, rV % NS
                rc = rec(ui, t)
                need = [k in rc and not s_ready[k] for k in range(2)]
                if any(need):
                    yield ("wait", full[sK], (rK // NS) & 1)
                    for k in range(2):
                        if need[k]:
                            yield S(ui, k, j, sK)
                            yield ("commit", bar_s[k])
                yield ("commit", empty[sK])
                if q_free_at == "first_step" and t == 0 and not released:
                    yield ("commit", q_free)
                    released = True
                yield ("wait", full[sV], (rV // NS) & 1)
                yield ("read", [(("rec", sV), after(ui, t))])
                # the chained record says this is the unit's last step
                last_step = t + 1 == len(steps_of[ui])
                assert last_step == all(rc[k] == "last" if k in rc else fin[k] for k in range(2))
                if last_step and not released:
                    yield ("commit", q_free)
                    released = True
                next_k_ready = False
                for k in range(2):
                    if k not in rc:
                        continue
                    s_ready[k] = False
                    for half in range(2):
                        yield ("wait", bar_p[k][half], np_[k] & 1)
                        yield PV(ui, k, j, half, sV, not started[k] and half == 0)
                    started[k] = True
                    np_[k] += 1
                    if rc[k] == "pre":
                        rK2 = rK + 2
                        if not next_k_ready:
                            yield ("wait", full[rK2 % NS], (rK2 // NS) & 1)
                            next_k_ready = True
                        yield S(ui, k, steps_of[ui][t + 1], rK2 % NS)
                        yield ("commit", bar_s[k])
                        s_ready[k] = True
                    elif rc[k] == "last":
                        yield ("commit", bar_o[k])
                        n_o[k] += 1
                        fin[k] = True
                yield ("commit", empty[sV])
            assert released  # the last step always releases Q
        yield ("commit", drain)
        yield ("wait", drain, 0)

    def softmax(k):
        n, n_o = 0, 0
        for ui in range(len(work)):
            sets = work[ui][k]
            for j in sets:
                yield ("wait", bar_s[k], n & 1)
                yield ("read", [(("S", k), ("S", ui, j))])
                for half in range(2):
                    yield ("write", {("P", k, half): ("P", ui, j, half)})
                    yield ("arrive", bar_p[k][half])
                n += 1
            if sets:
                yield ("wait", bar_o[k], n_o & 1)
                yield ("read", [(("O", k), ("O", ui))])
                n_o += 1

    roles = {"producer": producer(), "I": issuer(), "sm0": softmax(0), "sm1": softmax(1)}
    return roles, m.bars


@pytest.mark.parametrize("NS", [5, 12])
@pytest.mark.parametrize("kind", ["dense", "causal", "random"])
def test_forward_persistent_protocol(NS, kind):
    rng = random.Random(NS * 7 + len(kind))
    cases = [[_sets(rng, rng.choice([1, 2, 3, 5]), kind) for _ in range(rng.randint(1, 5))] for _ in range(30)]
    assert _schedules(lambda i: fwd_persistent_roles(cases[i], NS), len(cases)) == 0


def test_forward_persistent_without_q_free_is_caught():
    rng = random.Random(11)
    cases = [[_sets(rng, rng.choice([1, 2, 3]), "dense") for _ in range(4)] for _ in range(40)]
    assert _schedules(lambda i: fwd_persistent_roles(cases[i], 5, wait_q_free=False), len(cases)) > 0


def test_forward_persistent_q_released_early_is_caught():
    rng = random.Random(12)
    cases = [[_sets(rng, rng.choice([2, 3]), "dense") for _ in range(4)] for _ in range(40)]
    assert _schedules(lambda i: fwd_persistent_roles(cases[i], 5, q_free_at="first_step"), len(cases)) > 0


def _sets(rng, nk, kind):
    if kind == "dense":
        return [list(range(nk - 1, -1, -1))] * 2
    if kind == "causal":
        return [list(range(nk - 2, -1, -1)), list(range(nk - 1, -1, -1))]
    if kind == "one_empty":
        return [list(range(nk - 1, -1, -1)), []]
    sets = [sorted((u for u in range(nk) if rng.random() < 0.5), reverse=True) for _ in range(2)]
    return sets if (sets[0] or sets[1]) else [[0], []]


def _schedules(make, n, seed0=0):
    """Runs n random schedules; returns the number that deadlocked or read a stale tag."""
    bad = 0
    for i in range(n):
        roles, bars = make(i)
        try:
            run(roles, bars, seed0 + i, async_bias=(0.1, 0.5, 0.9)[i % 3])
        except (Hazard, Deadlock):
            bad += 1
    return bad


@pytest.mark.parametrize("issuers", ["two", "one"])
@pytest.mark.parametrize("NS", [5, 12])
@pytest.mark.parametrize("kind", ["dense", "causal", "one_empty", "random"])
def test_forward_protocol(NS, kind, issuers):
    rng = random.Random(NS * 31 + len(kind))
    cases = [_sets(rng, rng.choice([1, 2, 3, 5, 8]), kind) for _ in range(40)]
    assert _schedules(lambda i: fwd_roles(cases[i], NS, issuers), len(cases)) == 0


def test_forward_naive_second_issuer_is_caught():
    rng = random.Random(5)
    cases = [_sets(rng, rng.choice([5, 8, 12]), "one_empty") for _ in range(60)]
    assert _schedules(lambda i: fwd_roles(cases[i], 5, issuers="two_naive"), len(cases)) > 0


def test_forward_single_arrival_release_is_caught():
    rng = random.Random(6)
    cases = [_sets(rng, rng.choice([3, 5, 8]), "random") for _ in range(60)]
    assert _schedules(lambda i: fwd_roles(cases[i], 5, issuers="two_count1"), len(cases)) > 0


# ----------------------------------------------------------------------------- dQ

def dq_roles(n, KS, VS, k_release_after_s=False):
    """bwd_dq_kernel: producer K_0, V_0, K_1, then V_{t+1}, K_{t+2}; K ring KS slots, V ring
    VS slots.  k_release_after_s plants a mistake: the K slot is released once S has read
    it, before dQ has."""
    m = _Model()
    bar_q = m.bar("q")
    full = {"K": [m.bar(f"fk{s}") for s in range(KS)], "V": [m.bar(f"fv{s}") for s in range(VS)]}
    empty = {"K": [m.bar(f"ek{s}") for s in range(KS)], "V": [m.bar(f"ev{s}") for s in range(VS)]}
    sdp, ds = [m.bar("sdp0"), m.bar("sdp1")], [m.bar("ds0"), m.bar("ds1")]
    done = m.bar("done")

    def producer():
        yield ("expect", bar_q, TB)
        yield ("tma", ("Q",), "Q", bar_q, TB)
        order = [("K", 0), ("V", 0)] + ([("K", 1)] if n > 1 else [])
        for t in range(n - 1):
            order += [("V", t + 1)] + ([("K", t + 2)] if t + 2 < n else [])
        cnt, size = {"K": 0, "V": 0}, {"K": KS, "V": VS}
        for kind, tile in order:
            i = cnt[kind]
            slot = i % size[kind]
            yield ("wait", empty[kind][slot], ((i // size[kind]) & 1) ^ 1)
            yield ("expect", full[kind][slot], TB)
            yield ("tma", (kind, slot), (kind, tile), full[kind][slot], TB)
            cnt[kind] += 1
        for kind in ("K", "V"):
            for e in range(max(0, cnt[kind] - size[kind]), cnt[kind]):
                yield ("wait", full[kind][e % size[kind]], (e // size[kind]) & 1)

    kw = lambda t: ("wait", full["K"][t % KS], (t // KS) & 1)
    vw = lambda t: ("wait", full["V"][t % VS], (t // VS) & 1)
    S = lambda t: ("mma", [(("Q",), "Q"), (("K", t % KS), ("K", t))],
                   {("S", t & 1, 0): ("S", t), ("S", t & 1, 1): ("S", t)})
    dP = lambda t, h: ("mma", [(("Q",), "Q"), (("V", t % VS), ("V", t))], {("dP", h): ("dP", t)})

    def dQ(t, h):
        reads = [(("S", t & 1, h), ("dS", t, h)), (("K", t % KS), ("K", t))]
        if t or h:
            reads.append((("dQ",), 2 * t + h))
        return ("mma", reads, {("dQ",): 2 * t + h + 1})

    def issuer():
        yield ("wait", bar_q, 0)
        yield kw(0)
        yield S(0)
        if k_release_after_s:
            yield ("commit", empty["K"][0])
        yield vw(0)
        for h in range(2):
            yield dP(0, h)
            yield ("commit", sdp[h])
        yield ("commit", empty["V"][0])
        if n > 1:
            yield kw(1)
            yield S(1)
            if k_release_after_s:
                yield ("commit", empty["K"][1 % KS])
        for t in range(n):
            yield ("wait", ds[0], t & 1)
            yield dQ(t, 0)
            if t + 1 < n:
                yield vw(t + 1)
                yield dP(t + 1, 0)
                yield ("commit", sdp[0])
            yield ("wait", ds[1], t & 1)
            yield dQ(t, 1)
            if not k_release_after_s:
                yield ("commit", empty["K"][t % KS])
            if t + 1 < n:
                yield dP(t + 1, 1)
                yield ("commit", sdp[1])
                yield ("commit", empty["V"][(t + 1) % VS])
            if t + 2 < n:
                yield kw(t + 2)
                yield S(t + 2)
                if k_release_after_s:
                    yield ("commit", empty["K"][(t + 2) % KS])
        yield ("commit", done)

    def wg(h):
        for t in range(n):
            yield ("wait", sdp[h], t & 1)
            yield ("read", [(("S", t & 1, h), ("S", t)), (("dP", h), ("dP", t))])
            yield ("write", {("S", t & 1, h): ("dS", t, h)})
            yield ("arrive", ds[h])
        yield ("wait", done, 0)
        yield ("read", [(("dQ",), 2 * n)])

    return {"producer": producer(), "I": issuer(), "wg0": wg(0), "wg1": wg(1)}, m.bars


@pytest.mark.parametrize("KS,VS", [(3, 2), (6, 4)])
@pytest.mark.parametrize("n", [1, 2, 3, 5, 9])
def test_dq_protocol(n, KS, VS):
    assert _schedules(lambda i: dq_roles(n, KS, VS), 60) == 0


def test_dq_early_k_release_is_caught():
    assert _schedules(lambda i: dq_roles(6, 3, 2, k_release_after_s=True), 60) > 0


# ----------------------------------------------------------------------------- dK, dV

def dkdv_roles(n, NS, early_release=False):
    """bwd_dkdv_kernel: K, V resident; an NS-slot ring of (Q, dO, statistics) per step.
    early_release plants a mistake: the slot is released after the first query half's
    products, while the second half's still read it."""
    m = _Model()
    bar_kv = m.bar("kv")
    full, empty = [m.bar(f"f{s}") for s in range(NS)], [m.bar(f"e{s}") for s in range(NS)]
    sdp, pds = [m.bar("sdp0"), m.bar("sdp1")], [m.bar("pds0"), m.bar("pds1")]
    done = m.bar("done")

    def producer():
        yield ("expect", bar_kv, TB)
        yield ("tma", ("KV",), "KV", bar_kv, TB)
        for u in range(n):
            s = u % NS
            yield ("wait", empty[s], ((u // NS) & 1) ^ 1)
            yield ("expect", full[s], TB)
            yield ("tma", ("slot", s), ("QO", u), full[s], TB)
        for e in range(max(0, n - NS), n):
            yield ("wait", full[e % NS], (e // NS) & 1)

    sdp_op = lambda u, h: ("mma", [(("KV",), "KV"), (("slot", u % NS), ("QO", u))],
                           {("ST", h): ("S", u), ("dPT", h): ("dP", u)})

    def acc(u, h):
        reads = [(("ST", h), ("P", u, h)), (("dPT", h), ("dS", u, h)), (("slot", u % NS), ("QO", u))]
        if u or h:
            reads += [(("dV",), 2 * u + h), (("dK",), 2 * u + h)]
        return ("mma", reads, {("dV",): 2 * u + h + 1, ("dK",): 2 * u + h + 1})

    def issuer():
        yield ("wait", bar_kv, 0)
        yield ("wait", full[0], 0)
        for h in range(2):
            yield sdp_op(0, h)
            yield ("commit", sdp[h])
        for u in range(n):
            more = u + 1 < n
            yield ("wait", pds[0], u & 1)
            yield acc(u, 0)
            if early_release:
                yield ("commit", empty[u % NS])
            if more:
                yield ("wait", full[(u + 1) % NS], ((u + 1) // NS) & 1)
                yield sdp_op(u + 1, 0)
                yield ("commit", sdp[0])
            yield ("wait", pds[1], u & 1)
            yield acc(u, 1)
            if not early_release:
                yield ("commit", empty[u % NS])
            if more:
                yield sdp_op(u + 1, 1)
                yield ("commit", sdp[1])
        yield ("commit", done)

    def wg(h):
        for u in range(n):
            yield ("wait", sdp[h], u & 1)
            yield ("wait", full[u % NS], (u // NS) & 1)
            yield ("read", [(("ST", h), ("S", u)), (("dPT", h), ("dP", u)), (("slot", u % NS), ("QO", u))])
            yield ("write", {("ST", h): ("P", u, h), ("dPT", h): ("dS", u, h)})
            yield ("arrive", pds[h])
        yield ("wait", done, 0)
        yield ("read", [(("dV",), 2 * n), (("dK",), 2 * n)])

    return {"producer": producer(), "I": issuer(), "wg0": wg(0), "wg1": wg(1)}, m.bars


@pytest.mark.parametrize("NS", [2, 4])
@pytest.mark.parametrize("n", [1, 2, 3, 5, 9])
def test_dkdv_protocol(n, NS):
    assert _schedules(lambda i: dkdv_roles(n, NS), 60) == 0


def test_dkdv_early_slot_release_is_caught():
    assert _schedules(lambda i: dkdv_roles(6, 2, early_release=True), 80) > 0


# ----------------------------------------------------------------------------- decode

def decode_roles(chunk_tiles, NS, consumers=4, shared_ring=False):
    """decode_gqa_tma_kernel: one TMA producer, `consumers` warps taking the CTA's chunks
    round-robin (warp w: chunks w, w + consumers, ...); each chunk is a list of tiles, each
    tile a K then a V load.  The kernel gives every consumer a ring of NS slots of its
    own, which the producer fills in that consumer's order (polling the rings, so one full
    ring does not hold back the others).  shared_ring plants the mistake of one ring of
    consumers * NS slots shared in global order: a consumer whose chunk lies more than a
    ring cycle ahead waits with a parity that an earlier phase of the slot already shows."""
    m = _Model()
    n_slots = consumers * NS
    full = [m.bar(f"full{s}") for s in range(n_slots)]
    empty = [m.bar(f"empty{s}") for s in range(n_slots)]
    own = [[k for k in range(len(chunk_tiles)) if k % consumers == w] for w in range(consumers)]
    loads = {w: [(k, t, which) for k in own[w] for t in range(chunk_tiles[k]) for which in ("K", "V")]
             for w in range(consumers)}
    order = [(k, t, which) for k in range(len(chunk_tiles)) for t in range(chunk_tiles[k]) for which in ("K", "V")]
    gpos = {ld: r for r, ld in enumerate(order)}

    def slot_of(w, i, ld):
        if shared_ring:
            r = gpos[ld]
            return r % n_slots, r // n_slots
        return w * NS + i % NS, i // NS

    def producer():
        if shared_ring:
            for ld in order:
                w = ld[0] % consumers
                s, cyc = slot_of(w, None, ld)
                if cyc > 0:
                    yield ("wait", empty[s], (cyc & 1) ^ 1)
                yield ("expect", full[s], TB)
                yield ("tma", ("slot", s), ld, full[s], TB)
            return
        nxt = [0] * consumers
        while any(nxt[w] < len(loads[w]) for w in range(consumers)):
            progressed = False
            for w in range(consumers):
                i = nxt[w]
                if i >= len(loads[w]):
                    continue
                s, cyc = slot_of(w, i, loads[w][i])
                if cyc > 0 and not empty[s].passes((cyc & 1) ^ 1):
                    continue  # a non-blocking probe: this ring is full, try the next one
                yield ("expect", full[s], TB)
                yield ("tma", ("slot", s), loads[w][i], full[s], TB)
                nxt[w] += 1
                progressed = True
            if not progressed:  # every ring full: block on the oldest pending one
                w = min((w for w in range(consumers) if nxt[w] < len(loads[w])), key=lambda w: nxt[w])
                s, cyc = slot_of(w, nxt[w], loads[w][nxt[w]])
                yield ("wait", empty[s], (cyc & 1) ^ 1)

    def consumer(w):
        for i, ld in enumerate(loads[w]):
            s, cyc = slot_of(w, i, ld)
            yield ("wait", full[s], cyc & 1)
            yield ("read", [(("slot", s), ld)])
            yield ("arrive", empty[s])

    roles = {"producer": producer()}
    for w in range(consumers):
        roles[f"c{w}"] = consumer(w)
    return roles, m.bars


@pytest.mark.parametrize("NS", [3, 6])
def test_decode_ring_protocol(NS):
    rng = random.Random(NS)
    cases = [[rng.choice([1, 2, 3, 4]) for _ in range(rng.randint(1, 13))] for _ in range(50)]
    assert _schedules(lambda i: decode_roles(cases[i], NS), len(cases)) == 0


def test_decode_shared_ring_is_caught():
    rng = random.Random(9)
    cases = [[4] * rng.randint(6, 12) for _ in range(40)]
    assert _schedules(lambda i: decode_roles(cases[i], 3, shared_ring=True), len(cases)) > 0
