"""CPU check of the tcgen05 decode's barrier protocol (csrc/decode_tc_sm100.cuh):
a discrete-event model of every role (TMA producer with its cluster-launch-
control requests, MMA issuer, two groups of four softmax warps, four epilogue
warps) with the kernel's mbarrier counts and parities, the 16-entry unit ring
and its two closing -1 entries, written from the kernel and kept in step with
it by hand. It reuses the simulator of tests/test_backward_design.py: TMA
writes and cancellation responses land asynchronously, the MMAs of the one
issuing thread complete in order and a commit arrives once its earlier MMAs
have.

Under random schedules and unit counts no role deadlocks, and every read (an
MMA operand, a TMEM load of S, O or P, the row sums in shared memory, a
unit-ring entry, V zeroed for a ring that is not full yet) sees the version
it expects over its whole issue-to-completion window. A flipped parity, a
wrong arrival count and a skipped wait each fail some schedule.
"""
import random

import pytest

from test_backward_design import Sim

K_SLOTS, V_SLOTS = 3, 2
QUARTERS = range(4)


def model_decode_tc(sim, n, short_ring, RING=16):
    """n units for this CTA; short_ring[i]: unit i's ring is not full (its
    softmax zeroes V rows of the slot before releasing P); RING entries in the
    unit ring (16 in the kernel)."""
    for s in range(K_SLOTS):
        sim.bar("kq_full%d" % s, 1)
        sim.bar("kq_empty%d" % s, 1)
    for s in range(2):
        for nm, c in (("v_full", 1), ("v_empty", 1), ("s_full", 1), ("s_free", 1),
                      ("p_full", 4), ("l_free", 4)):
            sim.bar("%s%d" % (nm, s), c)
    sim.bar("o_full", 1)
    sim.bar("o_empty", 4)
    for e in range(RING):
        sim.bar("ur_full%d" % e, 1)
        sim.bar("ur_empty%d" % e, 9)
    sim.bar("clc", 1)

    def read_unit(i):
        e = i % RING
        yield ("wait", "ur_full%d" % e, (i // RING) & 1)
        yield ("read", [(("UR", e), ("U", i))])
        yield ("arrive", "ur_empty%d" % e)

    def producer():
        def publish(j):
            e = j % RING
            yield ("wait", "ur_empty%d" % e, ((j // RING) & 1) ^ 1)
            yield ("write", [(("UR", e), ("U", j))])
            yield ("arrive", "ur_full%d" % e)

        def load_v(jv):
            vs = jv & 1
            yield ("wait", "v_empty%d" % vs, ((jv >> 1) & 1) ^ 1)
            yield ("tma", "v_full%d" % vs, [(("V", vs), jv)], 1)

        yield ("tma", "clc", [(("CLC",), 0)], 1)  # the request for unit 1
        j = 0
        while True:
            yield from publish(j)
            if j == n:
                break
            ks = j % K_SLOTS
            yield ("wait", "kq_empty%d" % ks, ((j // K_SLOTS) & 1) ^ 1)
            yield ("tma", "kq_full%d" % ks, [(("Q", ks), j), (("K", ks), j)], 1)
            if j >= 2:
                yield from load_v(j - 2)
            yield ("wait", "clc", j & 1)
            yield ("read", [(("CLC",), j)])
            if j + 1 < n:
                yield ("tma", "clc", [(("CLC",), j + 1)], 1)
            j += 1
        yield from publish(n + 1)
        for jv in range(max(n - 2, 0), n):
            yield from load_v(jv)
        # the last load of every slot has landed
        for s in range(K_SLOTS):
            last = [x for x in range(n) if x % K_SLOTS == s]
            if last:
                yield ("wait", "kq_full%d" % s, (last[-1] // K_SLOTS) & 1)
        for s in range(V_SLOTS):
            last = [x for x in range(n) if x % V_SLOTS == s]
            if last:
                yield ("wait", "v_full%d" % s, (last[-1] >> 1) & 1)

    def mma():
        i = 0
        while True:
            yield from read_unit(i)
            has = i < n
            if has:
                b, ks = i & 1, i % K_SLOTS
                yield ("wait", "s_free%d" % b, ((i >> 1) & 1) ^ 1)
                yield ("wait", "kq_full%d" % ks, (i // K_SLOTS) & 1)
                yield ("mma", [(("Q", ks), i), (("K", ks), i)],
                       [(("S", b, q), ("S", i)) for q in QUARTERS])
                yield ("commit", "s_full%d" % b)
                yield ("commit", "kq_empty%d" % ks)
            if i >= 1:
                j = i - 1
                b = j & 1
                yield ("wait", "p_full%d" % b, (j >> 1) & 1)
                yield ("wait", "v_full%d" % b, (j >> 1) & 1)
                yield ("wait", "o_empty", (j & 1) ^ 1)
                reads = [(("S", b, q), ("P", j)) for q in QUARTERS] + [(("V", b), j)]
                if short_ring[j]:
                    reads.append((("VZ", b), j))
                yield ("mma", reads, [(("O", q), ("O", j)) for q in QUARTERS])
                yield ("commit", "o_full")
                yield ("commit", "v_empty%d" % b)
                yield ("commit", "s_free%d" % b)
            if not has:
                break
            i += 1

    def softmax(grp, q):
        yield from read_unit(grp)
        i = grp
        while i < n:
            yield from read_unit(i + 2)  # the next unit's position, fetched ahead
            yield ("wait", "s_full%d" % grp, (i >> 1) & 1)
            yield ("read", [(("S", grp, q), ("S", i))])
            yield ("write", [(("S", grp, q), ("P", i))])
            if short_ring[i]:
                yield ("wait", "v_full%d" % grp, (i >> 1) & 1)
                yield ("read", [(("V", grp), i)])
                yield ("write", [(("VZ", grp), i)])
            yield ("wait", "l_free%d" % grp, ((i >> 1) & 1) ^ 1)
            yield ("write", [(("L", grp, q), i)])
            yield ("arrive", "p_full%d" % grp)
            i += 2

    def epilogue(q):
        i = 0
        while True:
            yield from read_unit(i)
            if i == n:
                break
            b = i & 1
            yield ("wait", "o_full", i & 1)
            yield ("wait", "p_full%d" % b, (i >> 1) & 1)
            yield ("read", [(("L", b, q), i)])
            yield ("arrive", "l_free%d" % b)
            yield ("read", [(("O", q), ("O", i))])
            yield ("arrive", "o_empty")
            i += 1

    sim.roles["producer"] = (producer(), None)
    sim.roles["mma"] = (mma(), None)
    for grp in range(2):
        for q in QUARTERS:
            sim.roles["softmax%d.%d" % (grp, q)] = (softmax(grp, q), None)
    for q in QUARTERS:
        sim.roles["epilogue%d" % q] = (epilogue(q), None)


@pytest.mark.parametrize("ring", [16, 4])
def test_protocol_random_schedules(ring):
    """The kernel's ring of 16 entries, and a ring of 4, where the entries'
    release (not the slot rings) is what keeps the producer from overwriting
    an entry that a slow reader has not read."""
    rng = random.Random(11 + ring)
    for i in range(150):
        n = rng.choice([1, 2, 3, rng.randint(4, 40)])
        short = [rng.random() < 0.3 for _ in range(n)]
        s = Sim(5000 + i)
        model_decode_tc(s, n, short, ring)
        s.run()


@pytest.mark.parametrize("mistake", ["s_free parity", "p_full count", "no l_free wait",
                                     "ur_empty count", "o_empty count", "no v_full wait",
                                     "one closing entry"])
def test_protocol_model_catches_mistakes(mistake, monkeypatch):
    """Each mistake, put into the model, fails some schedule. The unit ring's
    release count is tried on a ring of 4 entries: at 16 the slot rings keep
    the producer within a few units of every reader anyway."""
    ring = 4 if mistake == "ur_empty count" else 16
    if mistake.endswith("count"):
        real_bar = Sim.bar
        which = mistake.split()[0]

        def bar(self, name, count):
            # fewer arrivals than writers (readers): the next side goes early
            real_bar(self, name, 1 if name.startswith(which) else count)
        monkeypatch.setattr(Sim, "bar", bar)
    real_step = Sim.step_role

    def step_role(self, name):
        gen, blocked = self.roles[name]
        if blocked is not None:
            b, par = blocked
            if mistake == "s_free parity" and b.startswith("s_free"):
                self.roles[name] = (gen, (b, par ^ 1))
            elif mistake == "no l_free wait" and b.startswith("l_free"):
                self.roles[name] = (gen, None)
            elif (mistake == "no v_full wait" and b.startswith("v_full")
                  and name.startswith("softmax")):
                self.roles[name] = (gen, None)
        return real_step(self, name)
    monkeypatch.setattr(Sim, "step_role", step_role)
    failed = 0
    rng = random.Random(4)
    for i in range(60):
        n = rng.randint(2, 24)
        short = [rng.random() < 0.5 for _ in range(n)]
        s = Sim(i)
        model_decode_tc(s, n, short, ring)
        if mistake == "one closing entry":
            # the producer publishes only one -1 entry: the other warp group
            # waits for an entry that never comes
            gen = s.roles["producer"][0]

            def one_closing(g=gen, n=n):
                for act in g:
                    if act[0] == "wait" and act[1] == "ur_empty%d" % ((n + 1) % ring):
                        # skip publish(n + 1): its wait, write and arrive
                        next(g)
                        next(g)
                        continue
                    yield act
            s.roles["producer"] = (one_closing(), None)
        try:
            s.run(limit=300000)
        except AssertionError:
            failed += 1
    assert failed > 0


def model_split_tc(sim, steps, rescale, zero_v, RING=16, mistake=None):
    """The split-KV kernel (csrc/decode_splitkv_tc_sm100.cuh): units with
    steps[i] steps each (0: a range with no position and no new token), K of
    step n into slot n % 3, V of step n - 2 into slot n % 2, Q per unit into
    slot q % 2, S double-buffered, one O. Units with no step stay out of the
    unit ring (the producer marks their state empty). rescale[n]: step n's
    softmax rescales O (it waits for P V of step n - 1 when the unit has one);
    zero_v[n]: it zeroes V rows of its step first (waits for V). mistake:
    "empty in ring" (the first draft: units with no step go through the ring
    too, and a long run of them fills it while a V load the epilogue waits for
    is still to be issued), "q by unit" (Q slots and parities counted over
    every unit) or "l by unit" (the row-state handoff counted likewise); the
    last two need the first."""
    for s in range(3):
        sim.bar("k_full%d" % s, 1)
        sim.bar("k_empty%d" % s, 1)
    for s in range(2):
        for nm, c in (("q_full", 1), ("q_empty", 1), ("v_full", 1), ("v_empty", 1),
                      ("s_full", 1), ("s_free", 1), ("p_full", 4)):
            sim.bar("%s%d" % (nm, s), c)
    for nm, c in (("o_full", 1), ("o_empty", 4), ("l_full", 4), ("l_free", 4)):
        sim.bar(nm, c)
    for e in range(RING):
        sim.bar("ur_full%d" % e, 1)
        sim.bar("ur_empty%d" % e, 9)
    in_ring = mistake in ("empty in ring", "q by unit", "l by unit")
    units = [i for i in range(len(steps)) if in_ring or steps[i] > 0]  # ring order
    nu = len(units)
    st = [steps[u] for u in units]
    first = [sum(st[:i]) for i in range(nu)]  # global index of each unit's first step
    qidx = []
    q = 0
    for i in range(nu):
        qidx.append(i if mistake == "q by unit" else q)
        q += st[i] > 0

    def read_unit(i, times=1):
        e = i % RING
        yield ("wait", "ur_full%d" % e, (i // RING) & 1)
        yield ("read", [(("UR", e), ("U", i))])
        for _ in range(times):
            yield ("arrive", "ur_empty%d" % e)

    def producer():
        nk = nv = 0
        for i in range(nu + 1):
            e = i % RING
            yield ("wait", "ur_empty%d" % e, ((i // RING) & 1) ^ 1)
            yield ("write", [(("UR", e), ("U", i))])
            yield ("arrive", "ur_full%d" % e)
            if i == nu:
                break
            if st[i] > 0:
                qs = qidx[i] % 2
                yield ("wait", "q_empty%d" % qs, ((qidx[i] // 2) & 1) ^ 1)
                yield ("tma", "q_full%d" % qs, [(("Q", qs), i)], 1)
            for k in range(st[i]):
                ks = nk % 3
                yield ("wait", "k_empty%d" % ks, ((nk // 3) & 1) ^ 1)
                yield ("tma", "k_full%d" % ks, [(("K", ks), nk)], 1)
                nk += 1
                if nk - 2 > nv:
                    vs = nv & 1
                    yield ("wait", "v_empty%d" % vs, ((nv >> 1) & 1) ^ 1)
                    yield ("tma", "v_full%d" % vs, [(("V", vs), nv)], 1)
                    nv += 1
        while nv < nk:
            vs = nv & 1
            yield ("wait", "v_empty%d" % vs, ((nv >> 1) & 1) ^ 1)
            yield ("tma", "v_full%d" % vs, [(("V", vs), nv)], 1)
            nv += 1

    def mma():
        n = 0
        units_o = 0
        prev = None  # (step index, first of its unit, last of its unit, its unit's o index)

        def pv(j, pfirst, plast, po):
            b = j & 1
            yield ("wait", "p_full%d" % b, (j >> 1) & 1)
            yield ("wait", "v_full%d" % b, (j >> 1) & 1)
            if pfirst:
                yield ("wait", "o_empty", (po & 1) ^ 1)
            reads = [(("S", b), ("P", j)), (("V", b), j)]
            if zero_v[j]:
                reads.append((("VZ", b), j))
            if not pfirst:
                reads.append((("O",), ("O", j - 1), "pipe"))
            yield ("mma", reads, [(("O",), ("O", j))])
            yield ("commit", "v_empty%d" % b)
            yield ("commit", "s_free%d" % b)
            if plast:
                yield ("commit", "o_full")

        for i in range(nu + 1):
            yield from read_unit(i)
            if i == nu:
                break
            qi = i if mistake == "q by unit" else units_o
            qs = qi % 2
            if st[i] > 0:
                yield ("wait", "q_full%d" % qs, (qi // 2) & 1)
            for k in range(st[i]):
                b, ks = n & 1, n % 3
                yield ("wait", "s_free%d" % b, ((n >> 1) & 1) ^ 1)
                yield ("wait", "k_full%d" % ks, (n // 3) & 1)
                yield ("mma", [(("Q", qs), i), (("K", ks), n)], [(("S", b), ("S", n))])
                yield ("commit", "s_full%d" % b)
                yield ("commit", "k_empty%d" % ks)
                if k == st[i] - 1:
                    yield ("commit", "q_empty%d" % qs)
                if prev is not None:
                    yield from pv(*prev)
                po = units_o
                if k == 0:
                    units_o += 1
                prev = (n, k == 0, k == st[i] - 1, po)
                n += 1
        if prev is not None:
            yield from pv(*prev)

    def softmax():
        n = 0
        handed = 0
        for i in range(nu + 1):
            yield from read_unit(i, 4)
            if i == nu:
                break
            for k in range(st[i]):
                b = n & 1
                yield ("wait", "s_full%d" % b, (n >> 1) & 1)
                yield ("read", [(("S", b), ("S", n))])
                if rescale[n] and k > 0:
                    pb = (n - 1) & 1
                    yield ("wait", "s_free%d" % pb, ((n - 1) >> 1) & 1)
                    yield ("read", [(("O",), ("O", n - 1))])
                    yield ("write", [(("O",), ("O", n - 1))])
                yield ("write", [(("S", b), ("P", n))])
                if zero_v[n]:
                    yield ("wait", "v_full%d" % b, (n >> 1) & 1)
                    yield ("read", [(("V", b), n)])
                    yield ("write", [(("VZ", b), n)])
                for _ in range(4):
                    yield ("arrive", "p_full%d" % b)
                n += 1
            if st[i] > 0:
                yield ("wait", "l_free", ((i if mistake == "l by unit" else handed) & 1) ^ 1)
                yield ("write", [(("L",), i)])
                for _ in range(4):
                    yield ("arrive", "l_full")
                handed += 1

    def epilogue():
        done = 0
        for i in range(nu + 1):
            yield from read_unit(i, 4)
            if i == nu:
                break
            if st[i] == 0:
                continue
            yield ("wait", "l_full", done & 1)
            yield ("wait", "o_full", done & 1)
            yield ("read", [(("L",), i), (("O",), ("O", first[i] + st[i] - 1))])
            for _ in range(4):
                yield ("arrive", "l_free")
                yield ("arrive", "o_empty")
            done += 1

    sim.roles["producer"] = (producer(), None)
    sim.roles["mma"] = (mma(), None)
    sim.roles["softmax"] = (softmax(), None)
    sim.roles["epilogue"] = (epilogue(), None)


def _split_case(rng):
    nu = rng.randint(1, 12)
    steps = [rng.choice([0, 1, 1, 2, 3, 5, 14]) for _ in range(nu)]
    if rng.random() < 0.4:  # a long run of empty ranges (short sequences)
        at = rng.randint(0, nu)
        steps[at:at] = [0] * rng.randint(16, 40)
    total = sum(steps)
    rescale = [rng.random() < 0.3 for _ in range(total)]
    zero_v = [rng.random() < 0.3 for _ in range(total)]
    return steps, rescale, zero_v


def test_split_protocol_random_schedules():
    rng = random.Random(31)
    for i in range(200):
        steps, rescale, zero_v = _split_case(rng)
        s = Sim(7000 + i)
        model_split_tc(s, steps, rescale, zero_v)
        s.run()


@pytest.mark.parametrize("mistake", ["empty in ring", "q by unit", "l by unit", "p_full count"])
def test_split_protocol_model_catches_mistakes(mistake, monkeypatch):
    """The first draft's empty units in the unit ring (a run of them fills it
    and the producer blocks before the V load the epilogue waits for), its
    counting over every unit (units with no step load no Q and hand over no
    row state) and too few P arrivals fail some schedule."""
    if mistake == "p_full count":
        real_bar = Sim.bar

        def bar(self, name, count):
            real_bar(self, name, 1 if name.startswith("p_full") else count)
        monkeypatch.setattr(Sim, "bar", bar)
    failed = 0
    rng = random.Random(6)
    for i in range(80):
        steps, rescale, zero_v = _split_case(rng)
        if mistake != "p_full count" and 0 not in steps:
            steps[rng.randrange(len(steps))] = 0
        if mistake == "empty in ring" and i % 2 == 0:
            steps = [3] + [0] * 20 + [2]
            rescale, zero_v = [False] * 5, [False] * 5
        s = Sim(300 + i)
        model_split_tc(s, steps, rescale, zero_v, mistake=None if mistake == "p_full count" else mistake)
        try:
            s.run(limit=300000)
        except AssertionError:
            failed += 1
    assert failed > 0
