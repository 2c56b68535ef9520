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
