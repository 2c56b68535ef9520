"""CPU checks of the tcgen05 backward's design (csrc/backward_sm100.cuh):
models of the two kernels' index arithmetic and barrier protocols, written
from the kernels and kept in step with them by hand.

* Coverage: bwd_dq_tc_kernel's enumeration (token tiles of 128/G tokens,
  heaviest first, 64-key chunks from the first key of the tile's first token,
  the per-row mask with its whole-chunk fast path) and bwd_dkdv_tc_kernel's
  (128-key tiles, 64-row blocks of 64/G tokens from k0 to the end of the last
  key's visibility, the per-key row-range mask) each produce every visible
  (token, head, key) pair exactly once, and nothing else: packed sequences
  (some empty), G = 1 .. 64, windows 0 (global), 1, 3, 37, 128, 150.
* Protocol: a discrete-event model of every role of each kernel (producer,
  two MMA issuers, eight elementwise warps, four epilogue warps) with the
  kernels' mbarrier counts and parities; TMA and cp.async writes complete
  asynchronously, tcgen05 MMAs of one thread complete in order and a commit
  arrives once the thread's earlier MMAs have. Under random schedules no role
  deadlocks and every read (MMA operand, TMEM load, shared-memory statistics)
  sees the version it expects over its whole issue-to-completion window. A
  removed wait, a flipped parity and a wrong arrival count each fail it, and
  index mistakes (a chunk too few, a mask or row range off by one, rows ending
  with the tile's first key) each fail the coverage check.
"""
import bisect
import random

import pytest

def seq_of(cu, t):
    return bisect.bisect_right(cu, t) - 1

def first_key(cu, W, t):
    s = seq_of(cu, t)
    lo = cu[s]
    return max(lo, t - W + 1) if W > 0 else lo

def vis_end(cu, W, j):
    s = seq_of(cu, j)
    e = cu[s + 1]
    return min(e, j + W) if W > 0 else e

def brute(cu, Hq, Hkv, W):
    total = cu[-1]
    G = Hq // Hkv
    out = set()
    for t in range(total):
        s = seq_of(cu, t)
        for j in range(cu[s], t + 1):
            if W > 0 and t - j >= W:
                continue
            for hh in range(G):
                for g in range(Hkv):
                    out.add((t, g * G + hh, j))
    return out

def emulate_dq(cu, Hq, Hkv, W):
    total = cu[-1]; G = Hq // Hkv; lg = G.bit_length() - 1
    TM = 128 // G
    n_units = (total + TM - 1) // TM
    seen = []
    for f in range(n_units * Hkv):
        rank, g = divmod(f, Hkv)
        tb = n_units - 1 - rank
        t0 = tb * TM
        t_last = min(t0 + TM, total) - 1
        lo = first_key(cu, W, t0)
        nchunk = (t_last - lo + 64) // 64
        assert nchunk >= 1
        all_lo = first_key(cu, W, t_last); all_hi = t0
        for c in range(nchunk):
            key0 = lo + c * 64
            assert key0 < total  # TMA box start inside (tail zero-filled)
            for r in range(128):
                tok = r >> lg; hh = r - (tok << lg)
                i = t0 + tok
                row_lo, row_hi = (first_key(cu, W, i), i) if i < total else (0, -1)
                for hw in range(2):
                    cb = key0 + 32 * hw
                    fast = cb >= all_lo and cb + 31 <= all_hi
                    for e in range(32):
                        if not fast:
                            cmin = row_lo - cb; cmax = row_hi - cb
                            if e < cmin or e > cmax:
                                continue
                        key = cb + e
                        if i >= total:
                            continue  # row not stored (its dS is computed but unused)
                        seen.append((i, g * G + hh, key))
    return seen

def emulate_dkdv(cu, Hq, Hkv, W):
    total = cu[-1]; G = Hq // Hkv; lg = G.bit_length() - 1
    TOK = 64 // G
    n_units = (total + 127) // 128
    seen = []
    for f in range(n_units * Hkv):
        kt, g = divmod(f, Hkv)
        k0 = kt * 128
        t_hi = vis_end(cu, W, min(k0 + 128, total) - 1)
        nblk = (t_hi - k0 + TOK - 1) // TOK
        assert nblk >= 1
        for n in range(nblk):
            t0 = k0 + n * TOK
            assert t0 < total  # box start inside
            for r in range(128):
                j = k0 + r
                j_end = vis_end(cu, W, j) if j < total else j
                for hw in range(2):
                    cmin = (min(max(j - t0, 0), TOK) << lg) - 32 * hw
                    cmax = (min(max(j_end - t0, 0), TOK) << lg) - 1 - 32 * hw
                    for e in range(32):
                        if (cmin > 0 or cmax < 31) and (e < cmin or e > cmax):
                            continue
                        rr = 32 * hw + e
                        t = t0 + (rr >> lg)
                        hh = rr & (G - 1)
                        # a kept column must be a real, visible pair
                        assert j < total and t < total, (j, t)
                        seen.append((t, g * G + hh, j))
    return seen

def check(cu, Hq, Hkv, W):
    ref = brute(cu, Hq, Hkv, W)
    for name, fn in (("dq", emulate_dq), ("dkdv", emulate_dkdv)):
        got = fn(cu, Hq, Hkv, W)
        assert len(got) == len(set(got)), (name, "duplicate pairs")
        assert set(got) == ref, (name, len(set(got) - ref), len(ref - set(got)))
    return len(ref)


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, self.name
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):  # the phase with this parity has completed
        return (self.phase & 1) != parity


class Sim:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.bars = {}
        self.ver = {}
        self.roles = {}
        self.events = []      # pending async: (kind, payload)
        self.mmaq = {}        # role -> list of queued MMA / commit markers

    def bar(self, name, count):
        self.bars[name] = Bar(name, count)

    def check(self, reads, what, issue=False):
        for res, want, *pipe in reads:
            if issue and pipe:
                continue  # written by this thread's earlier MMA: ordered in the pipe
            got = self.ver.get(res)
            assert got == want, "%s: %s holds %s, wants %s" % (what, res, got, want)

    def step_role(self, name):
        gen, blocked = self.roles[name]
        if blocked is not None:
            b, par = blocked
            if not self.bars[b].done(par):
                return False
        try:
            act = next(gen)
        except StopIteration:
            del self.roles[name]
            return True
        kind = act[0]
        if kind == "wait":
            self.roles[name] = (gen, (act[1], act[2]))
            return True
        self.roles[name] = (gen, None)
        if kind == "arrive":
            self.bars[act[1]].arrive()
        elif kind == "read":
            self.check(act[1], name)
        elif kind == "write":
            for res, v in act[1]:
                self.ver[res] = v
        elif kind in ("tma", "cpasync"):  # (kind, bar, writes, arrivals)
            for res, _ in act[2]:
                self.ver[res] = ("partial",)
            self.events.append(("async", act))
        elif kind == "mma":  # (mma, reads, writes)
            self.check(act[1], name + " mma issue", issue=True)
            q = self.mmaq.setdefault(name, [])
            q.append(act)
            if len(q) == 1:
                self.events.append(("mmaq", name))
        elif kind == "commit":
            q = self.mmaq.setdefault(name, [])
            q.append(act)
            if len(q) == 1:
                self.events.append(("mmaq", name))
        else:
            raise ValueError(kind)
        return True

    def step_event(self, i):
        kind, x = self.events.pop(i)
        if kind == "async":
            _, b, writes, arrivals = x
            for res, v in writes:
                self.ver[res] = v
            for _ in range(arrivals):
                self.bars[b].arrive()
        else:  # head of an MMA queue completes
            q = self.mmaq[x]
            act = q.pop(0)
            if act[0] == "mma":
                self.check(act[1], x + " mma completion")
                for res, v in act[2]:
                    self.ver[res] = v
            else:
                self.bars[act[1]].arrive()
            if q:
                self.events.append(("mmaq", x))

    def run(self, limit=10 ** 7):
        for _ in range(limit):
            if not self.roles and not self.events:
                return
            choices = [("r", n) for n in self.roles] + [("e", i) for i in range(len(self.events))]
            self.rng.shuffle(choices)
            progressed = False
            for c in choices:
                if c[0] == "e":
                    self.step_event(c[1])
                    progressed = True
                    break
                if self.step_role(c[1]):
                    progressed = True
                    break
            if not progressed:
                blocked = {n: b for n, (g, b) in self.roles.items()}
                raise AssertionError("deadlock: %s" % blocked)
        raise AssertionError("step limit")


def model_dq(sim, nchunks, NKV):
    for s in range(2):
        for nm, c in (("q_full", 1), ("q_empty", 5), ("s_full", 1), ("s_empty", 1),
                      ("p_full", 8), ("a_full", 1), ("a_empty", 4), ("dl_full", 4),
                      ("dl_empty", 8)):
            sim.bar("%s%d" % (nm, s), c)
    for s in range(NKV):
        sim.bar("kv_full%d" % s, 1)
        sim.bar("kv_empty%d" % s, 1)

    def producer():
        n = 0
        for k, nc in enumerate(nchunks):
            qs = k & 1
            yield ("wait", "q_empty%d" % qs, ((k >> 1) & 1) ^ 1)
            yield ("tma", "q_full%d" % qs, [(("Q", qs), k)], 1)
            for c in range(nc):
                st = n % NKV
                yield ("wait", "kv_empty%d" % st, ((n // NKV) & 1) ^ 1)
                yield ("tma", "kv_full%d" % st, [(("KV", st), n)], 1)
                n += 1

    def s_issuer():
        n = 0
        for k, nc in enumerate(nchunks):
            qs = k & 1
            yield ("wait", "q_full%d" % qs, (k >> 1) & 1)
            for c in range(nc):
                b, st = n & 1, n % NKV
                yield ("wait", "s_empty%d" % b, ((n >> 1) & 1) ^ 1)
                yield ("wait", "kv_full%d" % st, (n // NKV) & 1)
                yield ("mma", [(("Q", qs), k), (("KV", st), n)],
                       [(("S", b, w), ("S", n)) for w in range(8)])
                yield ("commit", "s_full%d" % b)
                if c == nc - 1:
                    yield ("commit", "q_empty%d" % qs)
                n += 1

    def softmax(w):
        n = 0
        for k, nc in enumerate(nchunks):
            # the tile's Delta (the rows of warp w % 4), from the epilogue warps
            yield ("wait", "dl_full%d" % (k & 1), (k >> 1) & 1)
            yield ("read", [(("DL", k & 1, w % 4), ("D", k))])
            yield ("arrive", "dl_empty%d" % (k & 1))
            for c in range(nc):
                b = n & 1
                yield ("wait", "s_full%d" % b, (n >> 1) & 1)
                yield ("read", [(("S", b, w), ("S", n))])
                yield ("write", [(("S", b, w), ("dS", n))])
                yield ("arrive", "p_full%d" % b)
                n += 1

    def acc_issuer():
        n = 0
        for k, nc in enumerate(nchunks):
            a = k & 1
            for c in range(nc):
                b, st = n & 1, n % NKV
                yield ("wait", "p_full%d" % b, (n >> 1) & 1)
                if c == 0:
                    yield ("wait", "a_empty%d" % a, ((k >> 1) & 1) ^ 1)
                reads = [(("S", b, w), ("dS", n)) for w in range(8)] + [(("KV", st), n)]
                if c > 0:
                    reads.append((("ACC", a), ("A", k, c - 1), "pipe"))
                yield ("mma", reads, [(("ACC", a), ("A", k, c))])
                yield ("commit", "s_empty%d" % b)
                yield ("commit", "kv_empty%d" % st)
                if c == nc - 1:
                    yield ("commit", "a_full%d" % a)
                n += 1

    def epilogue(w):
        def delta(k):  # Delta of tile k's rows (dO from its Q stage) into slot k & 1
            yield ("wait", "q_full%d" % (k & 1), (k >> 1) & 1)
            yield ("wait", "dl_empty%d" % (k & 1), ((k >> 1) & 1) ^ 1)
            yield ("read", [(("Q", k & 1), k)])
            yield ("arrive", "q_empty%d" % (k & 1))
            yield ("write", [(("DL", k & 1, w), ("D", k))])
            yield ("arrive", "dl_full%d" % (k & 1))
        if nchunks:
            yield from delta(0)
        for k, nc in enumerate(nchunks):
            if k + 1 < len(nchunks):
                yield from delta(k + 1)
            a = k & 1
            yield ("wait", "a_full%d" % a, (k >> 1) & 1)
            yield ("read", [(("ACC", a), ("A", k, nc - 1))])
            yield ("arrive", "a_empty%d" % a)

    sim.roles["producer"] = (producer(), None)
    sim.roles["s_issuer"] = (s_issuer(), None)
    sim.roles["acc_issuer"] = (acc_issuer(), None)
    for w in range(8):
        sim.roles["softmax%d" % w] = (softmax(w), None)
    for w in range(4):
        sim.roles["epilogue%d" % w] = (epilogue(w), None)


def model_dkdv(sim, nblks, NS):
    sim.bar("kv_full", 1)
    sim.bar("kv_empty", 1)
    for s in range(NS):
        sim.bar("qd_full%d" % s, 33)
        sim.bar("qd_empty%d" % s, 1)
    for s in range(2):
        sim.bar("s_full%d" % s, 1)
        sim.bar("s_empty%d" % s, 1)
        sim.bar("p_full%d" % s, 8)
    sim.bar("a_full", 1)
    sim.bar("a_empty", 4)

    def producer():
        m = 0
        for k, nb in enumerate(nblks):
            yield ("wait", "kv_empty", (k & 1) ^ 1)
            yield ("tma", "kv_full", [(("KV",), k)], 1)
            for n in range(nb):
                st = m % NS
                yield ("wait", "qd_empty%d" % st, ((m // NS) & 1) ^ 1)
                yield ("tma", "qd_full%d" % st, [(("QD", st), m)], 1)
                yield ("cpasync", "qd_full%d" % st, [(("LS", st), m)], 32)
                m += 1

    def s_issuer():
        m = 0
        for k, nb in enumerate(nblks):
            yield ("wait", "kv_full", k & 1)
            for n in range(nb):
                b, st = m & 1, m % NS
                yield ("wait", "s_empty%d" % b, ((m >> 1) & 1) ^ 1)
                yield ("wait", "qd_full%d" % st, (m // NS) & 1)
                yield ("mma", [(("KV",), k), (("QD", st), m)],
                       [(("S", b, w), ("S", m)) for w in range(8)])
                yield ("commit", "s_full%d" % b)
                if n == nb - 1:
                    yield ("commit", "kv_empty")
                m += 1

    def softmax(w):
        m = 0
        for k, nb in enumerate(nblks):
            for n in range(nb):
                b, st = m & 1, m % NS
                yield ("wait", "s_full%d" % b, (m >> 1) & 1)
                yield ("wait", "qd_full%d" % st, (m // NS) & 1)
                yield ("read", [(("S", b, w), ("S", m)), (("LS", st), m)])
                yield ("write", [(("S", b, w), ("P", m))])
                yield ("arrive", "p_full%d" % b)
                m += 1

    def acc_issuer():
        m = 0
        for k, nb in enumerate(nblks):
            for n in range(nb):
                b, st = m & 1, m % NS
                yield ("wait", "p_full%d" % b, (m >> 1) & 1)
                if n == 0:
                    yield ("wait", "a_empty", (k & 1) ^ 1)
                reads = [(("S", b, w), ("P", m)) for w in range(8)] + [(("QD", st), m)]
                if n > 0:
                    reads.append((("ACC",), ("A", k, n - 1), "pipe"))
                yield ("mma", reads, [(("ACC",), ("A", k, n))])
                yield ("commit", "qd_empty%d" % st)
                yield ("commit", "s_empty%d" % b)
                if n == nb - 1:
                    yield ("commit", "a_full")
                m += 1

    def epilogue(w):
        for k, nb in enumerate(nblks):
            yield ("wait", "a_full", k & 1)
            yield ("read", [(("ACC",), ("A", k, nb - 1))])
            yield ("arrive", "a_empty")

    sim.roles["producer"] = (producer(), None)
    sim.roles["s_issuer"] = (s_issuer(), None)
    sim.roles["acc_issuer"] = (acc_issuer(), None)
    for w in range(8):
        sim.roles["softmax%d" % w] = (softmax(w), None)
    for w in range(4):
        sim.roles["epilogue%d" % w] = (epilogue(w), None)


COVER_CASES = [([0, 300], 8, 1, 128), ([0, 140], 64, 8, 128), ([0, 257, 260, 420], 16, 2, 128),
               ([0, 130, 131, 400], 4, 4, 0), ([0, 1], 8, 1, 3), ([0, 70, 71, 72, 160], 64, 1, 37),
               ([0, 129, 200], 32, 1, 0), ([0, 64, 64, 320], 8, 8, 150), ([0, 513], 2, 1, 1)]


@pytest.mark.parametrize("cu,Hq,Hkv,W", COVER_CASES)
def test_tiles_cover_every_visible_pair_once(cu, Hq, Hkv, W):
    check(cu, Hq, Hkv, W)


@pytest.mark.parametrize("kernel", ["dq", "dkdv"])
def test_protocol_random_schedules(kernel):
    rng = random.Random(7 if kernel == "dq" else 8)
    for i in range(120):
        tiles = [rng.randint(1, 6) for _ in range(rng.randint(1, 7))]
        s = Sim(1000 * (kernel == "dkdv") + i)
        if kernel == "dq":
            model_dq(s, tiles, rng.choice([2, 3, 4]))
        else:
            model_dkdv(s, tiles, rng.choice([2, 3, 4]))
        s.run()


@pytest.mark.parametrize("mistake", ["no a_empty wait", "s_empty parity", "qd_full count",
                                     "dl_full parity", "dl_full count", "q_empty count"])
def test_protocol_model_catches_mistakes(mistake, monkeypatch):
    """Each mistake, put into the model, fails some schedule."""
    if mistake in ("qd_full count", "dl_full count", "q_empty count"):
        real_bar = Sim.bar
        which = mistake.split()[0]

        def bar(self, name, count):
            # fewer arrivals than writers (readers): the next side goes early
            real_bar(self, name, (1 if which == "q_empty" else 2) if name.startswith(which)
                     else count)
        monkeypatch.setattr(Sim, "bar", bar)
    real_step = Sim.step_role

    def step_role(self, name):
        gen, blocked = self.roles[name]
        if blocked is not None:
            b, par = blocked
            if mistake == "no a_empty wait" and b == "a_empty":
                self.roles[name] = (gen, None)  # the wait is skipped
            elif mistake == "s_empty parity" and b.startswith("s_empty"):
                self.roles[name] = (gen, (b, par ^ 1))
            elif mistake == "dl_full parity" and b.startswith("dl_full"):
                self.roles[name] = (gen, (b, par ^ 1))
        return real_step(self, name)
    monkeypatch.setattr(Sim, "step_role", step_role)
    failed = 0
    rng = random.Random(3)
    for i in range(60):
        tiles = [rng.randint(1, 6) for _ in range(rng.randint(2, 7))]
        s = Sim(i)
        if mistake in ("no a_empty wait", "qd_full count"):
            model_dkdv(s, tiles, 3)
        else:
            model_dq(s, tiles, 3)
        try:
            s.run(limit=200000)
        except AssertionError:
            failed += 1
    assert failed > 0


COVER_MISTAKES = {
    "dq: one chunk too few": ("nchunk = (t_last - lo + 64) // 64", "nchunk = (t_last - lo + 1) // 64"),
    "dq: mask off by one": ("cmin = row_lo - cb; cmax = row_hi - cb",
                            "cmin = row_lo - cb; cmax = row_hi - cb - 1"),
    "dkdv: rows end with the first key's": ("t_hi = vis_end(cu, W, min(k0 + 128, total) - 1)",
                                            "t_hi = vis_end(cu, W, k0)"),
    "dkdv: row range off by one": ("cmax = (min(max(j_end - t0, 0), TOK) << lg) - 1 - 32 * hw",
                                   "cmax = (min(max(j_end - t0, 0), TOK) << lg) - 2 - 32 * hw"),
}


@pytest.mark.parametrize("mistake", sorted(COVER_MISTAKES))
def test_coverage_model_catches_mistakes(mistake):
    """Each index mistake, put into a copy of the coverage model, fails it on
    some of the shapes above."""
    import inspect
    old, new = COVER_MISTAKES[mistake]
    src = "\n".join(inspect.getsource(f) for f in (emulate_dq, emulate_dkdv, check))
    assert src.count(old) == 1, old
    ns = dict(seq_of=seq_of, first_key=first_key, vis_end=vis_end, brute=brute)
    exec(src.replace(old, new), ns)
    failed = False
    for cu, Hq, Hkv, W in COVER_CASES[:6]:
        try:
            ns["check"](cu, Hq, Hkv, W)
        except AssertionError:
            failed = True
            break
    assert failed
