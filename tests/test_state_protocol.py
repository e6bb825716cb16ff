"""Randomised check of the state passes' hand-over protocols (CPU only).

`state_bwd_tc_kernel` (csrc/sf_tc_state.cu) runs one CTA per head over the chunks in
reverse: a chain thread issues dS'^T K^T, dO^T (diag(gamma) Q) and - dDelta^T W; a copy
thread issues the loads into a two-stage ring, the stores of dS'^T and dDelta^T, and
dO^T P of the next chunk; sixteen element-wise warps write the TMEM operands, scale Q in
place, stage the stores and carry dS^T.  This test replays that protocol as a model
(NW element-wise agents standing for the warps; TMA loads, an in-order UMMA pipe whose
commits arrive once every earlier product of the committing thread is done, stores that
read their tile after a delay) over random interleavings.  It asserts that no parity
wait sees a phase two ahead of the one it means, that every read sees the current
chunk's data, and that no tile or TMEM region is overwritten while it is still read;
each guard, removed, must make some schedule fail.  `state_fwd_tc_kernel` (the forward
pass: X^T = S^T W^T and P^T = (scaled Delta)^T K on the chain, a three-stage ring, the
stores of S^T and Delta^T) is checked the same way.
"""
import random

import pytest

NW = 3


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arr, self.done = name, count, 0, 0

    def arrive(self):
        self.arr += 1
        assert self.arr <= self.count, f"{self.name}: too many arrivals"
        if self.arr == self.count:
            self.arr = 0
            self.done += 1


def run_model(NC, seed, drop=None, store_delay=60):
    rnd = random.Random(seed)
    B = {n: _Bar(n, c) for n, c in [
        ("ld0", 1), ("ld1", 1), ("y", 1), ("y2", 1), ("z", 1), ("sfree", 1), ("dfree", 1),
        ("s", NW), ("q", NW), ("d", NW), ("sst", NW), ("dst", NW)]}
    pending, now = [], [0]

    def later(fn, lo, hi):
        pending.append((now[0] + rnd.randint(lo, hi), fn))

    def phase(bar, k):
        b = B[bar]
        assert b.done <= k + 1, f"{bar} ran ahead: {b.done} phases done, wait for phase {k}"
        return b.done > k

    content, readers = {}, {}

    def read(reg, tag, who):
        assert content.get(reg) == tag, f"{who}: {reg} holds {content.get(reg)}, wants {tag}"

    def write(reg, tag, who):
        assert readers.get(reg, 0) == 0, f"{who}: {reg} overwritten while read asynchronously"
        content[reg] = tag

    # one UMMA pipe, in order; each commit covers its own thread's earlier products
    pipe, busy = [], [False]

    def mma(reads, writes, tag):
        for r, t in reads:
            read(r, t, "UMMA issue")
            readers[r] = readers.get(r, 0) + 1
        pipe.append(("mma", reads, writes, tag))

    def commit(bar):
        pipe.append(("commit", bar))

    def pump():
        if busy[0] or not pipe:
            return
        busy[0] = True
        op = pipe.pop(0)

        def done():
            busy[0] = False
            if op[0] == "commit":
                B[op[1]].arrive()
            else:
                _, reads, writes, tag = op
                for r, t in reads:
                    read(r, t, "UMMA")
                    readers[r] -= 1
                for w in writes:
                    content[w] = tag
            pump()
        later(done, 5, 30)

    stores = []

    def store(reg, tag):
        read(reg, tag, "store issue")
        readers[reg] = readers.get(reg, 0) + 1
        st = {"read": False}
        stores.append(st)

        def fin():
            read(reg, tag, "store")
            readers[reg] -= 1
            st["read"] = True
        later(fin, 5, store_delay)

    def load(n):
        s = n % 2
        tiles = [f"{t}{s}" for t in ("K", "dO", "Q", "W", "P", "E")]
        for t in tiles:
            assert readers.get(t, 0) == 0, f"load of chunk {n}: {t} still read asynchronously"
            assert content.get(t) in (None, n - 2, ("scaled", n - 2)), f"load of chunk {n} over {content.get(t)}"
            assert all(done >= n - 2 for done in warps_done.values()) or n < 2, \
                f"load of chunk {n}: a warp still works on chunk {n - 2}"
            content[t] = ("landing", n)

        def land():
            for t in tiles:
                content[t] = n
            B[f"ld{s}"].arrive()
        later(land, 10, 120)

    def chain():
        for n in range(NC):
            s = n % 2
            yield lambda: phase("s", n)
            yield lambda: phase(f"ld{s}", n // 2)
            mma([("tS", n), (f"K{s}", n)], ["tY1"], n)
            commit("y")
            yield lambda: phase("q", n)
            mma([(f"dO{s}", n), (f"Q{s}", ("scaled", n))], ["tZ"], n)
            if drop != "chain_d":
                yield lambda: phase("d", n)
            mma([("tD", n), (f"W{s}", n)], ["tZ"], n)
            commit("z")

    def copy():
        issued = 0
        for _ in range(min(2, NC)):
            load(issued)
            issued += 1

        def y2(n):
            s = n % 2
            yield lambda: phase(f"ld{s}", n // 2)
            mma([(f"dO{s}", n), (f"P{s}", n)], ["tY2"], n)
            commit("y2")
        yield from y2(0)
        for n in range(NC):
            yield lambda: phase("s", n)
            if n >= 1 and issued < NC:
                load(issued)
                issued += 1
            yield lambda: phase("sst", n)
            store("St", n)
            snap = list(stores[:-1])
            yield lambda: all(st["read"] for st in snap)
            if n > 0:
                B["dfree"].arrive()
            if drop != "copy_d":
                yield lambda: phase("d", n)
            if n + 1 < NC:
                yield from y2(n + 1)
            yield lambda: phase("dst", n)
            store("Dst", n)
            snap2 = list(stores[:-1])
            if drop != "sfree_read":
                yield lambda: all(st["read"] for st in snap2)
            B["sfree"].arrive()
        snap3 = list(stores)
        yield lambda: all(st["read"] for st in snap3)

    warps_done = {}

    def warps(ag):
        for n in range(NC):
            s = n % 2
            write("tS", n, f"agent {ag} dS'^T")
            B["s"].arrive()
            if drop != "ld":
                yield lambda: phase(f"ld{s}", n // 2)
            read(f"E{s}", n, f"agent {ag}")
            assert content.get(f"Q{s}") in (n, ("scaled", n)), f"agent {ag}: Q of chunk {n} not in place"
            write(f"Q{s}", ("scaled", n), f"agent {ag} scaling Q")
            B["q"].arrive()
            if n > 0 and drop != "sfree":
                yield lambda: phase("sfree", n - 1)
            write("St", n, f"agent {ag} staging dS'^T")
            B["sst"].arrive()
            yield lambda: phase("y", n)
            if drop != "y2":
                yield lambda: phase("y2", n)
            read("tY1", n, f"agent {ag}")
            read("tY2", n, f"agent {ag}")
            write("tD", n, f"agent {ag} dDelta^T")
            B["d"].arrive()
            if n > 0 and drop != "dfree":
                yield lambda: phase("dfree", n - 1)
            write("Dst", n, f"agent {ag} staging dDelta^T")
            B["dst"].arrive()
            yield lambda: phase("z", n)
            read("tZ", n, f"agent {ag}")
            read(f"E{s}", n, f"agent {ag}")
            warps_done[ag] = n

    threads = {"chain": chain(), "copy": copy(), **{f"warps{i}": warps(i) for i in range(NW)}}
    for i in range(NW):
        warps_done[i] = -1
    waiting = {}
    for k, th in threads.items():
        try:
            waiting[k] = next(th)
        except StopIteration:
            waiting[k] = None
    for _ in range(200000):
        live = [k for k in threads if waiting[k] is not None]
        if not live and not pending and not pipe and not busy[0]:
            return
        rnd.shuffle(live)
        moved = False
        for k in live:
            if waiting[k]():
                try:
                    waiting[k] = next(threads[k])
                except StopIteration:
                    waiting[k] = None
                moved = True
                break
        if not moved or (pending and rnd.random() < 0.3):
            assert pending, "deadlock: " + ", ".join(live)
            pending.sort(key=lambda x: x[0])
            t, fn = pending.pop(0)
            now[0] = max(now[0], t)
            fn()
        pump()
    raise AssertionError("schedule did not finish")


def run_model_fwd(NC, seed, drop=None, store_delay=60):
    rnd = random.Random(seed)
    B = {n: _Bar(n, c) for n, c in [
        ("ld0", 1), ("ld1", 1), ("ld2", 1), ("x", 1), ("p", 1), ("sfree", 1), ("dfree", 1),
        ("s", NW), ("d", NW), ("sst", NW), ("dst", NW)]}
    pending, now = [], [0]

    def later(fn, lo, hi):
        pending.append((now[0] + rnd.randint(lo, hi), fn))

    def phase(bar, k):
        b = B[bar]
        assert b.done <= k + 1, f"{bar} ran ahead: {b.done} phases done, wait for phase {k}"
        return b.done > k

    content, readers = {}, {}

    def read(reg, tag, who):
        assert content.get(reg) == tag, f"{who}: {reg} holds {content.get(reg)}, wants {tag}"

    def write(reg, tag, who):
        assert readers.get(reg, 0) == 0, f"{who}: {reg} overwritten while read asynchronously"
        content[reg] = tag

    pipe, busy = [], [False]

    def mma(reads, writes, tag):
        for r, t in reads:
            read(r, t, "UMMA issue")
            readers[r] = readers.get(r, 0) + 1
        pipe.append(("mma", reads, writes, tag))

    def commit(bar):
        pipe.append(("commit", bar))

    def pump():
        if busy[0] or not pipe:
            return
        busy[0] = True
        op = pipe.pop(0)

        def done():
            busy[0] = False
            if op[0] == "commit":
                B[op[1]].arrive()
            else:
                _, reads, writes, tag = op
                for r, t in reads:
                    read(r, t, "UMMA")
                    readers[r] -= 1
                for w in writes:
                    content[w] = tag
            pump()
        later(done, 5, 30)

    stores = []

    def store(reg, tag):
        read(reg, tag, "store issue")
        readers[reg] = readers.get(reg, 0) + 1
        st = {"read": False}
        stores.append(st)

        def fin():
            read(reg, tag, "store")
            readers[reg] -= 1
            st["read"] = True
        later(fin, 5, store_delay)

    warps_done = {i: -1 for i in range(NW)}

    def load(c):
        s = c % 3
        tiles = [f"{t}{s}" for t in ("W", "K", "U", "E")]
        for t in tiles:
            assert readers.get(t, 0) == 0, f"load of chunk {c}: {t} still read asynchronously"
            assert content.get(t) in (None, c - 3), f"load of chunk {c} over {content.get(t)}"
            assert c < 3 or all(done >= c - 3 for done in warps_done.values()), \
                f"load of chunk {c}: a warp still works on chunk {c - 3}"
            content[t] = ("landing", c)

        def land():
            for t in tiles:
                content[t] = c
            B[f"ld{s}"].arrive()
        later(land, 10, 120)

    def chain():
        for c in range(NC):
            s = c % 3
            yield lambda: phase(f"ld{s}", c // 3)
            yield lambda: phase("s", c)
            mma([("tS", c), (f"W{s}", c)], ["tX"], c)
            commit("x")
            if drop != "chain_d":
                yield lambda: phase("d", c)
            mma([("tD", c), (f"K{s}", c)], ["tP"], c)
            commit("p")

    def copy():
        issued = 0
        for _ in range(min(3, NC)):
            load(issued)
            issued += 1
        for c in range(NC):
            if drop != "copy_s":
                yield lambda: phase("s", c)
            if c >= 1 and issued < NC:
                load(issued)
                issued += 1
            yield lambda: phase("sst", c)
            store("St", c)
            snap = list(stores[:-1])
            yield lambda: all(st["read"] for st in snap)
            if c > 0:
                B["dfree"].arrive()
            yield lambda: phase("dst", c)
            store("Dst", c)
            snap2 = list(stores[:-1])
            if drop != "sfree_read":
                yield lambda: all(st["read"] for st in snap2)
            B["sfree"].arrive()
        snap3 = list(stores)
        yield lambda: all(st["read"] for st in snap3)

    def warps(ag):
        for c in range(NC):
            s = c % 3
            write("tS", c, f"agent {ag} S^T")
            B["s"].arrive()
            if c > 0 and drop != "sfree":
                yield lambda: phase("sfree", c - 1)
            write("St", c, f"agent {ag} staging S^T")
            B["sst"].arrive()
            if drop != "ld":
                yield lambda: phase(f"ld{s}", c // 3)
            if drop != "x":
                yield lambda: phase("x", c)
            read("tX", c, f"agent {ag}")
            read(f"U{s}", c, f"agent {ag}")
            read(f"E{s}", c, f"agent {ag}")
            write("tD", c, f"agent {ag} Delta^T")
            B["d"].arrive()
            if c > 0 and drop != "dfree":
                yield lambda: phase("dfree", c - 1)
            write("Dst", c, f"agent {ag} staging Delta^T")
            B["dst"].arrive()
            yield lambda: phase("p", c)
            read("tP", c, f"agent {ag}")
            read(f"E{s}", c, f"agent {ag}")
            warps_done[ag] = c

    threads = {"chain": chain(), "copy": copy(), **{f"warps{i}": warps(i) for i in range(NW)}}
    waiting = {}
    for k, th in threads.items():
        try:
            waiting[k] = next(th)
        except StopIteration:
            waiting[k] = None
    for _ in range(200000):
        live = [k for k in threads if waiting[k] is not None]
        if not live and not pending and not pipe and not busy[0]:
            return
        rnd.shuffle(live)
        moved = False
        for k in live:
            if waiting[k]():
                try:
                    waiting[k] = next(threads[k])
                except StopIteration:
                    waiting[k] = None
                moved = True
                break
        if not moved or (pending and rnd.random() < 0.3):
            assert pending, "deadlock: " + ", ".join(live)
            pending.sort(key=lambda x: x[0])
            t, fn = pending.pop(0)
            now[0] = max(now[0], t)
            fn()
        pump()
    raise AssertionError("schedule did not finish")


def _failures(drop, schedules, store_delay=60, model=run_model):
    n = 0
    for seed in range(schedules):
        for NC in (1, 2, 3, 4, 7):
            try:
                model(NC, seed * 11 + NC, drop, store_delay)
            except AssertionError:
                n += 1
    return n


def test_protocol_holds_on_random_schedules():
    assert _failures(None, 300) == 0
    assert _failures(None, 100, store_delay=600) == 0


@pytest.mark.parametrize("drop", ["chain_d", "sfree", "dfree", "y2", "ld", "sfree_read"])
def test_each_guard_is_needed(drop):
    assert _failures(drop, 300, store_delay=600) > 0


def test_forward_protocol_holds_on_random_schedules():
    assert _failures(None, 300, model=run_model_fwd) == 0
    assert _failures(None, 100, store_delay=600, model=run_model_fwd) == 0


# (the element-wise warps' own wait on the stage's copies is implied in this model by the
# wait for X^T, whose product waited on them; the kernel keeps it so that those warps
# observe the copies' completion themselves)
@pytest.mark.parametrize("drop", ["chain_d", "sfree", "dfree", "x", "sfree_read", "copy_s"])
def test_each_forward_guard_is_needed(drop):
    assert _failures(drop, 300, store_delay=600, model=run_model_fwd) > 0
