"""Randomised check of the fused gradient kernel's hand-over protocol (CPU only).

`grad_fused_tc_kernel` (csrc/sf_tc_grad_fused.cu) overlaps the chunk-heads ("items") a
CTA takes: the issuing thread loads item j+1's tiles and issues its first product while
the element-wise warps finish item j.  What keeps that correct is a set of mbarrier
hand-overs, each completing one phase per item, and two named barriers.  This test
replays the protocol as a small model:

- an issuer thread and NW element-wise agents (stand-ins for the 16 warps: the
  hand-over barriers count NW arrivals; agents in EPI stand for warps 0-3, which read
  the per-row sums in the epilogue);
- asynchronous engines: TMA loads that land after a random delay, an in-order UMMA
  pipe whose commits arrive once every earlier product is done, TMA stores that read
  their tile after a delay;
- random interleavings of all of them.

It asserts that no wait sees a phase two ahead of the one it means (parity waits
alias then), that every read sees the current item's data, and that no tile or TMEM
region is overwritten while an asynchronous reader is pending or before every agent
has done its last read of the previous item.  Each guard the kernel has, removed
from the model, must make some schedule fail.
"""
import random

import pytest

NW = 3
EPI = {0, 1}


class _Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arr, self.done = name, count, 0, 0

    def arrive(self):
        self.arr += 1
        assert self.arr <= self.count, f"{self.name}: too many arrivals"
        if self.arr == self.count:
            self.arr = 0
            self.done += 1


def run_model(n_items, seed, drop=None, store_delay=60):
    """One random schedule of `n_items` items; `drop` removes one guard."""
    rnd = random.Random(seed)
    B = {n: _Bar(n, c) for n, c in [
        ("ld0", 1), ("ld1", 1), ("ld2", 1), ("ld3", 1), ("ld4", 1),
        ("a0", 1), ("a1", 1), ("a2", 1), ("a3", 1), ("c0", 1), ("c1", 1), ("c2", 1),
        ("s_c", NW), ("s_ab", NW), ("s_d", NW), ("s_q", NW), ("dk", NW), ("pdfree", 1), ("pub", 1)]}
    pending = []
    now = [0]

    def later(fn, lo, hi):
        pending.append((now[0] + rnd.randint(lo, hi), fn))

    def phase(bar, j):  # a wait for phase j (parity j & 1) of `bar`
        b = B[bar]
        assert b.done <= j + 1, f"{bar} ran ahead: {b.done} phases done, wait for phase {j}"
        return b.done > j

    content, async_readers, last_reads = {}, {}, {}

    def read_done_by_all(reg, item):
        if item < 0:
            return
        done = last_reads.get((reg, item), set())
        assert len(done) == NW, f"{reg} overwritten before every agent's last read of item {item}"

    def last_read(reg, item, ag):
        assert content.get(reg) == item, f"agent {ag}: {reg} holds {content.get(reg)}, wants {item}"
        last_reads.setdefault((reg, item), set()).add(ag)

    def read(reg, item, who):
        assert content.get(reg) == item, f"{who}: {reg} holds {content.get(reg)}, wants {item}"

    # ---- asynchronous engines
    pipe, busy = [], [False]

    def mma(reads, writes, j, acc=False):
        for t in reads:
            read(t, j, "UMMA issue")
            async_readers[t] = async_readers.get(t, 0) + 1
        pipe.append((reads, writes, j, acc))

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
                reads, writes, j, acc = op
                for t in reads:
                    read(t, j, "UMMA")
                    async_readers[t] -= 1
                for t in writes:
                    if acc:
                        assert content.get(t) == j, f"UMMA accumulates onto {t} = {content.get(t)}, item {j}"
                    content[t] = j
            pump()
        later(done, 5, 30)

    stores = []

    def store(reg, tag):
        read(reg, tag, "store issue")
        async_readers[reg] = async_readers.get(reg, 0) + 1
        st = {"read": False}
        stores.append(st)

        def fin():
            read(reg, tag, "store")
            async_readers[reg] -= 1
            st["read"] = True
        later(fin, 5, store_delay)

    def load(g, j):
        tiles = {0: ["dDt", "T"], 1: ["dO", "Dt", "St"], 2: ["Q", f"K{j & 1}", f"G{j & 1}"], 3: ["dSt"],
                 4: ["dVs"]}[g]
        for t in tiles:
            assert async_readers.get(t, 0) == 0, f"load {g} of item {j}: {t} still read asynchronously"
            if t == "dVs":
                assert content.get(t) in (None, ("dv", j - 1)), f"V of item {j} over {content.get(t)}"
            elif t.startswith("K"):
                assert content.get(t) in (None, ("dk", j - 2)), f"K of item {j} over {content.get(t)}"
                read_done_by_all(t, j - 2)
            elif t.startswith("G"):
                read_done_by_all(t, j - 2)
            elif t in ("St", "Q", "dSt"):
                read_done_by_all(t, j - 1)
            content[t] = ("landing", j)

        def land():
            for t in tiles:
                content[t] = j
            B[f"ld{g}"].arrive()
        later(land, 10, 120)

    slot = [0, None]
    slot_reads = {0: set(range(NW))}

    def issuer():
        for g in range(5):
            load(g, 0)

        def dvhat_product(j):  # T^T dDelta into lo [256, 384)
            yield lambda: phase("ld0", j)
            read_done_by_all("lo256", j - 1)
            mma(["T", "dDt"], ["lo256"], j)
            commit("a0")
        yield from dvhat_product(0)
        for j in range(n_items):
            has_next = j + 1 < n_items
            old = slot[(j + 1) & 1]
            if old is not None and old >= 0:
                assert len(slot_reads.get(old, set())) == NW, f"slot of item {old} overwritten before read"
            slot[(j + 1) & 1] = j + 1 if has_next else -1
            B["pub"].arrive()
            if j > 0:
                snap = list(stores)
                yield lambda: all(st["read"] for st in snap)
                B["pdfree"].arrive()
            yield lambda: phase("ld1", j)
            read_done_by_all("lo64", j - 1)
            read_done_by_all("lo128", j - 1)
            mma(["dO", "Dt", "St"], ["lo64", "lo128"], j)
            commit("a1")
            yield lambda: phase("ld2", j)
            read_done_by_all("lo0", j - 1)
            mma(["Q", f"K{j & 1}"], ["lo0"], j)
            commit("a2")
            if j > 0:
                if drop != "dk":
                    yield lambda: phase("dk", j - 1)
                store(f"K{(j - 1) & 1}", ("dk", j - 1))
            yield lambda: phase("ld3", j)
            read_done_by_all("hi128", j - 1)
            mma(["Dt", "dSt"], ["hi128"], j)
            commit("a3")
            read_done_by_all("lo384", j - 1)
            mma([f"K{j & 1}"], ["lo384"], j)  # K K^T, under the commit c0
            yield lambda: phase("s_c", j)
            store("dVs", ("dv", j))
            read_done_by_all("hi256", j - 1)
            mma(["dDt", "Dt", "St"], ["hi256"], j)
            commit("c0")
            yield lambda: phase("s_ab", j)
            mma(["F", f"K{j & 1}", "Q"], ["lo128", "hi128"], j, acc=True)
            commit("c1")
            if has_next:
                if drop != "c1":
                    yield lambda: phase("c1", j)
                snap = list(stores)
                if drop != "store_read":
                    yield lambda: all(st["read"] for st in snap)
                for g in (0, 4, 1, 2):
                    load(g, j + 1)
            yield lambda: phase("s_d", j)
            mma(["EE", f"K{j & 1}"], ["hi256"], j, acc=True)
            commit("c2")
            if has_next:
                load(3, j + 1)
            yield lambda: phase("s_q", j)
            store("PD", ("dq", j))
            if has_next:
                yield from dvhat_product(j + 1)
        yield lambda: phase("dk", n_items - 1)
        store(f"K{(n_items - 1) & 1}", ("dk", n_items - 1))
        snap = list(stores)
        yield lambda: all(st["read"] for st in snap)

    sync1 = {"gen": 0, "arr": 0}
    sync4 = {"gen": 0, "arr": 0}
    bar2 = {"phases": 0, "arr": 0}
    epilogue_read = {}

    def barrier(b, n):
        g = b["gen"]
        b["arr"] += 1
        if b["arr"] == n:
            b["arr"] = 0
            b["gen"] += 1
        yield lambda: b["gen"] > g

    def warps(ag):
        for j in range(n_items):
            # (c) dVhat: dv over V in the dv staging tile, dVhat in bf16 over dDelta^T
            yield lambda: phase("a0", j)
            if drop != "ld4":
                yield lambda: phase("ld4", j)
            last_read("lo256", j, ag)
            if j > 0 and ag not in EPI:
                last_reads.setdefault((f"G{(j - 1) & 1}", j - 1), set()).add(ag)
            assert content.get("dVs") in (j, ("dv", j)), f"agent {ag}: V of item {j} not in place"
            assert async_readers.get("dVs", 0) == 0, "dv staged while a store reads the tile"
            content["dVs"] = ("dv", j)
            assert async_readers.get("dDt", 0) == 0, "dVhat written over dDelta^T while read"
            content["dDt"] = j
            B["s_c"].arrive()
            yield lambda: phase("pub", j)
            nx = slot[(j + 1) & 1]
            assert nx == (j + 1 if j + 1 < n_items else -1), f"agent {ag} reads item {nx} as the next"
            if nx >= 0:
                slot_reads.setdefault(nx, set()).add(ag)
            if j > 0 and ag in EPI:  # the last item's epilogue
                read(f"G{(j - 1) & 1}", j - 1, "epilogue")
                epilogue_read.setdefault(j - 1, set()).add(ag)
                last_reads.setdefault((f"G{(j - 1) & 1}", j - 1), set()).add(ag)
                if drop != "bar4":
                    yield from barrier(sync4, len(EPI))
                bar2["arr"] += 1
                if bar2["arr"] == len(EPI):
                    bar2["arr"] = 0
                    bar2["phases"] += 1
            # (a) P, dP, F; the per-row sums are written again from here on
            yield lambda: phase("ld2", j)
            yield lambda: phase("a2", j)
            if j > 0:
                yield lambda: phase("pdfree", j - 1)
                if ag not in EPI and drop != "bar2":
                    yield lambda: bar2["phases"] >= j
                assert epilogue_read.get(j - 1) == EPI, f"agent {ag}: sums of item {j} over unread ones"
            last_read("lo0", j, ag)
            last_read("lo64", j, ag)
            read(f"G{j & 1}", j, "warps")
            assert async_readers.get("F", 0) == 0, "F written while read"
            content["F"] = j
            assert async_readers.get("PD", 0) == 0, "PD written while the dq store reads it"
            # (b) rescaled dO S^T and Delta dS'^T, <S, dS'>
            yield lambda: phase("ld1", j)
            yield lambda: phase("ld3", j)
            yield lambda: phase("a3", j)
            read("lo128", j, "warps")
            read("hi128", j, "warps")
            last_read("Q", j, ag)
            read(f"K{j & 1}", j, "warps")
            last_read("St", j, ag)
            read("dSt", j, "warps")
            B["s_ab"].arrive()
            # (d) B, dA, E over dS'^T, dKhat; E + E^T
            yield lambda: phase("c0", j)
            yield from barrier(sync1, NW)
            read("hi256", j, "warps")
            last_read("lo384", j, ag)
            assert async_readers.get("dSt", 0) == 0, "E written over dS'^T while read"
            last_read("dSt", j, ag)
            yield from barrier(sync1, NW)
            assert async_readers.get("EE", 0) == 0, "E + E^T written while read"
            content["EE"] = j
            B["s_d"].arrive()
            # dq into the PD region
            yield lambda: phase("c1", j)
            last_read("lo128", j, ag)
            last_read(f"K{j & 1}", j, ag)
            yield from barrier(sync1, NW)
            content["PD"] = ("dq", j)
            B["s_q"].arrive()
            # dk into this item's K tile
            yield lambda: phase("c2", j)
            last_read("hi128", j, ag)
            last_read("hi256", j, ag)
            assert async_readers.get(f"K{j & 1}", 0) == 0, "dk staged while K is read"
            content[f"K{j & 1}"] = ("dk", j)
            B["dk"].arrive()

    for t in ("F", "EE", "dVs", "PD"):
        content[t] = None
    threads = {"issuer": issuer(), **{f"warps{i}": warps(i) for i in range(NW)}}
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


def _failures(drop, schedules, store_delay=60):
    n = 0
    for seed in range(schedules):
        for items in (1, 2, 3, 5):
            try:
                run_model(items, seed * 7 + items, drop, store_delay)
            except AssertionError:
                n += 1
    return n


def test_protocol_holds_on_random_schedules():
    assert _failures(None, 400) == 0
    assert _failures(None, 100, store_delay=600) == 0


@pytest.mark.parametrize("drop", ["dk", "c1", "store_read", "ld4", "bar2", "bar4"])
def test_each_guard_is_needed(drop):
    # removing one guard must break some schedule (slow stores expose the store-read wait)
    assert _failures(drop, 400, store_delay=600) > 0
