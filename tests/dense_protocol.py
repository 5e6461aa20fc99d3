"""Host model of the dense prefill kernel's barrier protocol (not collected).

The kernel (csrc/dense_fwd.cuh) runs on CTA pairs.  Its roles -- the
producer warp of each CTA, the MMA warp of the leader, and the 16 softmax
warps (2 sub-tiles x 4 warps x 2 CTAs) -- synchronise only through
mbarriers, and the hardware only lets a thread wait for a phase by its
parity.  This module restates that protocol as Python generators, one per
role, next to an engine for the asynchronous work (TMA loads and st.async
stores that land later; tcgen05 MMAs and commits that execute in issue
order), and runs it in random interleavings.  It checks:

* no deadlock: the run ends with every role finished;
* phases: every parity wait finds its barrier either in the phase it
  waits for or just past it -- two phases on, the parity would name a
  later phase and the wait would hang or pass early on the hardware;
* data: every read of a buffer (the tile ring, Q, the K/V ring, S/P/O in
  TMEM) sees the contents it expects, i.e. nothing is overwritten before
  its last reader and nothing is read before it has landed.

The model follows the kernel's control flow step by step; a change to the
kernel's protocol has to be made here as well (the test that runs it says
which cases it covers).
"""
from __future__ import annotations

import random

SLOTS = 3        # K and V ring slots (two at the 256-wide qk geometry)
TILE_SLOTS = 4   # tile hand-off ring
Q_BYTES = 2      # transaction units: Q of a sub-tile per CTA
KV_BYTES = 2     # K + V half of a block per CTA
TILE_BYTES = 2   # a ring slot is two 16-byte stores


class ProtocolError(AssertionError):
    pass


class Barrier:
    def __init__(self, name: str, count: int):
        self.name, self.count = name, count
        self.pending, self.tx, self.phase = count, 0, 0   # phase = completed phases

    def _check(self):
        if self.pending < 0:
            raise ProtocolError(f"{self.name}: more arrivals than its count in phase {self.phase}")
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self, expect_tx: int = 0):
        self.tx += expect_tx
        self.pending -= 1
        self._check()

    def complete_tx(self, n: int):
        self.tx -= n
        self._check()


class Wait:
    """A parity wait for the completion of phase `target` (parity target & 1)."""

    def __init__(self, bar: Barrier, target: int, who: str):
        self.bar, self.target, self.who = bar, target, who

    def ready(self) -> bool:
        ph = self.bar.phase
        if ph > self.target + 1 or ph < self.target:
            raise ProtocolError(
                f"{self.who}: waits on {self.bar.name} for phase {self.target} "
                f"(parity {self.target & 1}) but the barrier has completed {ph} phases")
        return ph == self.target + 1


INVALID = None


def sub_blocks(tile, i):
    return 0 if tile is INVALID else tile[i]


class Model:
    """One CTA pair working through `tiles`, a list of (n0, n1) KV block counts."""

    def __init__(self, tiles, rng: random.Random, q_full_both: bool = True,
                 early_fetch: bool = False, slots: int = SLOTS):
        # The two switches restate designs the kernel does not use, for the
        # test that shows the model catches them: q_full_both=False lets only
        # the leader's producer arrive on q_full; early_fetch=True has the
        # MMA warp read the next tile at the start of the current one.
        self.tiles, self.rng, self.q_full_both = list(tiles), rng, q_full_both
        self.early_fetch = early_fetch
        self.slots = slots
        B = Barrier
        # Barriers of each CTA (index 0 = leader, 1 = peer), as the kernel initialises them.
        self.bar = []
        for r in range(2):
            d = {}
            for i in range(2):
                d[f"q_full{i}"] = B(f"q_full{i}@{r}", 2 if q_full_both else 1)
                d[f"q_empty{i}"] = B(f"q_empty{i}@{r}", 1)
                d[f"s_full{i}"] = B(f"s_full{i}@{r}", 1)
                d[f"p_full{i}"] = B(f"p_full{i}@{r}", 8)
                d[f"o_full{i}"] = B(f"o_full{i}@{r}", 1)
                d[f"o_empty{i}"] = B(f"o_empty{i}@{r}", 8)
            for s in range(self.slots):
                d[f"full_kv{s}"] = B(f"full_kv{s}@{r}", 1)
                d[f"empty_k{s}"] = B(f"empty_k{s}@{r}", 1)
                d[f"empty_v{s}"] = B(f"empty_v{s}@{r}", 1)
            for s in range(TILE_SLOTS):
                d[f"tile_full{s}"] = B(f"tile_full{s}@{r}", 1)
                d[f"tile_empty{s}"] = B(f"tile_empty{s}@{r}", 18)
            d["drain"] = B(f"drain@{r}", 1)
            self.bar.append(d)
        # Buffer contents (tags), per CTA.
        self.ring = [[("init",)] * TILE_SLOTS for _ in range(2)]
        self.q = [[None, None] for _ in range(2)]
        self.kbuf = [[None] * self.slots for _ in range(2)]
        self.vbuf = [[None] * self.slots for _ in range(2)]
        # TMEM of each CTA, per sub-tile: S_i (P_i overwrites half of it) and
        # O_i, with how many of the group's 4 warps have read S / written P /
        # read O (each warp owns 32 of the 128 rows).
        self.s = [[None, None] for _ in range(2)]
        self.s_reads = [[0, 0] for _ in range(2)]
        self.p = [[None, None] for _ in range(2)]
        self.p_writes = [[0, 0] for _ in range(2)]
        self.o = [[None, None] for _ in range(2)]
        self.o_reads = [[0, 0] for _ in range(2)]
        self.async_ops = []   # landing loads / stores: (fn)
        self.mma_queue = []   # tcgen05 ops in issue order

    # ------------------------------------------------------------ async work
    def land_later(self, fn):
        self.async_ops.append(fn)

    def tma(self, r, buf, idx, tag, bar, n):
        def land():
            buf[r][idx] = tag
            bar.complete_tx(n)
        self.land_later(land)

    def mma(self, fn):
        self.mma_queue.append(fn)

    def commit(self, names, mask):
        def arrive():
            for r in (0, 1):
                if mask & (1 << r):
                    for nm in names:
                        self.bar[r][nm].arrive()
        self.mma_queue.append(arrive)

    # --------------------------------------------------------------- roles
    def producer(self, r):
        leader = r == 0
        bl, bme = self.bar[0], self.bar[r]
        blk = 0
        k = 0
        while True:
            ts = k % TILE_SLOTS
            if leader:
                yield Wait(bl[f"tile_empty{ts}"], k // TILE_SLOTS - 1, "producer@0 tile_empty")
                ti = self.tiles[k] if k < len(self.tiles) else INVALID
                for rr in (0, 1):
                    fb = self.bar[rr][f"tile_full{ts}"]
                    fb.arrive(expect_tx=TILE_BYTES)

                    def land(rr=rr, fb=fb, ti=ti, k=k, ts=ts):
                        self.ring[rr][ts] = ("tile", k, ti)
                        fb.complete_tx(TILE_BYTES)
                    self.land_later(land)
            else:
                yield Wait(bme[f"tile_full{ts}"], k // TILE_SLOTS, "producer@1 tile_full")
                tag = self.ring[1][ts]
                want = self.tiles[k] if k < len(self.tiles) else INVALID
                if tag != ("tile", k, want):
                    raise ProtocolError(f"producer@1 read {tag} for tile {k}")
                ti = want
                if ti is not INVALID:
                    bl[f"tile_empty{ts}"].arrive()
            if ti is INVALID:
                return
            nb = (sub_blocks(ti, 0), sub_blocks(ti, 1))

            def load_kv(blk):
                slot = blk % self.slots
                yield Wait(bme[f"empty_k{slot}"], blk // self.slots - 1, f"producer@{r} empty_k")
                if leader:
                    bl[f"full_kv{slot}"].arrive(expect_tx=2 * KV_BYTES)
                self.tma(r, self.kbuf, slot, ("k", blk), bl[f"full_kv{slot}"], KV_BYTES // 2)
                yield Wait(bme[f"empty_v{slot}"], blk // self.slots - 1, f"producer@{r} empty_v")
                self.tma(r, self.vbuf, slot, ("v", blk), bl[f"full_kv{slot}"], KV_BYTES // 2)

            # the tile's first K/V block goes out before its Q
            if max(nb) > 0:
                yield from load_kv(blk)
            for i in (0, 1):
                yield Wait(bme[f"q_empty{i}"], k - 1, f"producer@{r} q_empty{i} tile {k}")
                qf = bl[f"q_full{i}"]
                if nb[i] > 0:
                    if leader:
                        qf.arrive(expect_tx=2 * Q_BYTES)
                    elif self.q_full_both:
                        qf.arrive()
                    self.tma(r, self.q, i, ("q", k, i), qf, Q_BYTES)
                elif leader or self.q_full_both:
                    qf.arrive()
            for n in range(1, max(nb)):
                yield from load_kv(blk + n)
            blk += max(nb)
            k += 1

    def mma_warp(self):
        bl = self.bar[0]
        p_cnt, o_cnt = [0, 0], [0, 0]

        def expect(buf, tag, what):
            for r in (0, 1):
                if buf[r] != tag:
                    raise ProtocolError(f"MMA {what}: CTA {r} holds {buf[r]}, expected {tag}")

        def issue_s(i, b, k, n):
            def op():
                expect([self.q[r][i] for r in (0, 1)], ("q", k, i), f"S{i} reads Q")
                expect([self.kbuf[r][b % self.slots] for r in (0, 1)], ("k", b), f"S{i} reads K")
                for r in (0, 1):
                    if self.s[r][i] is not None and self.s_reads[r][i] < 4:
                        raise ProtocolError(f"S{i}({k},{n}) overwrites S {self.s[r][i]} before "
                                            f"every warp read it")
                    if self.p[r][i] is not None:
                        raise ProtocolError(f"S{i}({k},{n}) overwrites P {self.p[r][i]} not yet read")
                    self.s[r][i], self.s_reads[r][i] = ("s", k, n), 0
            self.mma(op)
            self.commit([f"s_full{i}"], 0x3)

        def issue_pv(i, b, k, n):
            def op():
                expect([self.vbuf[r][b % self.slots] for r in (0, 1)], ("v", b), f"PV{i} reads V")
                for r in (0, 1):
                    if self.p[r][i] != ("p", k, n) or self.p_writes[r][i] != 4:
                        raise ProtocolError(f"PV{i}({k},{n}) reads P {self.p[r][i]} written by "
                                            f"{self.p_writes[r][i]} of 4 warps")
                    self.p[r][i], self.p_writes[r][i] = None, 0
                    if n == 0:
                        if self.o[r][i] is not None:
                            raise ProtocolError(f"PV{i}({k},0) overwrites O {self.o[r][i]} not yet read")
                    elif self.o[r][i] != ("o", k, n - 1):
                        raise ProtocolError(f"PV{i}({k},{n}) accumulates into O {self.o[r][i]}")
                    self.o[r][i] = ("o", k, n)
            self.mma(op)

        def fetch(k):
            ts = k % TILE_SLOTS
            yield Wait(bl[f"tile_full{ts}"], k // TILE_SLOTS, "mma tile_full")
            want = self.tiles[k] if k < len(self.tiles) else INVALID
            if self.ring[0][ts] != ("tile", k, want):
                raise ProtocolError(f"mma read {self.ring[0][ts]} for tile {k}")
            if want is not INVALID:
                bl[f"tile_empty{ts}"].arrive()
            return want

        def start_tile(n, b, k):
            for i in (0, 1):
                yield Wait(bl[f"q_full{i}"], k, f"mma q_full{i}")
            if max(n) > 0:
                yield Wait(bl[f"full_kv{b % self.slots}"], b // self.slots, "mma full_kv")
                for i in (0, 1):
                    if n[i] > 0:
                        issue_s(i, b, k, 0)
                    if n[i] <= 1:
                        self.commit([f"q_empty{i}"], 0x3)
                self.commit([f"empty_k{b % self.slots}"], 0x3)
            else:
                for i in (0, 1):
                    self.commit([f"q_empty{i}"], 0x3)

        blk, k = 0, 0
        cur = yield from fetch(0)
        if cur is not INVALID:
            yield from start_tile(cur, blk, k)
        while cur is not INVALID:
            nb = cur
            nblk = max(nb)
            nxt = INVALID
            if nblk == 0 or self.early_fetch:
                nxt = yield from fetch(k + 1)
            for n in range(nblk):
                b = blk + n
                last = n + 1 == nblk
                if last and not self.early_fetch:
                    nxt = yield from fetch(k + 1)
                nbn = (sub_blocks(nxt, 0), sub_blocks(nxt, 1))
                next_s = [nbn[0] > 0, nbn[1] > 0] if last else [n + 1 < nb[0], n + 1 < nb[1]]
                more = next_s[0] or next_s[1]
                if more:
                    yield Wait(bl[f"full_kv{(b + 1) % self.slots}"], (b + 1) // self.slots, "mma full_kv")
                for i in (0, 1):
                    if n < nb[i]:
                        if n == 0:
                            yield Wait(bl[f"o_empty{i}"], o_cnt[i] - 1, f"mma o_empty{i}")
                        yield Wait(bl[f"p_full{i}"], p_cnt[i], f"mma p_full{i}")
                        p_cnt[i] += 1
                        issue_pv(i, b, k, n)
                        if n == nb[i] - 1:
                            self.commit([f"o_full{i}"], 0x3)
                            o_cnt[i] += 1
                    if i == 1:
                        self.commit([f"empty_v{b % self.slots}"], 0x3)
                    if last and nxt is not INVALID:
                        yield Wait(bl[f"q_full{i}"], k + 1, f"mma q_full{i}")
                    if next_s[i]:
                        kk, nn = (k + 1, 0) if last else (k, n + 1)
                        issue_s(i, b + 1, kk, nn)
                        nbi = nbn[i] if last else nb[i]
                        if nn == nbi - 1:
                            self.commit([f"q_empty{i}"], 0x3)
                    elif last and nxt is not INVALID:
                        self.commit([f"q_empty{i}"], 0x3)
                if more:
                    self.commit([f"empty_k{(b + 1) % self.slots}"], 0x3)
            if nblk == 0 and nxt is not INVALID:
                yield from start_tile(nxt, blk, k + 1)
            blk += nblk
            k += 1
            cur = nxt
        self.commit(["drain"], 0x1)
        yield Wait(bl["drain"], 0, "mma drain")

    def softmax(self, r, sub, w):
        bme, bl = self.bar[r], self.bar[0]
        s_cnt = o_cnt = 0
        k = 0
        who = f"softmax@{r} sub{sub} warp{w}"
        while True:
            ts = k % TILE_SLOTS
            yield Wait(bme[f"tile_full{ts}"], k // TILE_SLOTS, who + " tile_full")
            want = self.tiles[k] if k < len(self.tiles) else INVALID
            if self.ring[r][ts] != ("tile", k, want):
                raise ProtocolError(f"{who} read {self.ring[r][ts]} for tile {k}")
            if want is INVALID:
                return
            nb = sub_blocks(want, sub)
            for n in range(nb):
                yield Wait(bme[f"s_full{sub}"], s_cnt, who + " s_full")
                s_cnt += 1
                if self.s[r][sub] != ("s", k, n):
                    raise ProtocolError(f"{who} reads S {self.s[r][sub]}, expected {(k, n)}")
                self.s_reads[r][sub] += 1
                # O(n-1) may be rescaled here: PV(n-1) must be complete
                if n > 0 and self.o[r][sub] != ("o", k, n - 1):
                    raise ProtocolError(f"{who} rescales O {self.o[r][sub]} before PV({k},{n - 1})")
                yield None  # other warps run between the read of S and the write of P
                if self.p_writes[r][sub] == 0:
                    self.p[r][sub] = ("p", k, n)
                elif self.p[r][sub] != ("p", k, n):
                    raise ProtocolError(f"{who} writes P({k},{n}) over {self.p[r][sub]}")
                self.p_writes[r][sub] += 1
                bl[f"p_full{sub}"].arrive()
            if self.ring[r][ts] != ("tile", k, want):
                raise ProtocolError(f"{who} re-read {self.ring[r][ts]} for tile {k}")
            bl[f"tile_empty{ts}"].arrive()
            if nb > 0:
                yield Wait(bme[f"o_full{sub}"], o_cnt, who + " o_full")
                if self.o[r][sub] != ("o", k, nb - 1):
                    raise ProtocolError(f"{who} reads O {self.o[r][sub]}, expected {(k, nb - 1)}")
                self.o_reads[r][sub] += 1
                if self.o_reads[r][sub] == 4:
                    self.o[r][sub], self.o_reads[r][sub] = None, 0
                bl[f"o_empty{sub}"].arrive()
                o_cnt += 1
            k += 1

    # --------------------------------------------------------------- engine
    def run(self, max_steps: int = 2_000_000):
        acts = {"producer@0": self.producer(0), "producer@1": self.producer(1),
                "mma": self.mma_warp()}
        for r in (0, 1):
            for sub in (0, 1):
                for w in range(4):
                    acts[f"softmax@{r}.{sub}.{w}"] = self.softmax(r, sub, w)
        waits = {name: None for name in acts}
        rng = self.rng
        for _ in range(max_steps):
            # re-check every blocked wait (the phase invariant holds at all times)
            runnable = [n for n, wt in waits.items() if n in acts and (wt is None or wt.ready())]
            choices = [("act", n) for n in runnable]
            if self.async_ops:
                choices.append(("land", None))
            if self.mma_queue:
                choices.append(("mma", None))
            if not choices:
                if acts:
                    blocked = {n: (w.bar.name, w.target, w.bar.phase) for n, w in waits.items()
                               if n in acts and w is not None}
                    raise ProtocolError(f"deadlock: {blocked}")
                return
            kind, name = rng.choice(choices)
            if kind == "land":
                self.async_ops.pop(rng.randrange(len(self.async_ops)))()
            elif kind == "mma":
                self.mma_queue.pop(0)()
            else:
                try:
                    waits[name] = next(acts[name])
                except StopIteration:
                    del acts[name]
                    waits.pop(name)
        raise ProtocolError("step limit reached")


def run_case(tiles, seed: int, **kw):
    Model(tiles, random.Random(seed), **kw).run()
