"""Host model of the sparse prefill kernel's barrier protocol (not collected).

The kernel (csrc/sparse_fwd.cuh) runs each (token, value half) on one CTA
whose roles -- the loader warps, the MMA warp and the 4 softmax warps --
synchronise only through mbarriers: a chunk's slot is filled by the
loaders (full), read by S(c) and PV(c) and freed by PV(c)'s commit
(empty); S(c) goes to TMEM buffer c % 2, whose softmax writes P(c) over it
(p_full) after waiting for PV(c - 1) (pv_done), so that it may rescale O.
The MMA warp issues S(c) and PV(c) in whichever order their inputs arrive,
S(c) never before PV(c - 2).  The hardware only lets a thread wait for a
phase by its parity.  This module restates that protocol as Python
generators, one per role, next to an engine for the asynchronous work
(cp.async copies that land later; tcgen05 MMAs and commits that execute in
issue order), and runs it in random interleavings.  It checks:

* no deadlock: the run ends with every role finished;
* phases: every parity wait finds its barrier either in the phase it waits
  for or just past it (anything else would hang or pass early on the
  hardware);
* data: every read of a buffer (a chunk slot, S/P/O in TMEM) sees the
  contents it expects: nothing is overwritten before its last reader and
  nothing is read before it has landed.

The model follows the kernel's control flow step by step; a change to the
kernel's protocol has to be made here as well.
"""
from __future__ import annotations

import random

from dense_protocol import Barrier, ProtocolError, Wait

SLOTS = 2        # chunk slots
WARPS = 4        # softmax warps (32 rows each)


class Model:
    """One CTA's chunks (`nchunks`).

    `rescale` is the set of (warp, chunk) whose rows raise the running
    maximum enough to rescale O.  The switches restate designs the kernel
    does not use, for the tests that show the model catches them:
    stale_pv_wait=True has the softmax wait for PV(c - 2) where it means
    PV(c - 1) before rescaling O; free_after_s=True frees a chunk's slot
    once S(c) is done instead of after PV(c), which still reads its V.
    (With two slots the explicit rule that S(c) follows PV(c - 2) is
    implied: S(c) needs chunk c's rows, whose slot PV(c - 2) frees.)
    One relaxation the model accepts and the kernel does not take: a warp
    could skip the wait for PV(c - 1) when none of its rows rescales (S(c),
    which it waited for, was issued after PV(c - 2), so the barrier is at
    most one phase behind) -- that would rest on tcgen05 commits arriving
    in issue order.
    """

    def __init__(self, nchunks: int, rng: random.Random, rescale=frozenset(),
                 stale_pv_wait: bool = False, free_after_s: bool = False):
        self.n, self.rng, self.rescale = nchunks, rng, set(rescale)
        self.stale_pv_wait, self.free_after_s = stale_pv_wait, free_after_s
        B = Barrier
        self.bar = {}
        for s in range(SLOTS):
            self.bar[f"full{s}"] = B(f"full{s}", 1)
            self.bar[f"empty{s}"] = B(f"empty{s}", 1)
        for i in range(2):
            self.bar[f"s_full{i}"] = B(f"s_full{i}", 1)
            self.bar[f"p_full{i}"] = B(f"p_full{i}", WARPS)
        for nm in ("pv_done", "o_full", "drain"):
            self.bar[nm] = B(nm, 1)
        self.slot = [None] * SLOTS
        self.s = [None, None]
        self.s_reads = [0, 0]
        self.p = [None, None]
        self.p_writes = [0, 0]
        self.o = None
        self.async_ops = []
        self.mma_queue = []

    def commit(self, names):
        def arrive():
            for nm in names:
                self.bar[nm].arrive()
        self.mma_queue.append(arrive)

    # --------------------------------------------------------------- roles
    def loaders(self):
        b = self.bar
        for c in range(self.n):
            s = c % SLOTS
            yield Wait(b[f"empty{s}"], c // SLOTS - 1, f"loaders empty{s}")

            def land(s=s, c=c):
                self.slot[s] = c
                b[f"full{s}"].arrive()     # cp.async.mbarrier.arrive.noinc: after the copies
            self.async_ops.append(land)

    def mma_warp(self):
        b = self.bar

        def issue_s(c):
            i = c & 1

            def op():
                if self.slot[c % SLOTS] != c:
                    raise ProtocolError(f"S({c}) reads a slot holding {self.slot[c % SLOTS]}")
                if self.s[i] is not None and self.s_reads[i] < WARPS:
                    raise ProtocolError(f"S({c}) overwrites S {self.s[i]} before every warp read it")
                if self.p[i] is not None:
                    raise ProtocolError(f"S({c}) overwrites P {self.p[i]} not yet read")
                self.s[i], self.s_reads[i] = c, 0
            self.mma_queue.append(op)
            self.commit([f"s_full{i}"] + ([f"empty{c % SLOTS}"] if self.free_after_s else []))

        def issue_pv(c):
            i = c & 1

            def op():
                if self.slot[c % SLOTS] != c:
                    raise ProtocolError(f"PV({c}) reads V of chunk {self.slot[c % SLOTS]}")
                if self.p[i] != c or self.p_writes[i] != WARPS:
                    raise ProtocolError(f"PV({c}) reads P {self.p[i]} written by "
                                        f"{self.p_writes[i]} warps")
                self.p[i], self.p_writes[i] = None, 0
                if self.o != (c - 1 if c > 0 else None):
                    raise ProtocolError(f"PV({c}) accumulates into O {self.o}")
                self.o = c
            self.mma_queue.append(op)
            self.commit(["pv_done"] + ([] if self.free_after_s else [f"empty{c % SLOTS}"]))

        s_next = pv_next = 0
        while pv_next < self.n:
            # the kernel polls both conditions (test_wait) and issues whatever is ready
            opts = []
            if pv_next < s_next and Wait(b[f"p_full{pv_next & 1}"], pv_next >> 1,
                                         "mma p_full").ready():
                opts.append("pv")
            if s_next < self.n and s_next <= pv_next + 1 and \
                    Wait(b[f"full{s_next % SLOTS}"], s_next // SLOTS, "mma full").ready():
                opts.append("s")
            if not opts:
                yield None
                continue
            if self.rng.choice(opts) == "pv":
                issue_pv(pv_next)
                pv_next += 1
            else:
                issue_s(s_next)
                s_next += 1
            yield None
        self.commit(["o_full"])
        self.commit(["drain"])
        yield Wait(b["drain"], 0, "mma drain")

    def softmax(self, w):
        b = self.bar
        who = f"softmax{w}"
        for c in range(self.n):
            i = c & 1
            yield Wait(b[f"s_full{i}"], c >> 1, who + " s_full")
            if self.s[i] != c:
                raise ProtocolError(f"{who} reads S {self.s[i]}, expected {c}")
            self.s_reads[i] += 1
            yield None
            if c > (1 if self.stale_pv_wait else 0):
                yield Wait(b["pv_done"], c - (2 if self.stale_pv_wait else 1), who + " pv_done")
                if (w, c) in self.rescale and self.o != c - 1:
                    raise ProtocolError(f"{who} rescales O {self.o} before PV({c - 1}) is done")
            if self.p_writes[i] == 0:
                self.p[i] = c
            elif self.p[i] != c:
                raise ProtocolError(f"{who} writes P({c}) over {self.p[i]}")
            self.p_writes[i] += 1
            b[f"p_full{i}"].arrive()
        yield Wait(b["o_full"], 0, who + " o_full")
        if self.o != (self.n - 1 if self.n else None):
            raise ProtocolError(f"{who} reads O {self.o}, expected {self.n - 1}")

    # --------------------------------------------------------------- engine
    def run(self, max_steps: int = 2_000_000):
        acts = {"loaders": self.loaders(), "mma": self.mma_warp()}
        for w in range(WARPS):
            acts[f"softmax{w}"] = self.softmax(w)
        waits = {name: None for name in acts}
        rng = self.rng
        for _ in range(max_steps):
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
            kind, arg = rng.choice(choices)
            if kind == "land":
                self.async_ops.pop(rng.randrange(len(self.async_ops)))()
            elif kind == "mma":
                self.mma_queue.pop(0)()
            else:
                try:
                    waits[arg] = next(acts[arg])
                except StopIteration:
                    del acts[arg]
                    waits.pop(arg)
        raise ProtocolError("step limit reached")


def run_case(nchunks: int, seed: int, rescale_rate: float = 0.1, **kw):
    rng = random.Random(seed)
    rescale = {(w, c) for w in range(WARPS) for c in range(nchunks) if rng.random() < rescale_rate}
    Model(nchunks, rng, rescale=rescale, **kw).run()
