"""Model check of the reverse state scan's barrier protocol (the schedule of
kimi_delta_attention_22_b200/csrc/kda_chunk_bwd_scan.cu), on the CPU.

As for the forward scan (test_scan_protocol.py, whose scheduler and checks this
reuses), the kernel's correctness rests on its barrier protocol, which one GPU
run only samples under one timing.  The program below restates, role by role,
the order in which the reverse scan's threads wait, arrive, issue and touch
memory: per step r (chunk nch - 1 - r) the state warps store dO^T and scale dS'
(then arrive on oready), the MMA thread forms dE^T (bar1), the warps store the
fp16 -dE^T (eready), the MMA thread accumulates the dS update (bar2, and the
stage's empty barrier), the warps store the fp16 dS (sready).  Under many random
interleavings it checks for deadlock, for a barrier running two phases ahead of
a waiter, and for the order of every pair of conflicting accesses to the fp32
dS, the fp16 operand copies (dS, dO^T, -dE^T) and the dE^T accumulator in
tensor memory, and each part of each stage (record, dO tile)."""
import random

import pytest

from test_scan_protocol import Barrier, Model


class BwdModel(Model):
    def __init__(self, nch, nstage, nw=4, seed=0):
        self.rng = random.Random(seed)
        self.nch, self.ns = nch, nstage
        B = Barrier
        self.bars = {"bar1": B("bar1", 1), "bar2": B("bar2", 1), "oready": B("oready", nw),
                     "eready": B("eready", nw), "sready": B("sready", nw)}
        for s in range(nstage):
            self.bars[f"full{s}"] = B(f"full{s}", 1)
            self.bars[f"empty{s}"] = B(f"empty{s}", 1)
        self.log, self.pipe, self.copies, self.blocked = {}, [], [], {}
        self.actors = {"mma": self.issuer(), "copy": self.copier()}
        self.warps = [f"w{w}" for w in range(nw)]
        for w in self.warps:
            self.actors[w] = self.state_warp(w)
        speeds = (0.02, 0.2, 1.0, 5.0)
        self.speed = {a: self.rng.choice(speeds) for a in list(self.actors) + ["pipe", "copy"]}

    def execute(self, op):
        kind, r = op
        if kind == "mma_e":        # dE^T = dS' Kd^T + dO^T Aqk
            self.touch_slices("de", (r, 0), True, "mma_e")
            self.touch_slices("as", (r, 1), False, "mma_e")
            self.touch_slices("ao", (r, 1), False, "mma_e")
            self.stage_touch("KD", r, 1, False, "mma_e")
            self.stage_touch("AQ", r, 1, False, "mma_e")
        elif kind == "mma_s":      # dS += dO^T Qg + (-dE^T) W, onto the scaled fp32 dS
            self.touch_slices("ds32", (r, 1), True, "mma_s")
            self.touch_slices("ao", (r, 2), False, "mma_s")
            self.touch_slices("ae", (r, 1), False, "mma_s")
            self.stage_touch("WQ", r, 1, False, "mma_s")
        elif kind == "commit":
            self.bars[r].arrive()

    def land(self, r):
        for part in ("WQ", "KD", "AQ", "DEC", "DO"):
            self.stage_touch(part, r, 0, True, "copy")
        self.bars[f"full{r % self.ns}"].arrive()

    def issuer(self):
        nch, ns = self.nch, self.ns
        for r in range(nch):
            if r > 0:
                yield ("wait", "sready", r - 1)
            yield ("wait", f"full{r % ns}", r // ns)
            yield ("wait", "oready", r)
            self.pipe += [("mma_e", r), ("commit", "bar1")]
            yield
            yield ("wait", "eready", r)
            self.pipe += [("mma_s", r), ("commit", "bar2"), ("commit", f"empty{r % ns}")]
            yield

    def state_warp(self, who):
        for r in range(self.nch):
            yield ("wait", f"full{r % self.ns}", r // self.ns)
            self.stage_touch("DO", r, 1, False, who)
            self.stage_touch("DEC", r, 1, False, who)
            self.touch(f"ao.{who}", (r, 0), True, who)       # fp16 dO^T stored
            self.touch(f"ds32.{who}", (r, 0), True, who)     # dS' read out, scaled in place
            yield
            self.bars["oready"].arrive()
            yield ("wait", "bar1", r)
            self.touch(f"de.{who}", (r, 1), False, who)      # dE^T read out
            self.touch(f"ae.{who}", (r, 0), True, who)       # fp16 -dE^T stored
            yield
            self.bars["eready"].arrive()
            yield ("wait", "bar2", r)
            self.touch(f"ds32.{who}", (r, 2), False, who)    # the updated dS read
            self.touch(f"as.{who}", (r + 1, 0), True, who)   # its fp16 copy stored
            yield
            self.bars["sready"].arrive()


@pytest.mark.parametrize("nstage", [2, 3])
@pytest.mark.parametrize("nch", [0, 1, 2, 3, 5, 9])
def test_reverse_scan_schedule_protocol(nch, nstage):
    for seed in range(150):
        m = BwdModel(nch, nstage, seed=seed)
        m.run()
        m.check_order()


@pytest.mark.parametrize("role,dropped", [("mma", "oready"), ("mma", "eready"), ("copy", "empty"),
                                          ("warp", "full"), ("warp", "bar1"), ("warp", "bar2")])
def test_reverse_protocol_check_catches_a_missing_wait(role, dropped):
    """Drop one of the waits that carries the protocol and some interleaving breaks an
    ordering or runs a barrier two phases ahead.  (The MMA thread's own waits on the
    stage's full barrier and on sready are implied by oready, which the state warps
    arrive on only after both: dropping either alone breaks nothing.)"""
    class Dropped(BwdModel):
        def _filter(self, gen, mine):
            for step in gen:
                if mine and step is not None and step[1].startswith(dropped):
                    continue
                yield step

        def issuer(self):
            return self._filter(super().issuer(), role == "mma")

        def copier(self):
            return self._filter(super().copier(), role == "copy")

        def state_warp(self, who):
            return self._filter(super().state_warp(who), role == "warp")

    caught = 0
    for seed in range(300):
        m = Dropped(6, 2, seed=seed)
        try:
            m.run()
            m.check_order()
        except AssertionError:
            caught += 1
    assert caught > 0


def test_mma_thread_waits_implied_by_oready():
    """The redundancy stated above, checked: without the MMA thread's full and sready
    waits every interleaving still keeps every order."""
    class Lean(BwdModel):
        def issuer(self):
            for step in super().issuer():
                if step is not None and step[1].startswith(("full", "sready")):
                    continue
                yield step

    for seed in range(200):
        m = Lean(5, 2, seed=seed)
        m.run()
        m.check_order()
