"""Model check of the state scan's barrier protocol (the MMA-warp schedule of
kimi_delta_attention_22_b200/csrc/kda_chunk_scan.cu), on the CPU.

The kernel's correctness rests on its barrier protocol, which one GPU run only
samples under one timing.  This test restates, role by role, the order in
which the kernel's threads wait, arrive, issue and touch memory, and runs that
program under many random interleavings (MMAs executing in issue order, record
copies landing at random times; each run gives every warp, the MMA pipe and the
copies a random speed, so that any of them can lag far behind).  It checks that

  * nothing deadlocks;
  * no barrier ever runs two phases ahead of a thread waiting on it (a parity
    wait would then stall: the hardware sees the same parity again);
  * every pair of conflicting accesses (at least one a write) to a shared
    buffer -- the halves of the two S [W ; Qg]^T / O^T column sets, the fp32 S
    (scaled by the threads, accumulated by E^T Kd, read for its fp16 copy), the
    fp16 copies of S and E^T that are MMA operands in tensor memory, and each
    part of each record stage -- happens in the order the algorithm needs.

Mbarrier semantics: a wait for the k-th completion (parity k & 1) passes when
exactly k + 1 completions have happened."""
import random

import pytest


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.completed = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.completed += 1
            self.pending = self.count


class Model:
    def __init__(self, nch, nstage, nw=8, seed=0):
        self.rng = random.Random(seed)
        self.nch, self.ns = nch, nstage
        B = Barrier
        self.bars = {"bar1": B("bar1", 1), "bar2": B("bar2", 1), "bar3": B("bar3", 1),
                     "eready": B("eready", nw), "sready": B("sready", nw)}
        for s in range(nstage):
            self.bars[f"full{s}"] = B(f"full{s}", 1)
            self.bars[f"empty{s}"] = B(f"empty{s}", 1)
        self.log = {}          # buffer -> [(key, is_write, who)]
        self.pipe = []         # issued tcgen05 work, executed in order
        self.copies = []       # record copies in flight
        self.actors = {"mma": self.issuer(), "copy": self.copier()}
        self.warps = [f"w{w}" for w in range(nw)]
        for w in self.warps:
            self.actors[w] = self.state_warp(w)
        self.blocked = {}      # actor -> (barrier, k)
        # per-run speeds, so that some warps, the MMA pipe or the copies lag far behind
        speeds = (0.02, 0.2, 1.0, 5.0)
        self.speed = {a: self.rng.choice(speeds) for a in list(self.actors) + ["pipe", "copy"]}

    # ---- accesses: key = (use of the buffer, order within that use)
    def touch(self, buf, key, write, who):
        self.log.setdefault(buf, []).append((key, write, who))

    def touch_slices(self, buf, key, write, who):
        """An MMA reads or accumulates every state warp's slice (lanes x columns) of a
        tensor-memory operand; each warp touches only its own slice."""
        for w in self.warps:
            self.touch(f"{buf}.{w}", key, write, who)

    def stage_touch(self, part, m, rank, write, who):
        self.touch(f"stage{m % self.ns}.{part}", (m // self.ns, rank), write, who)

    def execute(self, op):
        kind, m = op
        if kind == "mma1":         # S_m [W ; Qg]^T -> both halves of d1[m & 1]
            self.touch(f"d1lo_{m & 1}", (m // 2, 0), True, "mma1")
            self.touch(f"d1hi_{m & 1}", (m // 2, 0), True, "mma1")
            self.touch_slices("as", (m, 1), False, "mma1")
            self.stage_touch("WQ", m, 1, False, "mma1")
        elif kind == "mma2":       # E^T Kd accumulated onto the decayed fp32 S
            self.touch_slices("s32", (m, 1), True, "mma2")
            self.touch_slices("ae", (m, 1), False, "mma2")
            self.stage_touch("KD", m, 1, False, "mma2")
        elif kind == "mma3":       # E^T Aqk^T accumulated onto the upper half of d1[m & 1]
            self.touch(f"d1hi_{m & 1}", (m // 2, 1), True, "mma3")
            self.touch_slices("ae", (m, 1), False, "mma3")
            self.stage_touch("AQ", m, 1, False, "mma3")
        elif kind == "commit":
            self.bars[m].arrive()

    def land(self, m):
        for part in ("WQ", "KD", "AQ", "UT", "DEC"):
            self.stage_touch(part, m, 0, True, "copy")
        self.bars[f"full{m % self.ns}"].arrive()

    # ---- programs (generators yielding ("wait", bar, k) or nothing)
    def copier(self):
        nch, ns = self.nch, self.ns
        for m in range(min(nch, ns)):
            self.copies.append(m)
        yield
        for m in range(ns, nch):
            # stage m % ns takes chunk m once chunk m - ns's MMAs are done
            yield ("wait", f"empty{m % ns}", m // ns - 1)
            self.copies.append(m)
            yield

    def issuer(self):
        nch, ns = self.nch, self.ns
        for m in range(nch):
            if m > 0:
                yield ("wait", "sready", m - 1)
            yield ("wait", f"full{m % ns}", m // ns)
            self.pipe += [("mma1", m), ("commit", "bar1")]
            yield
            yield ("wait", "eready", m)
            self.pipe += [("mma2", m), ("commit", "bar2"), ("mma3", m), ("commit", "bar3"),
                          ("commit", f"empty{m % ns}")]
            yield

    def state_warp(self, who):
        for m in range(self.nch):
            yield ("wait", f"full{m % self.ns}", m // self.ns)
            self.stage_touch("UT", m, 1, False, who)                # U^T read ahead of S W^T
            self.stage_touch("DEC", m, 1, False, who)
            self.touch(f"s32.{who}", (m, 0), True, who)             # S <- S Diag(dec)
            yield ("wait", "bar1", m)
            self.touch(f"d1lo_{m & 1}", (m // 2, 1), False, who)   # S W^T read out
            self.touch(f"ae.{who}", (m, 0), True, who)              # E^T stored
            yield
            self.bars["eready"].arrive()
            yield ("wait", "bar2", m)
            self.touch(f"s32.{who}", (m, 2), False, who)            # S_{m+1} read for its copy
            self.touch(f"as.{who}", (m + 1, 0), True, who)          # fp16 S_{m+1} stored
            yield
            self.bars["sready"].arrive()
            yield ("wait", "bar3", m)
            self.touch(f"d1hi_{m & 1}", (m // 2, 2), False, who)   # outputs read out
            yield

    # ---- scheduler
    def check_alias(self):
        for a, (b, k) in self.blocked.items():
            assert self.bars[b].completed <= k + 1, f"{a} waits on {b} #{k}: barrier ran two phases ahead"

    def run(self):
        live = dict(self.actors)
        while True:
            self.check_alias()
            ready = [a for a in live if a not in self.blocked or
                     self.bars[self.blocked[a][0]].completed == self.blocked[a][1] + 1]
            choices = [("actor", a) for a in ready]
            weights = [self.speed[a] for a in ready]
            if self.pipe:
                choices.append(("pipe", None))
                weights.append(self.speed["pipe"])
            if self.copies:
                choices += [("copy", i) for i in range(len(self.copies))]
                weights += [self.speed["copy"]] * len(self.copies)
            if not choices:
                assert not live, f"deadlock: blocked {self.blocked}"
                return
            kind, x = self.rng.choices(choices, weights)[0]
            if kind == "pipe":
                self.execute(self.pipe.pop(0))
            elif kind == "copy":
                self.land(self.copies.pop(x))
            else:
                self.blocked.pop(x, None)
                try:
                    step = next(live[x])
                except StopIteration:
                    del live[x]
                    continue
                if step is not None:
                    _, b, k = step
                    assert self.bars[b].completed <= k + 1, f"{x}: {b} ran two phases ahead of wait #{k}"
                    self.blocked[x] = (b, k)

    def check_order(self):
        for buf, events in self.log.items():
            for i, (ka, wa, a) in enumerate(events):
                for kb, wb, b in events[i + 1:]:
                    if (wa or wb) and kb < ka:
                        raise AssertionError(f"{buf}: {b} {kb} after {a} {ka}")


@pytest.mark.parametrize("nstage", [2, 3])
@pytest.mark.parametrize("nch", [0, 1, 2, 3, 5, 9])
def test_mma_warp_schedule_protocol(nch, nstage):
    for seed in range(150):
        m = Model(nch, nstage, nw=4, seed=seed)
        m.run()
        m.check_order()


@pytest.mark.parametrize("dropped", ["sready", "eready", "full", "empty"])
def test_protocol_check_catches_a_missing_wait(dropped):
    """The check has teeth: drop any one of the MMA or copy thread's waits and some
    interleaving breaks an ordering or runs a barrier two phases ahead."""
    class Dropped(Model):
        def issuer(self):
            for step in super().issuer():
                if step is not None and step[1].startswith(dropped) and step[2] > 0:
                    continue
                yield step

        def copier(self):
            for step in super().copier():
                if step is not None and step[1].startswith(dropped):
                    continue
                yield step

    caught = 0
    for seed in range(300):
        m = Dropped(6, 3, nw=4, seed=seed)
        try:
            m.run()
            m.check_order()
        except AssertionError:
            caught += 1
    assert caught > 0
