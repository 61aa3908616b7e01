"""A model of bsa_attn's mbarrier protocol, run on the CPU.

The attention kernel (block_sparse_kv_bsa_b200/csrc/attn_sm100.cu) is a
pipeline of five roles -- the TMA producer, the P V issuer, the Q K^T issuer
and two softmax warpgroups -- that wait on mbarriers by phase parity.  A
parity wait is only exact while the barrier is neither a phase behind nor
two phases ahead of the completion the waiter means.  This test replays the
kernel's slot, buffer and parity arithmetic with every copy and every
product completing at random times, and checks in every interleaving that

* no wait is satisfied by a different completion than the one it stands
  for (the model knows each barrier's completion count), and
* the pipeline never deadlocks,

whether a tile waits for the previous P V (it does so only when its
reference maximum moved and O must be rescaled) or not.

It also checks that the model has teeth: with one S-ready barrier per
warpgroup (instead of per S buffer) some interleavings stop, because
S_{t+2} depends only on the other warpgroup and can complete before the
waiting warpgroup looks.
"""
import random

import pytest

KS = VS = SB = 3        # K ring, V ring, S buffers
KLEAD = 2               # K tiles issued ahead of the V tile


class Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.done = 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, "more arrivals than the barrier's count in one phase"
        self._check()

    def expect_tx(self, b):
        self.tx += b
        self.arrive()

    def complete_tx(self, b):
        self.tx -= b
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def passes(self, parity):
        return (self.done & 1) != parity


class Named:
    def __init__(self, need):
        self.need, self.count, self.gen = need, 0, 0

    def arrive(self):
        self.count += 1
        if self.count == self.need:
            self.count, self.gen = 0, self.gen + 1


class Pipe:
    def __init__(self, rng, per_warpgroup_s):
        self.rng = rng
        self.per_wg_s = per_warpgroup_s
        B = {"Q_FULL": Bar(1)}
        for s in range(3):
            for name in ("K_FULL", "K_EMPTY", "V_FULL", "V_EMPTY", "S_FULL"):
                B[f"{name}{s}"] = Bar(1)
            B[f"PV_READY{s}"] = Bar(2)          # a warpgroup's arrivals, scaled down
        self.B = B
        self.tma = []                            # (barrier, bytes)
        self.mma = {"qk": [], "pv": []}          # in-order commits per issuer

    def s_full(self, t, g):
        if self.per_wg_s:
            return f"S_FULL{g}", (t >> 1) & 1, t >> 1
        return f"S_FULL{t % SB}", (t // SB) & 1, t // SB

    def progress(self):
        did = False
        if self.tma and self.rng.random() < 0.6:
            bar, b = self.tma.pop(self.rng.randrange(len(self.tma)))
            self.B[bar].complete_tx(b)
            did = True
        for who in ("qk", "pv"):
            if self.mma[who] and self.rng.random() < 0.6:
                self.B[self.mma[who].pop(0)].arrive()
                did = True
        return did


def producer(p, n):
    p.B["Q_FULL"].expect_tx(2)
    p.tma.append(("Q_FULL", 2))
    for step in range(n + KLEAD):
        if step < n:
            t, sl = step, step % KS
            if t >= KS:
                yield ("wait", f"K_EMPTY{sl}", ((t // KS) - 1) & 1, t // KS - 1)
            p.B[f"K_FULL{sl}"].expect_tx(2)
            p.tma.append((f"K_FULL{sl}", 2))
        t = step - KLEAD
        if 0 <= t < n:
            sl = t % VS
            if t >= VS:
                yield ("wait", f"V_EMPTY{sl}", ((t // VS) - 1) & 1, t // VS - 1)
            p.B[f"V_FULL{sl}"].expect_tx(2)
            p.tma.append((f"V_FULL{sl}", 2))


def qk_issuer(p, n):
    yield ("wait", "Q_FULL", 0, 0)
    for t in range(n):
        sl = t % KS
        yield ("wait", f"K_FULL{sl}", (t // KS) & 1, t // KS)
        if t >= SB:
            yield ("wait", f"V_EMPTY{sl}", ((t // VS) - 1) & 1, t // VS - 1)
        p.mma["qk"] += [f"K_EMPTY{sl}", p.s_full(t, t & 1)[0]]


def pv_issuer(p, n):
    for i in range(n):
        sl = i % VS
        yield ("wait", f"PV_READY{sl}", (i // VS) & 1, i // VS)
        p.mma["pv"] += [f"V_EMPTY{sl}"]


def softmax(p, n, g, tokens):
    for t in range(g, n, 2):
        bar, parity, idx = p.s_full(t, g)
        yield ("wait", bar, parity, idx)
        if t > 0:
            yield ("sync", tokens[g ^ 1])        # m_{t-1} from the other warpgroup
        if t + 1 < n:
            tokens[g].arrive()
        # The P V of tile t - 1 (V_EMPTY of its slot) is awaited only when
        # the reference maximum moved (O is then rescaled in between); the
        # model draws that event.
        if t > 0 and p.rng.random() < p.rescale:
            yield ("wait", f"V_EMPTY{(t - 1) % VS}", ((t - 1) // VS) & 1, (t - 1) // VS)
        yield ("wait", f"V_FULL{t % VS}", (t // VS) & 1, t // VS)
        p.B[f"PV_READY{t % VS}"].arrive(2)
    if n > 0 and g == ((n - 1) & 1):               # the warpgroup that saw S_{n-1}
        yield ("wait", f"V_EMPTY{(n - 1) % VS}", ((n - 1) // VS) & 1, (n - 1) // VS)


def simulate(n, seed, per_warpgroup_s=False, rescale=0.3):
    """Returns None when the pipeline drains, else a description of the fault.
    ``rescale`` is the chance that a tile moves its reference maximum (and so
    waits for the previous P V before releasing P)."""
    p = Pipe(random.Random(seed), per_warpgroup_s)
    p.rescale = rescale
    tokens = [Named(2), Named(2)]
    roles = {"producer": producer(p, n), "qk": qk_issuer(p, n), "pv": pv_issuer(p, n),
             "wg0": softmax(p, n, 0, tokens), "wg1": softmax(p, n, 1, tokens)}
    blocked = {k: None for k in roles}
    seen_gen = {}
    alive = dict.fromkeys(roles)                 # insertion order: the same every run
    idle = 0
    # Each role is slow to look by its own random amount in this run.
    slow = {k: p.rng.uniform(0.0, 0.9) for k in roles}
    for _ in range(400000):
        if not alive:
            return None
        moved = p.progress()
        for k in list(alive):
            if p.rng.random() < slow[k]:
                continue                         # this role is slow to look this time
            if blocked[k] is None:
                moved = True                     # the role ran up to its next wait
                try:
                    blocked[k] = next(roles[k])
                except StopIteration:
                    del alive[k]
                    continue
                if blocked[k][0] == "sync":
                    seen_gen[k] = blocked[k][1].gen
                    blocked[k][1].arrive()
            op = blocked[k]
            if op[0] == "wait":
                _, bar, parity, idx = op
                if p.B[bar].passes(parity):
                    if p.B[bar].done <= idx:
                        return f"{k}: {bar} passed parity {parity} before completion {idx}"
                    blocked[k], moved = None, True
            elif op[1].gen > seen_gen[k]:
                blocked[k], moved = None, True
        idle = 0 if (moved or p.tma or any(p.mma.values())) else idle + 1
        if idle > 200:                           # every role had many turns: stuck
            return "deadlock: " + ", ".join(f"{k} at {blocked[k][:2]}" for k in sorted(alive))
    return "no progress bound"


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 6, 7, 8, 13, 32, 49, 113])
@pytest.mark.parametrize("rescale", [0.0, 0.3, 1.0])
def test_protocol_drains_in_every_interleaving(n, rescale):
    for seed in range(40):
        assert simulate(n, seed, rescale=rescale) is None, \
            (n, seed, simulate(n, seed, rescale=rescale))


def test_model_catches_a_barrier_per_warpgroup():
    faults = [simulate(32, seed, per_warpgroup_s=True) for seed in range(200)]
    assert sum(f is not None for f in faults) >= 5     # 16 of these 200 interleavings stop
