"""Host-side model of the grouped GEMM's mbarrier protocol (one CTA).

The persistent GEMM kernel runs five roles that hand ring stages to each other
through mbarriers: the packed-weight producer (W ring), the token-tile loader
(B ring), the transform warps (W ring -> A ring, in groups that take
alternate chunks), the MMA warp (A and B rings -> TMEM accumulators) and the
epilogue warps (accumulators -> memory).  This test replays that protocol as
a discrete-event simulation with random delays, using the ring sizes, group
count and accumulator buffers read from the kernel source, and checks that

  - every role finishes (no deadlock), and
  - every stage read sees the iteration its consumer expects (no role is
    released by a parity wait one phase too early: mbarrier parity waits only
    tell a phase from the one before it).

A configuration that breaks the kernel's static_assert (ring sizes that are
not multiples of the transform group count) is shown to fail the model.
"""
import heapq
import os
import random
import re

import pytest

GEMM_SRC = os.path.join(os.path.dirname(__file__), "..", "int4_expert_grouped_b200", "csrc",
                        "moe_gemm.cu")
TRANSFORM_WARPS = 8
EPILOGUE_WARPS = 4


def kernel_configs():
    """(name, NW, NA, NB, G, acc_bufs) of the two projections in both ring
    variants (large blocks; weight streaming for small blocks), from the source.
    Units of one A tile (down, large blocks) and of two (gate/up; down in the
    streaming variant, where a unit pairs two output tiles) take the kOneTile
    and the other branch of each ring size."""
    src = open(GEMM_SRC).read()
    n = r"(\d+)"

    def find(pattern, name):
        m = re.search(pattern, src)
        assert m, name
        return [int(g) for g in m.groups()]

    nw_s1, nw_s2, nw1, nw2 = find(r"static constexpr int kNW = kStream \? \(kOneTile \? %s : %s\) : "
                                  r"\(kOneTile \? %s : %s\);" % (n, n, n, n), "kNW")
    na_s, na1, na2 = find(r"static constexpr int kNA = kStream \? %s : \(kOneTile \? %s : %s\);"
                          % (n, n, n), "kNA")
    nb_s, nb = find(r"static constexpr int kNB = kStream \? %s : %s;" % (n, n), "kNB")
    acc2, acc1 = find(r"static constexpr int kAccBufs = \(kDown \|\| kStream\) \? %s : %s;" % (n, n),
                      "kAccBufs")  # two buffers for down and for the streaming variant
    g1, g2 = find(r"static constexpr int kGroups = kOneTile \? %s : %s;" % (n, n), "kGroups")
    assert re.search(r"kTiles = \(kDown && !kPair\) \? kDownTiles : 2;", src), "kTiles"
    return [("gate/up", nw2, na2, nb, g2, acc1),
            ("down", nw1, na1, nb, g1, acc2),
            ("gate/up, streaming (half blocks)", nw_s2, na_s, nb_s, g2, acc2),
            ("down, streaming (half blocks, tile pairs)", nw_s2, na_s, nb_s, g2, acc2)]


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than expected in one phase"
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        # try_wait.parity(P) succeeds once the phase with parity P has completed
        return (self.phase & 1) != parity


def simulate(NW, NA, NB, G, acc_bufs, units=5, KC=7, seed=0):
    """Returns (finished, races): finished is False on a deadlock."""
    rng = random.Random(seed)
    wfull = [Barrier(1) for _ in range(NW)]
    wempty = [Barrier(TRANSFORM_WARPS // G) for _ in range(NW)]
    afull = [Barrier(TRANSFORM_WARPS // G) for _ in range(NA)]
    aempty = [Barrier(1) for _ in range(NA)]
    bfull = [Barrier(1) for _ in range(NB)]
    bempty = [Barrier(1) for _ in range(NB)]
    accfull = [Barrier(1) for _ in range(acc_bufs)]
    accempty = [Barrier(EPILOGUE_WARPS) for _ in range(acc_bufs)]
    # iteration held by each stage (what a reader must find there)
    w_slot, a_slot, b_slot = [None] * NW, [None] * NA, [None] * NB
    races = []
    clock = [0.0]
    queue, seq = [], [0]
    total = units * KC

    def later(delay, fn):
        seq[0] += 1
        heapq.heappush(queue, (clock[0] + delay, seq[0], fn))

    def w_producer():
        for it in range(total):
            s = it % NW
            yield wempty[s], ((it // NW) & 1) ^ 1

            def land(s=s, it=it):
                w_slot[s] = it
                wfull[s].arrive()
            later(rng.uniform(1, 30), land)

    def b_loader():
        for it in range(total):
            s = it % NB
            yield bempty[s], ((it // NB) & 1) ^ 1

            def land(s=s, it=it):
                b_slot[s] = it
                bfull[s].arrive()
            later(rng.uniform(1, 30), land)

    def transform_warp(group, member):
        for it in range(total):
            if it % G != group:
                continue
            sw, sa = it % NW, it % NA
            yield wfull[sw], (it // NW) & 1
            yield aempty[sa], ((it // NA) & 1) ^ 1
            if w_slot[sw] != it:
                races.append(("transform reads W", it, w_slot[sw]))
            yield None, rng.uniform(1, 10)  # expanding
            if member == 0:
                a_slot[sa] = it
            afull[sa].arrive()
            wempty[sw].arrive()

    def mma():
        it = 0
        for u in range(units):
            buf, use = u % acc_bufs, u // acc_bufs
            yield accempty[buf], (use & 1) ^ 1
            for _ in range(KC):
                sa, sb = it % NA, it % NB
                yield afull[sa], (it // NA) & 1
                yield bfull[sb], (it // NB) & 1
                if a_slot[sa] != it:
                    races.append(("MMA reads A", it, a_slot[sa]))
                if b_slot[sb] != it:
                    races.append(("MMA reads B", it, b_slot[sb]))
                done = rng.uniform(1, 8)  # the commits fire when the MMAs complete
                later(done, lambda sa=sa: aempty[sa].arrive())
                later(done, lambda sb=sb: bempty[sb].arrive())
                it += 1
            later(rng.uniform(1, 8), lambda buf=buf: accfull[buf].arrive())

    def epilogue_warp():
        for u in range(units):
            buf, use = u % acc_bufs, u // acc_bufs
            yield accfull[buf], use & 1
            yield None, rng.uniform(1, 40)
            accempty[buf].arrive()

    roles = [w_producer(), b_loader(), mma()]
    roles += [transform_warp(g, m) for g in range(G) for m in range(TRANSFORM_WARPS // G)]
    roles += [epilogue_warp() for _ in range(EPILOGUE_WARPS)]
    blocked = {}
    finished = [0]

    def run(i):
        gen = roles[i]
        while True:
            try:
                bar, arg = next(gen)
            except StopIteration:
                finished[0] += 1
                return
            if bar is None:  # work that takes time
                later(arg, lambda i=i: run(i))
                return
            if not bar.passed(arg):
                blocked[i] = (bar, arg)
                return

    for i in range(len(roles)):
        run(i)
    while True:
        progressed = True
        while progressed:
            progressed = False
            for i, (bar, parity) in list(blocked.items()):
                if bar.passed(parity):
                    del blocked[i]
                    run(i)
                    progressed = True
        if not queue:
            break
        clock[0], _, fn = heapq.heappop(queue)
        fn()
    return finished[0] == len(roles), races


@pytest.mark.parametrize("cfg", kernel_configs(), ids=lambda c: c[0])
def test_kernel_ring_configuration_is_sound(cfg):
    name, NW, NA, NB, G, acc = cfg
    assert NW % G == 0 and NA % G == 0, "the kernel's static_assert"
    for seed in range(150):
        finished, races = simulate(NW, NA, NB, G, acc, seed=seed)
        assert finished, (name, "deadlock", seed)
        assert not races, (name, races[:3], seed)


def test_shared_rings_break_the_parity_protocol():
    # four transform groups sharing a two-stage W ring (and a four-stage A
    # ring): a group can run two phases ahead of a stage, which the parity waits
    # cannot tell apart; the model must catch it (deadlock or a stale read)
    bad = 0
    for seed in range(150):
        finished, races = simulate(NW=2, NA=4, NB=3, G=4, acc_bufs=1, seed=seed)
        bad += (not finished) or bool(races)
    assert bad > 0
