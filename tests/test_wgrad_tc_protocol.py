"""CPU model of the tensor-core weight gradient's barrier protocol.

The kernel's roles (producer, in-place transform warps, MMA issuer, and the
transform warps that also run the epilogue after their share of a unit's last
slot, in both CTAs of a pair) synchronise only through mbarriers: per ring
slot s a full barrier (TMA landed, local), an empty barrier (the MMAs that read
the slot are done; the issuer's commit arrives on both CTAs' copies) and an xf
barrier (the slot is transformed: every transform warp arrives on its own CTA's
copy, and the peer CTA's forwarder warp waits for the peer's copy and then
arrives on the leader's), and per CTA an acc_full barrier (a unit's accumulators are
complete; committed to both CTAs) and the leader's acc_empty barrier (every
epilogue warp of both CTAs has read them).  This test restates each role's
waits (with the parities the kernel uses) and arrivals, runs the roles as
coroutines under random interleavings with mbarrier semantics (a wait on parity
P passes once the phase of parity P has completed; a fresh barrier's previous
phase, parity 1, counts as completed), and requires every run to finish: a
wrong parity, count or missing arrival deadlocks the model, and an issuer
that passes its xf wait before every transform warp of both CTAs is done with
the slot fails it.
"""

import os
import random
import re

import pytest

_SRC = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                         "group_wise_dft_b200", "csrc", "wgrad_tc.cu")).read()


def _const(name):
    m = re.search(r"constexpr int %s = (\d+);" % name, _SRC)
    assert m, name
    return int(m.group(1))


N_STAGES = _const("kWtStages")
N_TF = _const("kWtNumTf")     # transform warps per CTA
N_EPI = _const("kWtNumEpi")   # of which the last N_EPI also run the epilogue


class Barrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0          # phases completed so far

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, "more arrivals than the count"
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        # phase k (parity k & 1) is complete once phase > k; the wait on parity P
        # passes when the most recent phase of parity P has completed, i.e. the
        # current (incomplete) phase's parity differs from P
        return (self.phase & 1) != parity


def model(units_chunks, seed, bug=None):
    """units_chunks: chunks of each of the pair's units, in order.  bug plants
    one protocol mistake (for the test that the model can fail)."""
    rnd = random.Random(seed)
    cta = [dict(full=[Barrier(1) for _ in range(N_STAGES)], empty=[Barrier(1) for _ in range(N_STAGES)],
                xf=[Barrier(N_TF + (1 if r == 0 else 0)) for _ in range(N_STAGES)], acc_full=Barrier(1),
                acc_empty=Barrier(2 * N_EPI)) for r in range(2)]
    leader = cta[0]
    transformed = {}   # slot use q -> transform warps (both CTAs) done with it
    race = []

    def wait(bar, parity):
        while not bar.passed(parity):
            yield

    def producer(r):
        q = 0
        for nch in units_chunks:
            for _ in range(nch):
                s, ph = q % N_STAGES, (q // N_STAGES) & 1
                yield from wait(cta[r]["empty"][s], ph if bug == "empty_parity" else ph ^ 1)
                yield                                   # TMA in flight
                cta[r]["full"][s].arrive()              # complete_tx
                q += 1

    def transform(r, epi):
        q = 0
        for n, nch in enumerate(units_chunks):
            for _ in range(nch):
                s, ph = q % N_STAGES, (q // N_STAGES) & 1
                yield from wait(cta[r]["full"][s], ph)
                yield
                transformed[q] = transformed.get(q, 0) + 1
                if not (bug == "peer_xf_leader" and r == 1):
                    cta[r]["xf"][s].arrive()            # this CTA's own copy
                else:
                    leader["xf"][s].arrive()            # skipping the forwarder: the leader's count overflows
                q += 1
            if epi:                                     # the epilogue of unit n
                yield from wait(cta[r]["acc_full"], n & 1)
                yield                                   # TMEM loads, stores
                leader["acc_empty"].arrive()

    def forwarder():
        q = 0
        for nch in units_chunks:
            for _ in range(nch):
                s, ph = q % N_STAGES, (q // N_STAGES) & 1
                yield from wait(cta[1]["xf"][s], ph ^ 1 if bug == "forward_parity" else ph)
                leader["xf"][s].arrive()                # mapa to the leader, release at cluster scope
                q += 1

    def issuer():
        q = 0
        for n, nch in enumerate(units_chunks):
            yield from wait(leader["acc_empty"], (n & 1) if bug == "acc_empty_parity" else (n & 1) ^ 1)
            for _ in range(nch):
                s, ph = q % N_STAGES, (q // N_STAGES) & 1
                yield from wait(leader["xf"][s], ph)
                if transformed.get(q, 0) != 2 * N_TF:    # the MMAs would read untransformed atoms
                    race.append(q)
                yield                                   # the MMAs
                for c in cta:                           # commit, multicast to both CTAs
                    c["empty"][s].arrive()
                q += 1
            for c in (cta[:1] if bug == "acc_full_leader_only" else cta):
                c["acc_full"].arrive()

    roles = [producer(0), producer(1), issuer(), forwarder()]
    roles += [transform(r, w >= N_TF - N_EPI) for r in range(2) for w in range(N_TF)]
    live = list(roles)
    steps = 0
    while live:
        g = rnd.choice(live)
        try:
            next(g)
        except StopIteration:
            live.remove(g)
        steps += 1
        if steps > 200000:
            return False
    return not race


@pytest.mark.parametrize("units_chunks", [[1], [1, 1, 1], [2, 5, 1], [7], [3, 3, 3, 3], [1, 6, 2, 4, 1]])
def test_every_interleaving_finishes(units_chunks):
    for seed in range(20):
        assert model(units_chunks, seed), (units_chunks, seed)


@pytest.mark.parametrize("bug", ["empty_parity", "acc_empty_parity", "peer_xf_leader", "forward_parity",
                                 "acc_full_leader_only"])
def test_planted_protocol_mistakes_deadlock_the_model(bug):
    """The model can fail: each planted mistake (a wait on the wrong parity, an
    arrival on the wrong CTA's barrier, a commit that skips the peer) hangs it
    or lets the issuer read a slot before it is transformed."""
    assert not model([2, 3, 1], 0, bug=bug)
