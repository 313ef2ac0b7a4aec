"""CPU model of the fused tensor-core kernel's barrier protocol (spectral_tc.cu).

The kernel's roles in the two CTAs of a pair synchronise only through
mbarriers, and every wait is on a phase parity.  This test restates each role's
waits (with the parities the kernel uses) and arrivals, runs the roles as
coroutines under random interleavings, with the TMA copies and the tensor pipe
as asynchronous agents, and checks two things:

- every run finishes (a wrong parity, count or missing arrival deadlocks the
  model);
- nothing reads data that is not there yet or is already overwritten: an MMA
  issues only on block pairs of A that both CTAs have transformed for its tile
  and on a weight slot that holds its stage; a block pair is reloaded only once
  every chunk's MMAs on it have completed, and transformed only once its x has
  landed; a slot is refilled only once no MMA reads it; an accumulator buffer
  is read only after its chunk's MMAs completed and rewritten only after every
  epilogue warp of both CTAs (and the transform warps that share the epilogue)
  has read it.

Roles, as in the kernel:

- producer warp (each CTA): lane k owns weight-ring slot k and loads stages
  k, k + S, ... in lockstep iterations (the warp moves on once every lane is
  done); a lane whose released stage belonged to a tile's last chunk loads the
  next tile's x for that stage's block pairs;
- issuer (leader CTA): per chunk waits for its accumulator buffer to be free,
  per stage (a tile's first chunk) for the stage's block pairs in both CTAs
  and for the stage's weights, issues, commits the slot's release to both
  CTAs, and after the chunk commits the accumulator to both CTAs;
- transform warps (10 per CTA, five two-warp groups): each group transforms
  its block pairs as they land and reports each to the leader (the leader's
  warps with a CTA-scope release, the peer's with a cluster-scope one: the
  counts are the same);
- epilogue warps (8 per CTA): per chunk, wait for the accumulator, read it,
  report it free to the leader.  In the cyclic modes they also transform block
  pairs 5..8 of the first tile at once and of the next tile before a tile's
  last chunk; in the D8 and negacyclic modes transform warps 0..7 share the
  epilogue instead and transform the next tile before their share of a tile's
  last chunk.
"""

import random

import pytest

DFT_GROUPS = 5          # kDftGroups
EPI_HELP_GROUPS = 4     # kEpiHelpGroups
WARPS_PER_GROUP = 2     # kDftWarpsPerGroup
N_DFT = 10              # kNumDftWarps
N_EPI = 8               # kNumEpiWarps
N_THELP = 8             # kD8HelpWarps


class Barrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


def pair_by_epilogue(jp, epi_help):
    return epi_help and DFT_GROUPS <= jp < DFT_GROUPS + EPI_HELP_GROUPS


def pair_group(jp, epi_help):
    if not epi_help:
        return jp % DFT_GROUPS
    if jp < DFT_GROUPS:
        return jp
    return jp - DFT_GROUPS if pair_by_epilogue(jp, epi_help) else (jp - EPI_HELP_GROUPS) % DFT_GROUPS


def model(nstage, ks_full, ks_last, nchunks, nslots, ntile, help_mode, seed, bug=None):
    """help_mode: "epi" (epilogue warps transform, cyclic and p4 modes) or "tf"
    (transform warps share the epilogue, D8 and negacyclic modes).  Returns
    (finished, races)."""
    rnd = random.Random(seed)
    epi_help = help_mode == "epi"
    tf_help = help_mode == "tf"
    n_epi_arrivals = N_EPI + (N_THELP if tf_help else 0)
    ns_full, ns_last = nstage // ks_full, nstage // ks_last
    lead = (nchunks - 1) * ns_full
    per_tile = lead + ns_last
    total = ntile * per_tile
    total_chunks = ntile * nchunks
    races = []

    cta = [dict(x_full=[Barrier(1) for _ in range(nstage)],
                a_full=[Barrier(2 * WARPS_PER_GROUP) for _ in range(nstage)],
                b_full=[Barrier(1 + 2) for _ in range(nslots)],      # leader's expect_tx + both halves
                b_empty=[Barrier(1) for _ in range(nslots)],
                acc_full=[Barrier(1) for _ in range(2)],
                acc_empty=[Barrier(2 * n_epi_arrivals) for _ in range(2)]) for _ in range(2)]
    leader = cta[0]
    # data state
    a_state = [[("none", -1)] * nstage for _ in range(2)]       # per CTA, block pair: (state, tile)
    a_rows = [dict() for _ in range(2)]                          # (jp, tile) -> transforming warps done
    mma_reads = {}                                              # (r, jp) -> in-flight MMAs reading it
    slot_reads = {}                                             # (r, k) -> in-flight MMAs reading it
    slot_holds = [[None] * nslots for _ in range(2)]            # stage whose weights landed
    chunk_mmas_issued = {}                                      # (jp, tile) -> chunks issued on it
    acc_chunk = [None, None]                                    # chunk whose products a buffer holds
    acc_done = {}                                               # chunk -> MMAs all complete
    epi_reads = {}                                              # chunk -> epilogue warps done
    tma = []                                                    # pending copies: callables
    pipe = []                                                   # in-order tensor pipe: callables

    def wait(bar, parity):
        while not bar.passed(parity):
            yield

    def stage_info(st):
        tl, rem = divmod(st, per_tile)
        c = rem // ns_full if rem < lead else nchunks - 1
        return tl, c, rem - c * ns_full

    def load_x(r, ti, jp):
        if mma_reads.get((r, jp), 0) or (ti > 0 and chunk_mmas_issued.get((jp, ti - 1), 0) != nchunks):
            races.append(("x reload over live A", r, ti, jp))
        a_state[r][jp] = ("loading", ti)

        def land():
            a_state[r][jp] = ("landed", ti)
            cta[r]["x_full"][jp].arrive()
        tma.append(land)

    def producer(r):
        if ntile > 0:
            for jp in range(nstage):
                load_x(r, 0, jp)
        ph = 0
        it = 0
        while True:
            work = {}
            for lane in range(nslots):
                st = lane + it * nslots
                has_cur, has_prev = st < total, 0 <= st - nslots < total
                if has_cur or has_prev:
                    work[lane] = (st, has_cur, has_prev)
            if not work:
                return
            while work:
                lane = rnd.choice(list(work))
                st, has_cur, has_prev = work[lane]
                par = ph if bug == "b_empty_parity" else ph ^ 1
                if not cta[r]["b_empty"][lane].passed(par):
                    yield
                    continue
                del work[lane]
                if has_cur:
                    if slot_reads.get((r, lane), 0):
                        races.append(("weights over a slot in use", r, lane))
                    slot_holds[r][lane] = None
                    if r == 0:
                        leader["b_full"][lane].arrive()               # arrive.expect_tx

                    def land_w(r=r, lane=lane, st=st):
                        slot_holds[r][lane] = st
                        leader["b_full"][lane].arrive()               # complete_tx of this CTA's half
                    tma.append(land_w)
                if has_prev:
                    ptl, pc, ps = stage_info(st - nslots)
                    if pc == nchunks - 1 and ptl + 1 < ntile and bug != "no_reload":
                        for q in range(ks_last):
                            load_x(r, ptl + 1, ps * ks_last + q)
                yield
            ph ^= 1
            it += 1

    def issuer():
        k = ph = 0
        st = 0
        for g in range(total_chunks):
            ti, c = divmod(g, nchunks)
            buf = g & 1
            par = ((g >> 1) & 1) if bug == "acc_empty_parity" else ((g >> 1) & 1) ^ 1
            yield from wait(leader["acc_empty"][buf], par)
            if g >= 2 and epi_reads.get(g - 2, 0) != 2 * n_epi_arrivals:
                races.append(("accumulator rewritten before it was read", g))
            last = c == nchunks - 1
            ks, ns = (ks_last, ns_last) if last else (ks_full, ns_full)
            for s in range(ns):
                pairs = list(range(s * ks, s * ks + ks))
                if c == 0 and bug != "skip_a_full":
                    for jp in pairs:
                        yield from wait(leader["a_full"][jp], ti & 1)
                yield from wait(leader["b_full"][k], ph)
                for r in range(2):
                    for jp in pairs:
                        if a_state[r][jp] != ("transformed", ti):
                            races.append(("MMA on untransformed A", r, ti, jp, a_state[r][jp]))
                    if slot_holds[r][k] != st:
                        races.append(("MMA on a slot without its stage", r, k, st))
                for jp in pairs:
                    chunk_mmas_issued[(jp, ti)] = chunk_mmas_issued.get((jp, ti), 0) + 1
                    for r in range(2):
                        mma_reads[(r, jp)] = mma_reads.get((r, jp), 0) + 1
                for r in range(2):
                    slot_reads[(r, k)] = slot_reads.get((r, k), 0) + 1
                acc_chunk[buf] = g

                def done_stage(pairs=pairs, k=k):
                    for jp in pairs:
                        for r in range(2):
                            mma_reads[(r, jp)] -= 1
                    for r in range(2):
                        slot_reads[(r, k)] -= 1
                        cta[r]["b_empty"][k].arrive()                 # commit, multicast
                pipe.append(done_stage)
                st += 1
                k += 1
                if k == nslots:
                    k, ph = 0, ph ^ 1

            def done_chunk(g=g, buf=buf):
                acc_done[g] = True
                for r in range(2):
                    cta[r]["acc_full"][buf].arrive()
            pipe.append(done_chunk)
            yield

    def transform(r, jp, ti):
        if a_state[r][jp] != ("landed", ti) and a_state[r][jp] != ("transformed", ti):
            races.append(("transform before x landed", r, ti, jp, a_state[r][jp]))
        key = (jp, ti)
        a_rows[r][key] = a_rows[r].get(key, 0) + 1
        if a_rows[r][key] == WARPS_PER_GROUP:
            a_state[r][jp] = ("transformed", ti)

    def epilogue_read(r, g):
        if not acc_done.get(g) or acc_chunk[g & 1] != g:
            races.append(("epilogue read before its chunk completed", r, g))

    def transform_tile(r, grp, ti):
        for jp in range(grp, nstage):
            if pair_by_epilogue(jp, epi_help) or pair_group(jp, epi_help) != grp:
                continue
            yield from wait(cta[r]["x_full"][jp], ti & 1)
            yield
            transform(r, jp, ti)
            leader["a_full"][jp].arrive()

    def transform_warp(r, w):
        grp = w // WARPS_PER_GROUP
        if tf_help:
            helper = w < N_THELP
            if ntile:
                yield from transform_tile(r, grp, 0)
            for g in range(total_chunks):
                ti, c = divmod(g, nchunks)
                if c == nchunks - 1 and ti + 1 < ntile:
                    yield from transform_tile(r, grp, ti + 1)
                if not helper:
                    continue
                yield from wait(cta[r]["acc_full"][g & 1], (g >> 1) & 1)
                epilogue_read(r, g)
                yield
                epi_reads[g] = epi_reads.get(g, 0) + 1
                leader["acc_empty"][g & 1].arrive()
        else:
            for ti in range(ntile):
                yield from transform_tile(r, grp, ti)

    def help_transform(r, hgrp, ti):
        jp = DFT_GROUPS + hgrp
        while jp < nstage and pair_by_epilogue(jp, epi_help):
            yield from wait(cta[r]["x_full"][jp], ti & 1)
            yield
            transform(r, jp, ti)
            leader["a_full"][jp].arrive()
            jp += EPI_HELP_GROUPS

    def epilogue_warp(r, e):
        hgrp = e // WARPS_PER_GROUP
        for g in range(total_chunks):
            if epi_help:
                last_c = g % nchunks == nchunks - 1
                h0 = 0 if g == 0 else (g // nchunks + 1 if last_c else ntile)
                h1 = g // nchunks + 1 if last_c else 0
                if bug == "help_first_only":
                    h1 = 0 if g == 0 else h1
                hti = h0
                while hti <= h1 and hti < ntile:
                    yield from help_transform(r, hgrp, hti)
                    hti += 1
            yield from wait(cta[r]["acc_full"][g & 1], (g >> 1) & 1)
            epilogue_read(r, g)
            yield
            epi_reads[g] = epi_reads.get(g, 0) + 1
            leader["acc_empty"][g & 1].arrive()

    def agents():
        while True:
            if tma and rnd.random() < 0.5:
                tma.pop(rnd.randrange(len(tma)))()                  # copies land in any order
            if pipe and rnd.random() < 0.5:
                pipe.pop(0)()                                       # the tensor pipe is in order
            yield

    roles = [producer(0), producer(1), issuer()]
    roles += [transform_warp(r, w) for r in range(2) for w in range(N_DFT)]
    roles += [epilogue_warp(r, e) for r in range(2) for e in range(N_EPI)]
    live = list(roles)
    agent = agents()
    steps = 0
    while live:
        if rnd.random() < 0.3:
            next(agent)
        else:
            g = rnd.choice(live)
            try:
                next(g)
            except StopIteration:
                live.remove(g)
        steps += 1
        if steps > 400000:
            return False, races
    return True, races


# (block pairs per chunk, K-slices per stage of full / last chunks, chunks per tile, ring slots)
SHAPES = [
    (10, 2, 2, 3, 4),     # 160 -> 160 fields (config 4): a narrow last chunk
    (10, 2, 2, 10, 4),    # 160 -> 640 fields
    (6, 2, 2, 6, 6),      # 96 -> 384 fields (each C_16 pass)
    (4, 2, 2, 1, 8),      # 64 -> 64 fields: one chunk per tile
    (2, 2, 1, 2, 8),      # 32 -> 96 fields
    (10, 2, 2, 1, 4),     # 160 -> 32 fields: one chunk per tile, every help pair
    (8, 2, 4, 2, 3),      # a narrow last chunk with wider stages, few slots
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("help_mode", ["epi", "tf"])
def test_every_interleaving_finishes_without_a_race(shape, help_mode):
    nstage, ks_full, ks_last, nchunks, nslots = shape
    for ntile in (1, 2, 3):
        for seed in range(4):
            ok, races = model(nstage, ks_full, ks_last, nchunks, nslots, ntile, help_mode, seed)
            assert ok, (shape, help_mode, ntile, seed, "deadlock")
            assert not races, (shape, help_mode, ntile, seed, races[:3])


@pytest.mark.parametrize("bug", ["b_empty_parity", "acc_empty_parity", "skip_a_full", "no_reload",
                                 "help_first_only"])
def test_planted_protocol_mistakes_are_caught(bug):
    """The model can fail: each planted mistake (a wait on the wrong parity, a
    skipped wait, a missing reload or help round) deadlocks it or shows a race."""
    caught = False
    for seed in range(6):
        ok, races = model(10, 2, 2, 1 if bug == "help_first_only" else 3, 4, 3, "epi", seed, bug=bug)
        if not ok or races:
            caught = True
            break
    assert caught, bug
