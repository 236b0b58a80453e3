"""Randomised models of the kernels' synchronisation protocols (test infrastructure, CPU).

Each model replays one protocol under random interleavings with the
mbarrier's parity semantics: a wait on parity p of a barrier returns as soon
as the barrier's completed-phase count has the other parity, so a waiter that
runs two phases ahead is let through by an OLD phase.  They check the designs
the kernels follow, not the compiled kernels:

* the decode ring: one producer fills stage n % stages with tile n; the
  consumer warps of owner group n % groups read it.  When the stage count is
  not a multiple of the group count, a consumer can reach tile n's stage while
  the stage still waits for tile n - stages of another group, and the parity
  wait alone would pass on the older phase.  The kernel's guard is a sequence
  word the producer sets to n before it issues tile n, which the consumer
  waits for before the parity wait.
* the prefill MMA / softmax handshake: S blocks are issued ahead of the
  softmax, PV blocks after it, and the softmax waits for "PV done" before it
  rescales O in place or reads it at the end.  With one O-ready barrier a
  wait for PV block j can be satisfied by the phase of block j - 2; the
  kernel alternates two barriers by block parity.
"""

import random


class MBar:
    """An mbarrier: `count` arrivals (plus transaction bytes) complete a phase."""

    def __init__(self, count=1):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0  # completed phases

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        self._maybe_complete()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def try_wait(self, parity):
        return (self.phase & 1) != parity


def decode_ring(stages, groups, warps, ntiles, seed, guard):
    """Returns the list of violations (stale reads, deadlock) of one random schedule."""
    rnd = random.Random(seed)
    full = [MBar(1) for _ in range(stages)]
    empty = [MBar(warps) for _ in range(stages)]
    seq = [-1] * stages
    data = [None] * stages
    inflight = []
    errors = []

    def producer():
        for n in range(ntiles):
            s, k = n % stages, n // stages
            while not empty[s].try_wait((k & 1) ^ 1):
                yield
            seq[s] = n
            full[s].arrive_expect_tx(1)
            inflight.append((s, n))
            yield

    def consumer(g, w):
        for n in range(g, ntiles, groups):
            s, k = n % stages, n // stages
            if guard:
                while seq[s] != n:
                    yield
            while not full[s].try_wait(k & 1):
                yield
            if data[s] != n:
                errors.append(("stale read", g, w, n, data[s]))
            yield
            empty[s].arrive()
            yield

    actors = [producer()] + [consumer(g, w) for g in range(groups) for w in range(warps)]
    alive = list(actors)
    for _ in range(200000):
        if not alive and not inflight:
            return errors
        if inflight and rnd.random() < 0.25:  # a copy lands
            s, n = inflight.pop(rnd.randrange(len(inflight)))
            data[s] = n
            full[s].complete_tx(1)
            continue
        if not alive:
            continue
        a = rnd.choice(alive)
        try:
            next(a)
        except StopIteration:
            alive.remove(a)
    return errors + ["deadlock"]


def prefill_handshake(nb, two_barriers, seed):
    """The MMA issuer and the softmax of one 128-row tile over nb key blocks."""
    rnd = random.Random(seed)
    s_full = [MBar(), MBar()]
    p_full = [MBar(), MBar()]
    o_ready = [MBar(), MBar()] if two_barriers else [MBar()]
    queue = []  # the tensor core runs issued work in order: ("S" | "PV", j) or ("C", barrier)
    done = set()
    errors = []

    def o_wait(j):
        if two_barriers:
            return o_ready[j & 1].try_wait((j >> 1) & 1)
        return o_ready[0].try_wait(j & 1)

    def mma():
        for jb in range(nb + 1):
            if jb < nb:  # S of the next block goes ahead of PV of this one
                queue.append(("S", jb))
                queue.append(("C", s_full[jb & 1]))
            if jb >= 1:
                j = jb - 1
                while not p_full[j & 1].try_wait((j >> 1) & 1):
                    yield
                queue.append(("PV", j))
                queue.append(("C", o_ready[j & 1] if two_barriers else o_ready[0]))
            yield

    def softmax():
        for jb in range(nb):
            while not s_full[jb & 1].try_wait((jb >> 1) & 1):
                yield
            if ("S", jb) not in done:
                errors.append(("S read early", jb))
            if jb > 0 and rnd.random() < 0.3:  # the row max moved: rescale O in place
                while not o_wait(jb - 1):
                    yield
                for j in range(jb):
                    if ("PV", j) not in done:
                        errors.append(("rescale before PV", j, jb))
            p_full[jb & 1].arrive()
            yield
        while not o_wait(nb - 1):
            yield
        for j in range(nb):
            if ("PV", j) not in done:
                errors.append(("epilogue before PV", j))

    alive = [mma(), softmax()]
    for _ in range(100000):
        if not alive and not queue:
            return errors
        if queue and rnd.random() < 0.4:
            op = queue.pop(0)
            if op[0] == "C":
                op[1].arrive()
            else:
                done.add(op)
            continue
        if not alive:
            continue
        a = rnd.choice(alive)
        try:
            next(a)
        except StopIteration:
            alive.remove(a)
    return errors + ["deadlock"]


def test_decode_ring_with_sequence_words_never_reads_a_stale_stage():
    for stages in range(2, 9):
        for groups in (2, 3, 4):  # 2 for 24-row items, 3 for up to 16, 4 for split 8-row items
            for warps in (1, 3):
                for seed in range(12):
                    errs = decode_ring(stages, groups, warps, 40, seed, guard=True)
                    assert not errs, (stages, groups, warps, seed, errs[:3])


def test_decode_ring_parity_alone_can_read_a_stale_stage():
    # whenever the stage count is not a multiple of the group count (5 stages and 2 groups
    # is the 24-row decode item), some schedule lets a parity wait pass on an old phase
    for stages, groups in ((3, 2), (5, 2), (4, 3), (5, 3)):
        bad = sum(1 for seed in range(60) if decode_ring(stages, groups, 3, 40, seed, guard=False))
        assert bad > 0, (stages, groups)
    # with a multiple, a group's consumer has itself consumed the stage's previous tile
    for stages, groups in ((4, 2), (6, 3)):
        assert not any(decode_ring(stages, groups, 3, 40, seed, guard=False) for seed in range(30))


def test_prefill_two_o_ready_barriers_order_every_read_of_o():
    for nb in range(1, 8):
        for seed in range(150):
            errs = prefill_handshake(nb, True, seed)
            assert not errs, (nb, seed, errs[:3])


def test_prefill_one_o_ready_barrier_can_pass_on_an_old_phase():
    bad = sum(1 for nb in range(3, 8) for seed in range(150) if prefill_handshake(nb, False, seed))
    assert bad > 0
