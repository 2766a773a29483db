"""A host model of the decode index scan's stage ring (no GPU).

The streaming scan has one producer lane and eight consumer warps; item k goes to
stage k % S and to consumer warp k % 8.  The producer waits (mbarrier parity) for
a stage's previous item to be consumed before loading the next one into it; a
consumer waits (parity) for its item's copy to land, reads the stage, then
arrives on the stage's "empty" barrier.  A parity wait only tells the current
phase of a barrier from the one before it, so it is sound only if no waiter can
be two phases ahead.  The kernel therefore takes S as a multiple of the warp
count: every stage is then consumed by a single warp, which has itself consumed
the stage's previous fill before it waits on the next.

The model below reproduces the barrier semantics (arrival counts, transaction
bytes, phase parity), lets the producer, the copy engine and the consumers act in
random order with copies landing out of order, and checks that no consumer ever
reads a stage holding another item and that no arrive falls on a phase with no
pending arrival.  It passes for S = 8 and 16 (what the kernel uses) and must
fail for stage counts that share stages between warps.
"""

import random

import pytest

NW = 8  # consumer warps of the streaming scan


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.completed = count, count, 0, 0

    def parity_done(self, parity):
        # the phase with this parity has completed iff the current one has the other parity
        return (self.completed & 1) != parity

    def arrive(self, tx=0):
        if self.pending <= 0:
            raise AssertionError("arrive on a phase with no pending arrival")
        self.tx += tx
        self.pending -= 1
        self._maybe_complete()

    def land(self, tx):
        self.tx -= tx
        if self.tx < 0:
            raise AssertionError("transaction count below zero")
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count


def run_ring(S, n_items, seed):
    rng = random.Random(seed)
    full = [Barrier(1) for _ in range(S)]
    empty = [Barrier(1) for _ in range(S)]
    data = [None] * S  # item whose copy has landed in each stage
    in_flight = []
    produced, done = 0, 0
    nxt = list(range(NW))  # next item of each consumer warp
    busy = [None] * NW
    while done < n_items:
        acts = []
        if produced < n_items:
            s = produced % S
            if produced < S or empty[s].parity_done(((produced // S) - 1) & 1):
                acts.append(("produce", None))
        if in_flight:
            acts.append(("land", None))
        for w in range(NW):
            if busy[w] is not None:
                acts.append(("release", w))
            elif nxt[w] < n_items and full[nxt[w] % S].parity_done((nxt[w] // S) & 1):
                acts.append(("consume", w))
        if not acts:
            raise AssertionError("no actor can move")
        kind, w = rng.choice(acts)
        if kind == "produce":
            s = produced % S
            full[s].arrive(tx=1)
            in_flight.append((s, produced))
            produced += 1
        elif kind == "land":
            s, k = in_flight.pop(rng.randrange(len(in_flight)))
            data[s] = k
            full[s].land(1)
        elif kind == "consume":
            k = nxt[w]
            if data[k % S] != k:
                raise AssertionError("warp %d read stage %d for item %d, it holds %s"
                                     % (w, k % S, k, data[k % S]))
            busy[w] = k
        else:
            k = busy[w]
            if data[k % S] != k:
                raise AssertionError("stage %d refilled while item %d was read" % (k % S, k))
            empty[k % S].arrive()
            busy[w] = None
            nxt[w] += NW
            done += 1


@pytest.mark.parametrize("S", [8, 16])
def test_stage_count_multiple_of_warps_is_safe(S):
    for seed in range(60):
        run_ring(S, 5 * S + 3, seed)


@pytest.mark.parametrize("S", [4, 12, 14])
def test_shared_stages_break_the_parity_wait(S):
    broken = 0
    for seed in range(60):
        try:
            run_ring(S, 5 * S + 3, seed)
        except AssertionError:
            broken += 1
    assert broken > 0, "the model should catch a stage shared between warps"
