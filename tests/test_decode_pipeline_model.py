"""Model check of the batched W4A16 decode kernel's pipeline (csrc/k_w4a16_dec.cu), on CPU.

One CTA's roles are restated as the sequence of waits, arrivals and copies that the
kernel performs, with the same ring indices, phase parities and barrier counts:

* producer warp, per tile of its range:
  - all lanes wait empty[slot];
  - lane 0 expects the tile's code bytes on full[slot] and issues the bulk copy;
  - every lane issues its part of the tile's header (scales, zero words) by
    cp.async, then an arrival that fires once those copies have landed (full
    counts 1 + lanes);
* consumer warps, per tile:
  - wait full[slot];
  - per 16-row sub-tile, wait rempty[r], write their partial sums into hand-over
    buffer r and arrive rfull[r];
  - after the tile, arrive empty[slot];
* epilogue warp, per sub-tile: waits rfull[r], reads buffer r, writes y and
  arrives rempty[r].

The bulk copy and each lane's header arrival complete asynchronously, in any
order.  A random scheduler interleaves the roles.  The checks:
- nothing deadlocks;
- no barrier completes a second phase past the one a waiter still waits for;
- a slot is read only after its whole tile (codes and header) landed, and
  refilled only after every consumer warp is done with it;
- a hand-over buffer is read only after every consumer warp wrote that sub-tile,
  and overwritten only after the epilogue read it.
"""
import random

import pytest

RBUFS = 4


class Bar:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.done = 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending -= 1
        assert self.pending >= 0
        self._maybe_complete()

    def complete_tx(self, n):
        self.tx -= n
        self._maybe_complete()

    def ready(self, j):
        assert self.done <= j + 1, ("waiter fell behind", self.done, j)
        return self.done >= j + 1


def run_cta(subtiles, S, C, lanes, seed, early_empty=False):
    """subtiles: number of 16-row sub-tiles of each tile of this CTA's range."""
    rnd = random.Random(seed)
    T = len(subtiles)
    full = [Bar(1 + lanes) for _ in range(S)]
    empty = [Bar(C) for _ in range(S)]
    rfull = [Bar(C) for _ in range(RBUFS)]
    rempty = [Bar(1) for _ in range(RBUFS)]
    codes = [None] * S                     # tile whose codes a slot holds
    header = [[None] * lanes for _ in range(S)]
    red = [[None] * C for _ in range(RBUFS)]
    written = []
    inflight = []

    def producer():
        for t in range(T):
            slot = t % S
            yield lambda slot=slot, t=t: empty[slot].ready(t // S - 1)
            full[slot].arrive(expect_tx=1)
            inflight.append(("codes", slot, None, t))
            for ln in range(lanes):
                inflight.append(("header", slot, ln, t))

    def consumer(w):
        tc = 0
        for t in range(T):
            slot = t % S
            yield lambda slot=slot, t=t: full[slot].ready(t // S)
            assert codes[slot] == t and all(h == t for h in header[slot]), ("slot read early", w, t, codes[slot], header[slot])
            for sub in range(subtiles[t]):
                r = tc % RBUFS
                yield lambda r=r, tc=tc: rempty[r].ready(tc // RBUFS - 1)
                assert codes[slot] == t, ("slot refilled while read", w, t, codes[slot])
                red[r][w] = (t, sub)
                rfull[r].arrive()
                tc += 1
                if early_empty and sub == 0:
                    empty[slot].arrive()
            if not early_empty:
                empty[slot].arrive()

    def epilogue():
        tc = 0
        for t in range(T):
            for sub in range(subtiles[t]):
                r = tc % RBUFS
                yield lambda r=r, tc=tc: rfull[r].ready(tc // RBUFS)
                assert all(v == (t, sub) for v in red[r]), ("hand-over buffer", r, red[r], (t, sub))
                written.append((t, sub))
                rempty[r].arrive()
                tc += 1

    def copy_step(k):
        kind, slot, ln, t = inflight.pop(k)
        if kind == "codes":
            codes[slot] = t
            full[slot].complete_tx(1)
        else:
            header[slot][ln] = t
            full[slot].arrive()             # the lane's cp.async arrival (no count increment)

    actors = [producer(), epilogue()] + [consumer(w) for w in range(C)]
    waits = [next(a, None) for a in actors]
    steps = 0
    while True:
        runnable = [i for i, wt in enumerate(waits) if wt is not None and wt()]
        choices = [("actor", i) for i in runnable]
        if inflight:
            choices.append(("copy", rnd.randrange(len(inflight))))
        if not choices:
            break
        kind, i = rnd.choice(choices)
        if kind == "actor":
            waits[i] = next(actors[i], None)
        else:
            copy_step(i)
        steps += 1
        assert steps < 10 ** 6
    assert all(wt is None for wt in waits), "deadlock: some role is still waiting"
    assert written == [(t, s) for t in range(T) for s in range(subtiles[t])]


@pytest.mark.parametrize("subtiles", [[1], [1] * 9, [2] * 7, [2, 2, 2, 1], [1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1]])
@pytest.mark.parametrize("S", [2, 3, 4, 6, 8])
def test_decode_pipeline_protocol(subtiles, S):
    for seed in range(8):
        run_cta(subtiles, S, C=3, lanes=2, seed=seed * 7907 + S)


def test_model_detects_an_early_slot_release():
    """Sanity check of the model: a consumer that hands its slot back after its first
    sub-tile (not after the whole tile) lets the producer refill a slot that other
    sub-tiles still read, which the model must catch."""
    caught = False
    for seed in range(300):
        try:
            run_cta([2] * 8, 2, C=3, lanes=2, seed=seed, early_empty=True)
        except AssertionError:
            caught = True
            break
    assert caught
