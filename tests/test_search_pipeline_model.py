"""Model check of the fused search kernel's CTA-pair pipeline (csrc/k_search.cu),
on CPU.

Every role of the two CTAs of a pair is restated as a sequence of the same
waits, arrivals and copies the kernel performs, with the same ring indices,
phase parities and barrier counts:

* input loader (each CTA): waits in_empty, expects the stage's bytes on its own
  in_full, issues the copy;
* X loader (each CTA): waits its x_empty; the leader expects both halves' bytes
  on its x_full; both CTAs' copies complete on the leader's x_full;
* producer warps (each CTA): wait in_full, read, arrive in_empty, wait a_empty,
  write their part of the dW stage, arrive on the leader's a_full;
* MMA (leader): waits a_full, each accumulator half's acc_empty before a
  unit's first slab writes it, x_full per N half; issues MMAs and commits that
  arrive on x_empty / a_empty / acc_full of both CTAs once the MMAs before them
  have completed;
* epilogue warps (each CTA): wait acc_full per half, read it, arrive on the
  leader's acc_empty.

Copies, MMAs and commits complete asynchronously, in a random order consistent
with the hardware's (a commit after every MMA issued before it).  A random
scheduler interleaves the roles.  The checks: nothing deadlocks; no barrier ever
completes a second phase past the one a waiter still waits for (its parity wait
would read "not yet" again); no stage is overwritten before it has been read, or read before it
was written; every accumulator half is read after its unit's last MMA and
overwritten only after both epilogues have read it.
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals and zero pending transaction bytes complete
    a phase.  wait(j) succeeds once phase j has completed (j = -1: at once)."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.done = 0                       # completed phases

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def arrive(self, expect_tx=0):
        self.tx += expect_tx
        self.pending -= 1
        assert self.pending >= 0
        self._maybe_complete()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def ready(self, j):
        # A parity wait for phase j sees the barrier's current phase parity: once
        # phase j + 1 has also completed it reads "not yet" again, so a waiter
        # still waiting for j must never find more than j + 1 phases done.
        assert self.done <= j + 1, ("waiter fell behind", self.done, j)
        return self.done >= j + 1


def run_pair(units, nK, XS, AS, IS, W, E, seed):
    """units: list of nsub (1 or 2) per work unit of this pair."""
    rnd = random.Random(seed)
    cta = (0, 1)
    bars = {c: dict(x_full=[Bar(1) for _ in range(XS)], x_empty=[Bar(1) for _ in range(XS)],
                    a_full=[Bar(2 * W) for _ in range(AS)], a_empty=[Bar(1) for _ in range(AS)],
                    in_full=[Bar(1) for _ in range(IS)], in_empty=[Bar(W) for _ in range(IS)],
                    acc_full=[Bar(1), Bar(1)], acc_empty=[Bar(2 * E), Bar(2 * E)])
            for c in cta}
    L = bars[0]
    xbuf = {c: [None] * XS for c in cta}           # tag of the data in each stage
    inbuf = {c: [None] * IS for c in cta}
    abuf = {c: [[None] * W for _ in range(AS)] for c in cta}
    acc = {c: [dict(unit=None, final=False, read=set()) for _ in range(2)] for c in cta}
    inflight = []                                    # async copy completions
    tensor_q = []                                    # MMAs and commits, completed in order

    slabs = [(u, kb) for u in range(len(units)) for kb in range(nK)]

    def input_loader(c):
        for it, (u, kb) in enumerate(slabs):
            st = it % IS
            yield lambda st=st, it=it: bars[c]["in_empty"][st].ready(it // IS - 1)
            bars[c]["in_full"][st].arrive(expect_tx=1)
            inflight.append(("in", c, st, (u, kb)))

    def x_loader(c):
        it = 0
        for u, nsub in enumerate(units):
            for kb in range(nK):
                for h in range(nsub):
                    st = it % XS
                    yield lambda st=st, it=it: bars[c]["x_empty"][st].ready(it // XS - 1)
                    if c == 0:
                        L["x_full"][st].arrive(expect_tx=2)
                    inflight.append(("x", c, st, (u, kb, h)))
                    it += 1

    def producer(c, w):
        for it, (u, kb) in enumerate(slabs):
            i_s, a_s = it % IS, it % AS
            yield lambda i_s=i_s, it=it: bars[c]["in_full"][i_s].ready(it // IS)
            assert inbuf[c][i_s] == (u, kb), ("input stage not loaded", c, w, it, inbuf[c][i_s])
            bars[c]["in_empty"][i_s].arrive()
            yield lambda a_s=a_s, it=it: bars[c]["a_empty"][a_s].ready(it // AS - 1)
            abuf[c][a_s][w] = (u, kb)
            L["a_full"][a_s].arrive()

    def mma():
        ait = xit = 0
        hit = [0, 0]
        for u, nsub in enumerate(units):
            for kb in range(nK):
                a_s = ait % AS
                yield lambda a_s=a_s, ait=ait: L["a_full"][a_s].ready(ait // AS)
                for h in range(nsub):
                    if kb == 0:
                        yield lambda h=h: L["acc_empty"][h].ready(hit[h] - 1)
                    xs = xit % XS
                    yield lambda xs=xs, xit=xit: L["x_full"][xs].ready(xit // XS)
                    tensor_q.append(("mma", a_s, xs, (u, kb, h), kb == 0, kb == nK - 1))
                    tensor_q.append(("commit", "x_empty", xs))
                    if kb == nK - 1:
                        tensor_q.append(("commit", "acc_full", h))
                    xit += 1
                tensor_q.append(("commit", "a_empty", a_s))
                ait += 1
            for h in range(nsub):
                hit[h] += 1

    def epilogue(c, e):
        hit = [0, 0]
        for u, nsub in enumerate(units):
            for h in range(nsub):
                yield lambda h=h: bars[c]["acc_full"][h].ready(hit[h])
                a = acc[c][h]
                assert a["unit"] == u and a["final"], ("accumulator read early", c, u, h, a)
                a["read"].add((c, e))
                L["acc_empty"][h].arrive()
                hit[h] += 1

    def tensor_step():
        op = tensor_q.pop(0)
        if op[0] == "mma":
            _, a_s, xs, (u, kb, h), first, last = op
            for c in cta:
                assert all(t == (u, kb) for t in abuf[c][a_s]), ("dW stage", c, a_s, abuf[c][a_s], (u, kb))
                assert xbuf[c][xs] == (u, kb, h), ("X stage", c, xs, xbuf[c][xs], (u, kb, h))
                a = acc[c][h]
                if first:
                    # overwriting: the previous unit in this half must have been read by
                    # every epilogue warp of this CTA (each CTA's TMEM holds its own rows)
                    assert a["unit"] is None or len(a["read"]) == E, ("accumulator overwritten", c, h, a)
                    acc[c][h] = dict(unit=u, final=last, read=set())
                else:
                    assert a["unit"] == u and not a["final"]
                    a["final"] = last
        else:
            _, name, idx = op
            for c in cta:
                bars[c][name][idx].arrive()

    def copy_step(k):
        kind, c, st, tag = inflight.pop(k)
        if kind == "in":
            inbuf[c][st] = tag
            bars[c]["in_full"][st].complete_tx(1)
        else:
            xbuf[c][st] = tag
            L["x_full"][st].complete_tx(1)

    actors = ([input_loader(c) for c in cta] + [x_loader(c) for c in cta]
              + [producer(c, w) for c in cta for w in range(W)] + [mma()]
              + [epilogue(c, e) for c in cta for e in range(E)])
    waits = [next(a, None) for a in actors]
    steps = 0
    while True:
        runnable = [i for i, w in enumerate(waits) if w is not None and w()]
        choices = [("actor", i) for i in runnable]
        if inflight:
            choices.append(("copy", rnd.randrange(len(inflight))))
        if tensor_q:
            choices.append(("tensor", 0))
        if not choices:
            break
        kind, i = rnd.choice(choices)
        if kind == "actor":
            waits[i] = next(actors[i], None)
        elif kind == "copy":
            copy_step(i)
        else:
            tensor_step()
        steps += 1
        assert steps < 10 ** 6
    assert all(w is None for w in waits), "deadlock: some role is still waiting"
    # the last unit's partials were read by every epilogue warp of each CTA
    for c in cta:
        for h in range(2):
            a = acc[c][h]
            assert a["unit"] is None or len(a["read"]) == E


UNIT_MIXES = [[2, 2, 2], [1], [2, 1, 2, 1], [1, 1, 2], [2] * 5]


@pytest.mark.parametrize("nK", [1, 2, 3])
@pytest.mark.parametrize("units", UNIT_MIXES)
@pytest.mark.parametrize("rings", [(6, 3, 3), (6, 3, 2), (8, 2, 3), (2, 1, 1), (4, 2, 2)])
def test_pair_pipeline_protocol(nK, units, rings):
    XS, AS, IS = rings
    for seed in range(8):
        run_pair(units, nK, XS, AS, IS, W=2, E=2, seed=seed * 7919 + nK)


def test_model_detects_a_broken_protocol():
    """Sanity check of the model itself: handing a half back before both CTAs'
    epilogues have read it must be caught (here: the leader's acc_empty counts
    one arrival instead of 2 CTAs x E warps, so the MMA may overwrite a half a
    warp of either CTA has not read yet)."""
    caught = False
    orig = Bar.__init__
    try:
        def low_count(self, count):
            orig(self, 1 if count == 4 else count)   # acc_empty of 2 CTAs x E = 2 warps
        Bar.__init__ = low_count
        for seed in range(50):
            try:
                run_pair([2, 2, 2, 2], 2, 6, 3, 3, W=2, E=2, seed=seed)
            except AssertionError:
                caught = True
                break
    finally:
        Bar.__init__ = orig
    assert caught
