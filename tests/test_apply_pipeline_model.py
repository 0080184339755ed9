"""Model check of the tensor-core W4A16 apply's pipeline (csrc/k_w4a16_tc.cu), on CPU.

Every role of one CTA is restated as the sequence of waits, arrivals and copies
that the kernel performs, with the same ring indices, phase parities and barrier
counts:

* code loader: for each chunk of TC_QC = 4 slabs, waits q_empty and expects the
  chunk's bytes on q_full, then issues the copy;
* activation loader: for each activation stage of TC_XSPS = 2 slabs, waits
  x_empty and expects the stage's bytes on x_full (one or two slabs: the last
  stage may hold one), then issues one copy per slab;
* dequantising warps: in blocks of TC_PF = 4 slabs, step by step (two slabs):
  - at a chunk's first step, wait q_full and read the step's codes;
  - after the chunk's last step (or the layer's last slab), arrive q_empty;
  - wait a_empty, write their part of the step's A stage, arrive a_full;
* MMA: per step, waits a_full and x_full, issues the step's MMAs, then commits
  x_empty and a_empty, and acc_full after the last step;
* epilogue: waits acc_full and reads the accumulator.

Copies and MMAs complete asynchronously: copies in any order, MMAs and commits in
issue order (a commit arrives once the MMAs issued before it have completed).  A
random scheduler interleaves the roles.  The checks:
- nothing deadlocks;
- no barrier completes a second phase past the one a waiter still waits for (its
  parity wait would read "not yet" again);
- no stage is read before it was written, or overwritten before its readers are done;
- the accumulator is read after the last step's MMAs.
"""
import random

import pytest

TC_QC, TC_XSPS, TC_PF, STEP = 4, 2, 4, 2


class Bar:
    """An mbarrier: `count` arrivals and zero pending transaction bytes complete a
    phase.  ready(j) is true once phase j has completed (j = -1: at once)."""

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


def run_cta(nslab, QS, XS, AS, W, seed, early_release=False):
    rnd = random.Random(seed)
    nchunk = -(-nslab // TC_QC)
    nxst = -(-nslab // TC_XSPS)
    nstep = -(-nslab // STEP)
    q_full = [Bar(1) for _ in range(QS)]
    q_empty = [Bar(W) for _ in range(QS)]
    x_full = [Bar(1) for _ in range(XS)]
    x_empty = [Bar(1) for _ in range(XS)]
    a_full = [Bar(W) for _ in range(AS)]
    a_empty = [Bar(1) for _ in range(AS)]
    acc_full = Bar(1)
    qbuf = [None] * QS                                # chunk held by each code stage
    xbuf = [[None] * TC_XSPS for _ in range(XS)]      # slab held by each activation tile
    abuf = [[None] * W for _ in range(AS)]            # step written by each warp's part
    acc = dict(steps=0)
    inflight, tensor_q = [], []

    def q_loader():
        for c in range(nchunk):
            st = c % QS
            yield lambda st=st, c=c: q_empty[st].ready(c // QS - 1)
            q_full[st].arrive(expect_tx=1)
            inflight.append(("q", st, 0, c))

    def x_loader():
        for t in range(nxst):
            st = t % XS
            cnt = min(TC_XSPS, nslab - t * TC_XSPS)
            yield lambda st=st, t=t: x_empty[st].ready(t // XS - 1)
            x_full[st].arrive(expect_tx=cnt)
            for u in range(cnt):
                inflight.append(("x", st, u, t * TC_XSPS + u))

    def dequant(w):
        qs = qs_ph = 0
        as_ = as_ph = 0
        for i0 in range(0, nslab, TC_PF):
            for s2 in range(TC_PF // STEP):
                ib = i0 + s2 * STEP
                if ib >= nslab:
                    break
                cnt = min(STEP, nslab - ib)
                if (s2 * STEP) % TC_QC == 0:
                    yield lambda qs=qs, ph=qs_ph: q_full[qs].ready(ph)
                for us in range(cnt):               # read the step's codes
                    assert qbuf[qs] == (ib + us) // TC_QC, ("codes read from the wrong chunk", w, ib, qbuf[qs])
                last_of_chunk = ((s2 + 1) * STEP) % TC_QC == 0 or ib + cnt == nslab
                if (last_of_chunk and not early_release) or (early_release and (s2 * STEP) % TC_QC == 0):
                    q_empty[qs].arrive()
                if last_of_chunk:
                    qs += 1
                    if qs == QS:
                        qs, qs_ph = 0, qs_ph + 1
                yield lambda a=as_, ph=as_ph: a_empty[a].ready(ph - 1)
                abuf[as_][w] = ib // STEP
                a_full[as_].arrive()
                as_ += 1
                if as_ == AS:
                    as_, as_ph = 0, as_ph + 1

    def mma():
        as_ = as_ph = xs = xs_ph = 0
        for t in range(nstep):
            yield lambda a=as_, ph=as_ph: a_full[a].ready(ph)
            cnt = min(STEP, nslab - t * STEP)
            for u in range(cnt):
                i = t * STEP + u
                ux = i % TC_XSPS
                if ux == 0:
                    yield lambda x=xs, ph=xs_ph: x_full[x].ready(ph)
                tensor_q.append(("mma", as_, xs, ux, t, i))
                if ux == TC_XSPS - 1 or i == nslab - 1:
                    tensor_q.append(("commit", x_empty, xs))
                    xs += 1
                    if xs == XS:
                        xs, xs_ph = 0, xs_ph + 1
            tensor_q.append(("commit", a_empty, as_))
            as_ += 1
            if as_ == AS:
                as_, as_ph = 0, as_ph + 1
        tensor_q.append(("commit", [acc_full], 0))

    def epilogue():
        yield lambda: acc_full.ready(0)
        assert acc["steps"] == nslab, ("accumulator read before the last MMA", acc)

    def tensor_step():
        op = tensor_q.pop(0)
        if op[0] == "mma":
            _, a_s, x_s, ux, t, i = op
            assert all(v == t for v in abuf[a_s]), ("A stage", a_s, abuf[a_s], t)
            assert xbuf[x_s][ux] == i, ("activation tile", x_s, ux, xbuf[x_s][ux], i)
            acc["steps"] += 1
        else:
            _, bars, k = op
            bars[k].arrive()

    def copy_step(k):
        kind, st, u, tag = inflight.pop(k)
        if kind == "q":
            qbuf[st] = tag
            q_full[st].complete_tx(1)
        else:
            xbuf[st][u] = tag
            x_full[st].complete_tx(1)

    actors = [q_loader(), x_loader(), mma(), epilogue()] + [dequant(w) for w in range(W)]
    waits = [next(a, None) for a in actors]
    steps = 0
    while True:
        runnable = [i for i, wt in enumerate(waits) if wt is not None and wt()]
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
    assert all(wt is None for wt in waits), "deadlock: some role is still waiting"
    assert acc["steps"] == nslab


@pytest.mark.parametrize("nslab", [1, 2, 3, 4, 5, 7, 8, 13, 16])
@pytest.mark.parametrize("rings", [(3, 2, 2), (3, 8, 4), (2, 3, 3), (3, 6, 8), (2, 2, 2)])
def test_apply_pipeline_protocol(nslab, rings):
    QS, XS, AS = rings
    for seed in range(10):
        run_cta(nslab, QS, XS, AS, W=2, seed=seed * 104729 + nslab)


def test_model_detects_an_early_code_release():
    """Sanity check of the model itself: releasing a code chunk after its first step
    (instead of its last) lets the loader overwrite codes the second step still
    reads, which the model must catch."""
    caught = False
    for seed in range(200):
        try:
            run_cta(16, 2, 3, 3, W=2, seed=seed, early_release=True)
        except AssertionError:
            caught = True
            break
    assert caught
