"""Host-side checks of the GPU kernels' work decomposition (no GPU needed).

These restate, in Python, the index arithmetic that the CUDA kernels perform,
and check the invariants the kernels rely on:

* W4A16 decode GEMV (csrc/k_w4a16_stream.cu): one CTA per SM over a contiguous
  row range, warp w taking rows w, w + NW, ...; each lane streams its 16-byte
  code groups, the Delta of their group and the zero word holding it by fixed
  pointer steps.  Every (row, 32-column chunk) must be loaded exactly once, by
  an in-bounds address equal to the direct index, and the lane's zero nibble
  must be the group's.
* W4A16 batched decode (csrc/k_w4a16_dec.cu): tiles of 8 rows weighing in / 64
  units over a list of linears; CTA c owns the tiles whose first unit is in
  [c U / P, (c + 1) U / P).  Every tile must be owned by exactly one CTA, the
  tiles a CTA walks must be consecutive, and no CTA may stream much more than
  its share; the staged activations must land in distinct, in-bounds 16-byte
  slots whose four fragment-thread reads of a token are one contiguous span.
* Tensor-core apply (csrc/k_w4a16_tc.cu): the plan's CTAs must cover every
  (row tile, token tile, slab) exactly once with no empty K split; the ring
  depths and TMEM columns a launch asks for must fit one or two CTAs per SM as
  intended; and the code chunks (128-byte swizzle) must be read unit by unit,
  once, without bank conflicts within a quarter warp.
* Fused search (csrc/k_search.cu): CTA pairs deal work units (grid point, 256-row
  pair tile, 512-token block) round-robin; every (grid point, row, token block)
  partial must be written exactly once.

The kernels themselves are checked against the oracle by the GPU parity tests;
these tests pin the decomposition for shapes those tests do not reach
(hundreds of SMs' worth of rows, ragged tails, every group size).
"""
import itertools

import pytest


def gemv_lane_streams(O, I, gs, sms, NW, RING):
    """Loads issued by the GEMV kernel: {(row, chunk): count}, checking every
    address against its direct index on the way."""
    lgs = {32: 5, 64: 6, 128: 7}[gs]
    nch = I // 32
    NBL = (nch + 31) // 32
    nG = I >> lgs
    nzw = (nG + 7) >> 3
    rpc = max(1, -(-O // sms))
    grid = -(-O // rpc)
    seen = {}
    for b in range(grid):
        row0 = b * rpc
        nrows = min(O - row0, rpc)
        for warp in range(NW):
            myrows = (nrows - warp + NW - 1) // NW if warp < nrows else 0
            ntot = myrows * NBL
            for lane in range(32):
                g0 = (lane * 32) >> lgs
                gstep = 1024 >> lgs
                r0 = row0 + warp
                qp = r0 * (I // 32) + lane
                sp = r0 * nG + g0
                zp = r0 * nzw + (g0 >> 3)
                qrow = NW * (I // 32) - NBL * 32
                srow = NW * nG - NBL * gstep
                zrow = NW * nzw - NBL * (gstep >> 3)
                tail_ok = lane < nch - 32 * (NBL - 1)
                zsh = 4 * (g0 & 7)
                ij = nis = 0

                def issue():
                    nonlocal qp, sp, zp, ij, nis
                    if nis < ntot and (ij < NBL - 1 or tail_ok):
                        row = r0 + NW * (nis // NBL)
                        t = lane + 32 * (nis % NBL)
                        assert row < row0 + nrows and t < nch
                        assert qp == row * (I // 32) + t
                        g = (t * 32) // gs
                        assert sp == row * nG + g and g < nG
                        assert zp == row * nzw + g // 8 and zsh == 4 * (g % 8)
                        seen[(row, t)] = seen.get((row, t), 0) + 1
                    nis += 1
                    qp += 32
                    sp += gstep
                    zp += gstep >> 3
                    ij += 1
                    if ij == NBL:
                        ij = 0
                        qp += qrow
                        sp += srow
                        zp += zrow

                for _ in range(RING):          # prologue
                    issue()
                for base in range(0, ntot, RING):
                    for s in range(RING):
                        if base + s >= ntot:
                            break
                        if base + s + RING < ntot:
                            issue()            # refill; skipped past the warp's end
    return seen, nch


SHAPES = [(4096, 4096, 128), (11008, 4096, 128), (4096, 11008, 128), (300, 1152, 128),
          (301, 1088, 64), (77, 1088, 32), (130, 2112, 32), (1, 64, 32), (5, 128, 64),
          (2369, 192, 64), (150, 11008, 32)]


@pytest.mark.parametrize("O,I,gs", SHAPES)
@pytest.mark.parametrize("NW,RING", [(32, 3), (16, 8)])
def test_gemv_streams_cover_every_chunk_once(O, I, gs, NW, RING):
    seen, nch = gemv_lane_streams(O, I, gs, 148, NW, RING)
    assert len(seen) == O * nch
    assert set(seen.values()) == {1}


def gemv_staging_table(I, MT):
    """Shared activation table of the GEMV: 16-byte slot index of every
    (chunk, token, slot) and the lanes' load addresses."""
    S = MT * 5 if (MT * 5) % 2 else MT * 5 + 1
    nch = I // 32
    ncp = ((nch + 31) // 32) * 32
    return S, nch, ncp


@pytest.mark.parametrize("MT", [1, 2, 4])
def test_gemv_activation_table_conflict_free(MT):
    """Per chunk, S slots of 16 bytes with S odd: the 8 lanes of one phase of a
    128-bit shared load (consecutive chunks) hit 8 distinct 16-byte bank groups."""
    S, _, _ = gemv_staging_table(4096, MT)
    assert S % 2 == 1 and S >= 5 * MT
    for phase in range(4):
        for slot in range(5 * MT):
            groups = {((phase * 8 + l) * S + slot) % 8 for l in range(8)}
            assert len(groups) == 8


SEARCH_TILE_N, SEARCH_SUB_N = 512, 256     # tokens per unit, per MMA (two halves per unit)


def search_units(O, N, G, pairs):
    """Partials the pair search kernel writes: {(g, tb, row): count}."""
    TILE_O, PAIR_O, TILE_N = 128, 256, SEARCH_TILE_N
    OT = -(-O // PAIR_O)
    TB = -(-N // TILE_N)
    U = OT * TB * G
    out = {}
    for cid in range(min(U, pairs)):
        for u in range(cid, U, min(U, pairs)):
            g = u % G
            rest = u // G
            ot, tb = rest % OT, rest // OT
            for rank in (0, 1):
                for r in range(TILE_O):
                    row = ot * PAIR_O + rank * TILE_O + r
                    if row < O:
                        key = (g, tb, row)
                        out[key] = out.get(key, 0) + 1
    return out, TB


@pytest.mark.parametrize("O,N,G", [(4096, 4096, 20), (300, 513, 11), (16, 2048, 3), (200, 700, 20),
                                   (22016, 8192, 20), (129, 100, 4)])
def test_search_pairs_write_every_partial_once(O, N, G):
    out, TB = search_units(O, N, G, 74)
    assert len(out) == G * TB * O
    assert set(out.values()) == {1}
    # the unit count per pair differs by at most one (balanced round-robin)
    U = -(-O // 256) * TB * G
    p = min(U, 74)
    per = [len(range(c, U, p)) for c in range(p)]
    assert max(per) - min(per) <= 1


@pytest.mark.parametrize("N", [1, 128, 129, 256, 257, 511, 512, 513, 4096, 65536 + 77])
def test_search_token_halves_cover_each_token_once(N):
    """Each unit of 512 tokens runs one or two MMA halves of 256 (two when more
    than 256 tokens are left); each CTA of the pair stages 128 tokens of a half.
    Every token below N is staged exactly once; staged rows past N are the
    zero-filled tail of the last box."""
    TB = -(-N // SEARCH_TILE_N)
    seen = {}
    for tb in range(TB):
        left = N - tb * SEARCH_TILE_N
        nsub = 2 if left > SEARCH_SUB_N else 1
        for h in range(nsub):
            for rank in (0, 1):
                y0 = tb * SEARCH_TILE_N + h * SEARCH_SUB_N + rank * SEARCH_SUB_N // 2
                for t in range(y0, y0 + SEARCH_SUB_N // 2):
                    if t < N:
                        seen[t] = seen.get(t, 0) + 1
                    else:
                        assert tb == TB - 1
    assert len(seen) == N and set(seen.values()) == {1}


def test_search_tmem_and_shared_memory_plan():
    """TMEM: the 2 x 256 fp32 accumulator columns fill the 512 columns; the X
    ring stage (128 tokens x 64 fp16) keeps the 1024-byte alignment the 128-byte
    swizzle needs; both shared-memory plans (6 X stages, 3 dW stages, 3 or 2
    input stages) fit 227 KB."""
    SLAB_K = 64
    assert 2 * SEARCH_SUB_N <= 512
    x_stage = (SEARCH_SUB_N // 2) * SLAB_K * 2
    assert x_stage % 1024 == 0
    a_stage = 128 * SLAB_K * 2
    for w_bytes, IS in ((16384, 3), (32768, 2)):
        in_stage = -(-(w_bytes + 512 + 4096) // 1024) * 1024
        bars = 2 * 6 + 2 * 3 + 2 * IS + 5
        assert 1024 + 6 * x_stage + 3 * a_stage + IS * in_stage + bars * 8 + 16 <= 232448


# ---- batched decode: CTAs per linear, tiles per CTA, staged activation slots
DEC_TILE_TARGET = 45056


def dec_plan(linears, sms, gs=128, zeros=True):
    """w4a16_dec_config restated: tile heights, CTAs per linear and the tile
    ranges [t0, t1) of every CTA."""
    rows, weight, tiles = [], [], []
    for O, I in linears:
        nG, nzw = I // gs, -(-(I // gs) // 8)
        R = 8 * max(1, DEC_TILE_TARGET // (4 * I))
        rows.append(R)
        weight.append(O * (I // 2 + nG * 2 + (nzw * 4 if zeros else 0)))
        tiles.append(-(-O // R))
    total = sum(weight)
    cnt = [min(max(1, sms * w // total), t) for w, t in zip(weight, tiles)]
    while sum(cnt) > sms:
        w = max((l for l in range(len(cnt)) if cnt[l] > 1), key=lambda l: (-weight[l] / cnt[l], -l))
        cnt[w] -= 1
    while sum(cnt) < sms:
        cand = [l for l in range(len(cnt)) if cnt[l] < tiles[l]]
        if not cand:
            break
        w = max(cand, key=lambda l: (weight[l] / cnt[l], -l))
        cnt[w] += 1
    ranges = []
    for l, c in enumerate(cnt):
        T = tiles[l]
        for ci in range(c):
            ranges.append((l, ci * T // c, (ci + 1) * T // c))
    return rows, weight, tiles, cnt, ranges


BLOCK7 = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]


@pytest.mark.parametrize("linears,sms", [
    (BLOCK7, 148), ([(4096, 4096)], 148), ([(12288, 4096), (4096, 4096), (22016, 4096), (4096, 11008)], 148),
    ([(17, 64), (5, 1088), (100, 2048)], 148), ([(16, 64)], 148), ([(4100, 4160)], 7),
    ([(1, 64)] * 8, 8), ([(33, 3072), (2000, 1024)], 148), ([(4096, 4096)] * 8, 148)])
def test_decode_tiles_owned_once_and_balanced(linears, sms):
    """Every tile of every linear belongs to exactly one CTA, each CTA has at
    least one tile, no more CTAs than SMs; on the decoder block no CTA streams
    more than 6% above the mean."""
    rows, weight, tiles, cnt, ranges = dec_plan(linears, sms)
    assert len(ranges) <= sms and all(c >= 1 for c in cnt)
    seen = {}
    for l, t0, t1 in ranges:
        assert t1 > t0
        for t in range(t0, t1):
            assert (l, t) not in seen
            seen[(l, t)] = True
    assert len(seen) == sum(tiles)
    if linears == BLOCK7:
        per = [weight[l] * (t1 - t0) / tiles[l] for l, t0, t1 in ranges]
        assert max(per) <= 1.06 * sum(weight) / len(ranges)
    # every tile holds at most the larger of 44 KB and one 8-row tile of codes
    assert all(R * I // 2 <= max(DEC_TILE_TARGET, 4 * I) for (_, I), R in zip(linears, rows))


@pytest.mark.parametrize("gs", [32, 64, 128])
def test_decode_staged_slots_distinct_and_contiguous(gs):
    """Word wg of a group (thread j = wg // NW, its kk = wg % NW) goes to slot
    4 kk + j: a bijection onto the group's slots, and thread j's kk-th read
    (slot 4 kk + j) for j = 0..3 covers 4 consecutive slots."""
    WPG, NW = gs // 8, gs // 32
    slots = [(wg % NW) * 4 + wg // NW for wg in range(WPG)]
    assert sorted(slots) == list(range(WPG))
    for kk in range(NW):
        got = [slots[NW * j + kk] for j in range(4)]
        assert got == [4 * kk + j for j in range(4)]


def test_decode_unpacking_identities():
    """The four masks of a packed word give fp16 (1024 + n_e, 1024 + n_e+4) for
    e = 0, 2 and (1024 + 16 n_e, 1024 + 16 n_e+4) for e = 1, 3, exactly, for
    every nibble value."""
    import numpy as np
    for n in range(16):
        for pos in range(8):
            w = n << (4 * pos)
            w8 = w >> 8
            halves = {}
            for e, (src, mask) in enumerate([(w, 0x000F000F), (w, 0x00F000F0), (w8, 0x000F000F), (w8, 0x00F000F0)]):
                v = (src & mask) | 0x64006400
                lo, hi = np.array([v & 0xFFFF, v >> 16], np.uint16).view(np.float16).astype(np.float64)
                halves[e] = (lo, hi)
            want = {e: [1024.0, 1024.0] for e in range(4)}
            e, half = {0: (0, 0), 4: (0, 1), 1: (1, 0), 5: (1, 1), 2: (2, 0), 6: (2, 1), 3: (3, 0), 7: (3, 1)}[pos]
            want[e][half] += n * (16 if e in (1, 3) else 1)
            for k in range(4):
                assert halves[k] == tuple(want[k]), (n, pos, k)


def test_decode_shared_memory_plan_fits():
    """Per linear of the decoder block at M = 1: 16-row tiles of the 4096-wide
    linears and 8-row tiles of the 11008-wide one, at least four slots (over
    130 KB of codes in flight per SM); at M = 8 the 4096-wide linears still fit;
    an 11008-wide linear at M = 8 does not."""
    FIXED = 256 + 256 + 4 * 8 * 16 * 8 * 4

    def plan(M, I, gs=128, zeros=True):
        nG, nzw = I // gs, -(-(I // gs) // 8)
        R = 8 * max(1, DEC_TILE_TARGET // (4 * I))
        slot = -(-(R * I // 2 + R * nG * 2 + (R * nzw * 4 if zeros else 0)) // 128) * 128
        xbuf = -(-(M * (I + 32) * 2 + M * nG * 16) // 128) * 128
        st = min(8, (227 * 1024 - FIXED - xbuf) // slot)
        assert FIXED + xbuf + st * slot <= 227 * 1024
        return (R, st, st * R * I // 2) if st >= 2 else None

    assert plan(1, 4096)[0] == 16 and plan(1, 11008)[0] == 8
    assert all(plan(1, I)[2] >= 130 * 1024 for I in (4096, 11008))
    assert plan(8, 4096) is not None
    assert plan(8, 11008) is None


# ---- tensor-core apply (w4a16_tc_kernel): rings, TMEM columns, code chunk reads

def tc_rings(n_tile):
    """The launch's ring and TMEM plan for a token tile of n_tile (restated)."""
    xs_b = n_tile * 128
    bar_bytes = (2 * 4 + 2 * 8 + 2 * 8 + 2) * 8 + 16
    two = n_tile <= 64
    budget = (113 if two else 227) * 1024
    qs = 3
    xsn = min(8, (budget - 1024 - bar_bytes - qs * 16384) // (2 * xs_b))   # stages of two slabs
    tmem = 256 if two else 512
    tcols = 32 if n_tile <= 32 else 64 if n_tile <= 64 else 128 if n_tile <= 128 else 256
    a_st = min(8, (tmem - tcols) // 64)                                      # 64 columns: two slabs
    smem = 1024 + xsn * 2 * xs_b + qs * 16384 + bar_bytes
    smem = max(smem, 80 * 1024) if two else max(smem, 120 * 1024)
    return dict(two=two, xsn=xsn, qs=qs, tmem=tmem, tcols=tcols, a_st=a_st, smem=smem, xs_b=xs_b)


@pytest.mark.parametrize("n_tile", list(range(16, 257, 16)))
def test_tc_rings_fit_shared_memory_and_tmem(n_tile):
    p = tc_rings(n_tile)
    assert p["xsn"] >= 2 and p["a_st"] >= 2
    assert p["smem"] <= 227 * 1024
    if p["two"]:
        # two CTAs per SM: shared memory (plus the 1 KB the driver reserves per CTA)
        # and TMEM (256 columns each) both fit twice
        assert 2 * (p["smem"] + 1024) <= 228 * 1024 and 2 * p["tmem"] <= 512
        assert 3 * (p["smem"] + 1024) > 228 * 1024
    else:
        # one CTA per SM: more than half the shared memory, so no second CTA is placed
        # beside one holding all 512 TMEM columns
        assert 2 * (p["smem"] + 1024) > 228 * 1024
    assert p["tcols"] >= n_tile and p["tcols"] + 64 * p["a_st"] <= p["tmem"]
    # the code ring starts on a 1024-byte boundary (128-byte swizzle atoms), and every
    # activation stage does too (SW128 operand tiles)
    assert (p["xsn"] * p["xs_b"]) % 1024 == 0 and p["xs_b"] % 1024 == 0


def test_tc_code_chunk_reads_cover_units_once_conflict_free():
    # TMA's 128-byte swizzle stores logical 16-byte unit u of row r (128-byte rows of a
    # 1024-aligned tile) at unit u ^ (r % 8); thread (row r, half h) reads slab sub's
    # unit 2 sub + h there.
    seen = {}
    for r in range(128):
        for sub in range(4):
            for h in range(2):
                logical = 2 * sub + h
                phys = (logical ^ (r & 7)) & 7
                addr = r * 128 + phys * 16
                assert 0 <= addr and addr + 16 <= 128 * 128
                assert (r, phys) not in seen
                seen[(r, phys)] = logical
    assert len(seen) == 128 * 8
    # a quarter warp (8 consecutive lanes = 8 consecutive rows, same sub and half)
    # reads 8 distinct 16-byte bank groups
    for r0 in range(0, 128, 8):
        for sub in range(4):
            for h in range(2):
                units = {((2 * sub + h) ^ (r & 7)) & 7 for r in range(r0, r0 + 8)}
                assert len(units) == 8


def test_tc_code_chunk_coordinates_aligned():
    # chunk c of a split starting at slab kb0 is copied from word column (kb0 + 4 c) * 8:
    # a multiple of 4 words (16 bytes), as a tiled copy's innermost coordinate must be
    for kb0 in range(0, 200, 7):
        for c in range(10):
            x = (kb0 + 4 * c) * 8
            assert (x * 4) % 16 == 0


def tc_plan(M, I, O, sms=148):
    """w4a16_tc_plan restated: token tile, K splits and slabs per split."""
    OT = -(-O // 128)
    nK = I // 64
    best, best_n = 0.0, 0
    for n in (256, 128, 64):
        if n > 64 and M <= n // 2:
            continue
        tiles = OT * (-(-M // n))
        if tiles * 2 < sms:
            continue
        waves = -(-tiles // sms)
        cost = waves * n * (1.5 if n == 64 else 1.0)
        if best_n == 0 or cost < best:
            best, best_n = cost, n
    if best_n > 0:
        n_tile = best_n if best_n < M else -(-M // 16) * 16
        return n_tile, 1, nK
    n_tile = 256 if M >= 256 else -(-M // 16) * 16
    MT = -(-M // n_tile)
    target = sms if M >= 128 else 2 * sms
    splits = max(1, target // (OT * MT))
    splits = min(splits, nK)
    spl = -(-nK // splits)
    splits = -(-nK // spl)
    return n_tile, splits, spl


@pytest.mark.parametrize("M", [17, 32, 33, 64, 100, 255, 256, 257, 300, 1024, 4096])
@pytest.mark.parametrize("O,I", [(96, 64), (200, 384), (4096, 4096), (11008, 4096), (4096, 11008), (520, 1024)])
def test_tc_plan_covers_every_tile_and_slab_once(M, O, I):
    # the kernel's decomposition: CTA b -> tile b / splits (row tile tile % OT, token
    # tile tile / OT), split b % splits covering slabs [split * spl, min(nK, (split+1) spl))
    n_tile, splits, spl = tc_plan(M, I, O)
    assert 16 <= n_tile <= 256 and n_tile % 16 == 0
    OT, MT, nK = -(-O // 128), -(-M // n_tile), I // 64
    assert MT * n_tile >= M and (MT - 1) * n_tile < M
    seen = {}
    for b in range(OT * MT * splits):
        tile, split = divmod(b, splits)
        ot, mt = tile % OT, tile // OT
        k0, k1 = split * spl, min(nK, (split + 1) * spl)
        assert k0 < k1, "a split with no slabs"
        for k in range(k0, k1):
            key = (ot, mt, k)
            assert key not in seen
            seen[key] = b
    assert len(seen) == OT * MT * nK
    if splits > 1:
        # K is split only when whole tiles would leave more than half the SMs idle
        assert all(OT * -(-M // n) * 2 < 148 or (n > 64 and M <= n // 2) for n in (256, 128, 64))
