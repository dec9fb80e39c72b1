"""The barrier protocol of the fused decode + GEMM kernel (df11_gemm.cu), as a
model: its agents take the kernel's waits and arrivals in the kernel's order,
on the block offsets of real tile-major streams, and must all finish (no
deadlock) for every number of exponent tiles E and operand stages S the
launch can choose.

Agents (one CTA, its units in order; tiles numbered q across units):
  * decode warp w (of 16, 20 or 27): for each of its blocks b = first + w,
    first + w + warps, ... of a unit, after decoding it (which waits for
    nothing): wait until the exponent tiles of the tiles the block covers are
    free (tile q - E merged), copy, add the block's elements to each tile's
    count;
  * control: per unit, activation copies of the first S - 1 chunks (each once
    its slot is free: the MMA S tiles back is complete), then the accumulator
    two units back must have been read; per tile: wait until the tile is full
    and its activations issued, MMA, wait for the MMA to complete and publish
    that, issue the chunk S - 1 ahead; then the accumulator is full;
  * merge and epilogue warps (four, modelled as one): per tile in order, wait
    until its count is complete and the control thread has published the MMA
    of tile q - S, merge (the tile is full for the MMA, its exponent tile
    free); after a unit's tiles the epilogue of the unit before (wait for its
    accumulator, free it), the last unit's at the end.
With one exponent tile a block that covers two tiles waits for the second
while its own elements are what the first still lacks: the model deadlocks
there, which is why the launch never takes fewer than two."""
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs

TILE = 8192


def _units(shapes):
    out, off = [], 0
    for r, c in shapes:
        kc = c // 64
        for rt in range(r // 128):
            for k0 in range(0, kc, 16):
                out.append((off + (rt * kc + k0) * TILE, min(16, kc - k0)))
        off += r * c
    return out


def _block_of(offs, x):
    lo, hi = 0, len(offs) - 2
    while lo < hi:
        mid = (lo + hi + 1) >> 1
        if offs[mid] <= x:
            lo = mid
        else:
            hi = mid - 1
    return lo


def _run_cta(offs, units, S, E, warps=16):
    """True when every agent of a CTA that takes all `units` finishes."""
    WARPS = warps
    count, merged, full, mma_done, x_issued, acc_full, acc_free = {}, set(), set(), set(), set(), set(), set()
    published = [0]  # the MMAs of tiles below this are known complete (the control thread's count)

    def slot_free(q):
        return q < S or (q - S) in mma_done

    def etile_free(q):
        return q < E or (q - E) in merged

    def decode(w):
        q0 = 0
        for e0, nt in units:
            e1 = e0 + nt * TILE
            first, end = _block_of(offs, e0), _block_of(offs, e1 - 1) + 1
            b = first + w
            while b < end:
                lo, hi = max(offs[b], e0), min(offs[b + 1], e1)
                if lo < hi:
                    tiles = range((lo - e0) // TILE, (hi - 1 - e0) // TILE + 1)
                    for t in tiles:
                        yield lambda q=q0 + t: etile_free(q)
                    for t in tiles:
                        q = q0 + t
                        a, z = e0 + t * TILE, e0 + (t + 1) * TILE
                        count[q] = count.get(q, 0) + min(hi, z) - max(lo, a)
                b += WARPS
            q0 += nt

    def control():
        q0 = 0
        for k, (e0, nt) in enumerate(units):
            def issue(t, q0=q0):
                q = q0 + t
                yield lambda q=q: slot_free(q)
                x_issued.add(q)

            for t in range(min(S - 1, nt)):
                yield from issue(t)
            if k >= 2:
                yield lambda k=k: (k - 2) in acc_free
            for t in range(nt):
                q = q0 + t
                yield lambda q=q: q in full and q in x_issued
                mma_done.add(q)
                published[0] = q + 1  # waits for the MMA's completion, then publishes it
                if t + S - 1 < nt:
                    yield from issue(t + S - 1)
            acc_full.add(k)
            q0 += nt

    def merge_epilogue():
        q0 = 0
        for k, (e0, nt) in enumerate(units):
            for t in range(nt):
                q = q0 + t
                yield lambda q=q: count.get(q, 0) >= TILE and (q < S or published[0] >= q - S + 1)
                full.add(q)
                merged.add(q)
            q0 += nt
            if k >= 1:
                yield lambda k=k: (k - 1) in acc_full
                acc_free.add(k - 1)
        if units:
            yield lambda: (len(units) - 1) in acc_full
            acc_free.add(len(units) - 1)

    agents = [decode(w) for w in range(WARPS)] + [control(), merge_epilogue()]
    waiting = [None] * len(agents)
    alive = set(range(len(agents)))
    while alive:
        moved = False
        for i in sorted(alive):
            while True:
                if waiting[i] is not None:
                    if not waiting[i]():
                        break
                    waiting[i] = None
                try:
                    waiting[i] = next(agents[i])
                except StopIteration:
                    alive.discard(i)
                    moved = True
                    break
                moved = True
        if not moved:
            return False
    # every tile was merged once and the MMA ran on it
    total = sum(nt for _, nt in units)
    return merged == set(range(total)) == mma_done


def _offsets(shapes, mats, T):
    stream = [df11.tile_major(w, r, c) for (r, c), w in zip(shapes, mats)]
    return [int(v) for v in df11.build_format(stream, T).arrays()["block_offset"]]


SMALL = [(128, 64), (256, 128), (384, 1088), (128, 2048)]


@pytest.mark.parametrize("warps", [16, 20, 27])
@pytest.mark.parametrize("T", [32, 64])
@pytest.mark.parametrize("E", [2, 3, 4, 6, 16])
def test_protocol_finishes(T, E, warps):
    mats = [inputs.gaussian(r * c, [73, m]) for m, (r, c) in enumerate(SMALL)]
    offs = _offsets(SMALL, mats, T)
    units = _units(SMALL)
    for S in (2, 3):
        for grid in (1, 3, 148):  # units blockIdx.x, + grid, ... per CTA
            for cta in range(min(grid, len(units))):
                assert _run_cta(offs, units[cta::grid], S, E, warps=warps), (S, grid, cta)


def test_one_exponent_tile_deadlocks():
    # a block that covers two tiles needs both exponent tiles at once
    shapes = [(128, 1088)]
    offs = _offsets(shapes, [inputs.gaussian(128 * 1088, [72, 128, 1088])], 64)
    units = _units(shapes)
    straddles = any((max(offs[b], 0) // TILE) != ((offs[b + 1] - 1) // TILE) for b in range(len(offs) - 1)
                    if offs[b + 1] > offs[b])
    assert straddles
    assert not _run_cta(offs, units[:1], 2, 1)
    assert _run_cta(offs, units[:1], 2, 2)


@pytest.mark.slow
def test_protocol_finishes_on_the_llama3_8b_block():
    # the fused GEMM's workload: 1,664 units over 148 CTAs, T = 64, in the
    # launch configurations of batch 16 to 256 (27 decode warps with 7, 6
    # and 4 exponent tiles, 20 warps with 3; two operand stages)
    shapes = [s for _, s in inputs.LLAMA3_8B]
    offs = _offsets(shapes, [m for _, _, m in inputs.block(2, 0)], 64)
    units = _units(shapes)
    for warps, E in ((27, 7), (27, 6), (27, 4), (20, 3)):
        for cta in range(148):
            assert _run_cta(offs, units[cta::148], 2, E, warps=warps), (warps, E, cta)
