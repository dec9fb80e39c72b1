"""The barrier protocol of the fused decode + GEMM kernel (df11_gemm.cu), as a
model: its agents take the kernel's waits and arrivals in the kernel's order,
on the block offsets of real tile-major streams, and must all finish (no
deadlock) for every ring depth the launch can choose (S = 2..8).

Agents (one CTA, its units in order; tiles numbered q across units):
  * decode warp w (of 16 or 20): for each of its blocks b = first + w,
    first + w + warps, ... of a unit: arrive on every tile before the
    block's first output, wait
    until the ring slots of the tiles the block writes are free (the MMA of
    tile q - S is done), then arrive on every tile before its next block's
    first output; at the end of the unit, arrive on the rest;
  * control: per unit, bulk copies of the first S - 1 activation chunks
    (each once its slot is free), then the accumulator two units back must
    have been read; per tile: wait until all decode warps arrived and its
    activations were issued, MMA (frees the slot), issue the chunk S - 1
    ahead; then the accumulator is full;
  * epilogue: per unit, wait for the full accumulator, then free it.
The order in which a warp arrived only AFTER its first block (the first
version of the kernel) deadlocks on these streams once the first block of the
last warp starts S or more tiles into a unit; the model shows that too, as
the kernel did on a B200 (its bounded waits ran out and it reported the
timeout instead of hanging)."""
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


def _run_cta(offs, units, S, arrive_first=True, warps=16):
    """True when every agent of a CTA that takes all `units` finishes."""
    WARPS = warps
    full, mma_done, x_issued, acc_full, acc_free = {}, set(), set(), set(), set()

    def slot_free(q):
        return q < S or (q - S) in mma_done

    def decode(w):
        q0 = 0
        for e0, nt in units:
            e1 = e0 + nt * TILE
            first, end = _block_of(offs, e0), _block_of(offs, e1 - 1) + 1
            arrived = [0]

            def tile_of(x):
                return nt if x >= e1 else (0 if x <= e0 else (x - e0) // TILE)

            def arrive_upto(t_end):
                while arrived[0] < t_end:
                    q = q0 + arrived[0]
                    yield lambda q=q: slot_free(q)
                    full[q] = full.get(q, 0) + 1
                    arrived[0] += 1

            b = first + w
            while b < end:
                if arrive_first:
                    yield from arrive_upto(tile_of(offs[b]))
                lo, hi = max(offs[b], e0), min(offs[b + 1], e1)
                if lo < hi:
                    for t in range((lo - e0) // TILE, (hi - 1 - e0) // TILE + 1):
                        yield lambda q=q0 + t: slot_free(q)
                nxt = b + WARPS
                yield from arrive_upto(tile_of(offs[nxt]) if nxt < end else nt)
                b = nxt
            yield from arrive_upto(nt)
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
                yield lambda q=q: full.get(q, 0) == WARPS and q in x_issued
                mma_done.add(q)
                if t + S - 1 < nt:
                    yield from issue(t + S - 1)
            acc_full.add(k)
            q0 += nt

    def epilogue():
        for k in range(len(units)):
            yield lambda k=k: k in acc_full
            acc_free.add(k)

    agents = [decode(w) for w in range(WARPS)] + [control(), epilogue()]
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
                    break
                moved = True
        if not moved:
            return False
    return True


def _offsets(shapes, mats, T):
    stream = [df11.tile_major(w, r, c) for (r, c), w in zip(shapes, mats)]
    return [int(v) for v in df11.build_format(stream, T).arrays()["block_offset"]]


SMALL = [(128, 64), (256, 128), (384, 1088), (128, 2048)]


@pytest.mark.parametrize("warps", [16, 20])
@pytest.mark.parametrize("T", [32, 64])
@pytest.mark.parametrize("S", [2, 3, 4, 8])
def test_protocol_finishes(T, S, warps):
    mats = [inputs.gaussian(r * c, [73, m]) for m, (r, c) in enumerate(SMALL)]
    offs = _offsets(SMALL, mats, T)
    units = _units(SMALL)
    for grid in (1, 3, 148):  # units blockIdx.x, + grid, ... per CTA
        for cta in range(min(grid, len(units))):
            assert _run_cta(offs, units[cta::grid], S, warps=warps), (grid, cta)


def test_arriving_only_after_the_first_block_deadlocks():
    # one 128 x 1088 matrix: a unit of 16 tiles; with T = 64 the last warp's
    # first block starts 3 tiles in, beyond a ring of 2 or 3 slots
    shapes = [(128, 1088)]
    offs = _offsets(shapes, [inputs.gaussian(128 * 1088, [72, 128, 1088])], 64)
    units = _units(shapes)
    for S in (2, 3):
        assert not _run_cta(offs, units[:1], S, arrive_first=False)
        assert _run_cta(offs, units[:1], S)


@pytest.mark.slow
def test_protocol_finishes_on_the_llama3_8b_block():
    # the fused GEMM's workload: 1,664 units over 148 CTAs, T = 64, the
    # launch configurations of batch 256 and 128 (16 decode warps, S = 2 and
    # 3), 64 and 16 (20 decode warps, S = 3 and 4)
    shapes = [s for _, s in inputs.LLAMA3_8B]
    offs = _offsets(shapes, [m for _, _, m in inputs.block(2, 0)], 64)
    units = _units(shapes)
    for warps, S in ((16, 2), (16, 3), (20, 3), (20, 4)):
        for cta in range(148):
            assert _run_cta(offs, units[cta::148], S, warps=warps), (warps, S, cta)
