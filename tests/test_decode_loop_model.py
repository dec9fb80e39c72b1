"""The pending-word decode loop of the block decoder (df11_block.cuh:
table_word, decode_bulk2, chain_roles, chain_put1), as a model of its 32-bit
arithmetic, on the CPU.

Per chain the loop holds a pending word w with n exponent bytes and mul =
2^(8 n).  A lookup adds the entry's exponents at byte n (w + syms * mul, the
bytes spilling past the word in the high half of the product), rotates mul
left by 8 x count bits, and when the rotation wraps (mul decreases) stores
the full word and keeps the spilled bytes.  The loop runs two passes per
trip with mul and w exchanging registers between them; a code longer than
12 bits has the entry 2^31, which takes 2^31 (first pass of a trip) or 2^30
(second) from the chain's bit count, so the chain stops, and which adds
2^24 x mul to w.  After the loop chain_roles sorts the registers out: for a
chain stopped on a long code the size of the bit-count drop tells the pass,
otherwise mul is the larger of the two (w < mul).  The caller then adds the
long code's exponent alone (chain_put1) and runs the loop again.

The model drives random code sequences (1 to 3 exponents per lookup, long
codes anywhere, any byte values including 0) through that arithmetic and
checks that the stored words plus the final pending bytes are exactly the
exponents in order, for every position of a long code within a trip and
within a word."""
import random

import pytest

M32 = 0xFFFFFFFF


def rotl(x, r):
    r &= 31
    return ((x << r) | (x >> (32 - r))) & M32 if r else x


def table_word(n, bits, syms):
    """The loop's entry form: count in bits 0..1, length in bits 2..6, the
    count's exponents in bits 7..30; 2^31 for a code longer than 12 bits."""
    if n == 0:
        return 0x80000000
    return (n & 3) | ((bits & 31) << 2) | ((syms & ((1 << (8 * n)) - 1)) << 7)


def asr(x, k):
    """Arithmetic shift right of a 32-bit pattern."""
    v = x - (1 << 32) if x & 0x80000000 else x
    return (v >> k) & M32


def to_int(x):
    return x - (1 << 32) if x & 0x80000000 else x


def run_loop(entries, rem, regs):
    """One call of the loop on one chain. entries: the lookups it meets in
    order (each consumed when active). regs: [X, Y] = the registers that
    hold (mul, w) at entry. Returns (stored words, rem, regs, lookups used)."""
    X, Y = regs
    stored = []
    used = 0
    pas = 0
    active = to_int(rem) > 0
    while active:
        e = entries[used]
        used += 1
        mask = 0x8000001F if pas % 2 == 0 else 0x4000001F
        mul, w = (X, Y) if pas % 2 == 0 else (Y, X)
        ca = asr(e, 2)
        t = ca & mask
        rem = (rem - t) & M32
        syms = e >> 7
        hi = (syms * mul) >> 32
        lo = (syms * mul + w) & M32
        new_mul = rotl(mul, (e << 3) & M32)
        po = new_mul < mul
        if po:
            stored.append(lo)
        new_w = hi if po else lo
        if pas % 2 == 0:
            X, Y = new_w, new_mul  # new w into mul's register, new mul into w's
        else:
            Y, X = new_w, new_mul
        pas += 1
        active = to_int(rem) > 0
    return stored, rem, [X, Y], used


def chain_roles(rem, regs):
    """(mul, w, rem) from the registers after a call (chain_roles)."""
    X, Y = regs  # X: the mul field (%6), Y: the w field (%5)
    r0, r1 = Y, X
    r = to_int(rem)
    if r < -(1 << 29):
        first = r < -(3 << 29)
        mul = r0 if first else r1
        w = ((r1 if first else r0) - 0x01000000 * mul) & M32
        rem = (rem + (0x80000000 if first else 0x40000000)) & M32
        return mul, w, rem
    return max(r0, r1), min(r0, r1), rem


def chain_put1(mul, w, sym):
    """One exponent from the long-code path; returns (stored word or None, mul, w)."""
    lo = (sym * mul + w) & M32
    nm = rotl(mul, 8)
    if nm < mul:
        return lo, nm, 0
    return None, nm, lo


def decode_chain(codes, rng):
    """codes: list of ('t', [bytes]) table lookups or ('l', byte) long codes.
    Returns the bytes the loop leaves in the slot plus its pending word."""
    entries = []
    for kind, v in codes:
        if kind == 't':
            syms = sum(b << (8 * i) for i, b in enumerate(v))
            entries.append(table_word(len(v), rng.randint(len(v), 12), syms))
        else:
            entries.append(table_word(0, 0, 0))
    stored = []
    mul, w = 1, 0
    rem = 10 ** 6  # bits left: ample; the model ends with the entries
    i = 0
    while i < len(entries):
        # the loop stops on a long code or at the end of the chain's entries
        run = entries[i:]
        stop = next((k for k, e in enumerate(run) if e == 0x80000000), None)
        seg_len = len(run) if stop is None else stop + 1
        # the chain's bits run out exactly after the last table entry
        rem = 1000 if stop is not None else 1
        bits = [((e >> 2) & 31) for e in run[:seg_len]]
        if stop is None:
            rem = sum(bits)
        else:
            rem = sum(bits[:-1]) + 1 + rng.randint(0, 40)
        st, rem, regs, used = run_loop(run[:seg_len], rem, [mul, w])
        assert used == seg_len
        stored += st
        mul, w, rem = chain_roles(rem, regs)
        i += seg_len
        if stop is not None:
            assert to_int(rem) > 0  # a long-stopped chain hands back bits
            word, mul, w = chain_put1(mul, w, codes[i - 1][1])
            if word is not None:
                stored.append(word)
        else:
            assert to_int(rem) <= 0
    assert w < mul and mul in (1, 1 << 8, 1 << 16, 1 << 24)
    n = {1: 0, 1 << 8: 1, 1 << 16: 2, 1 << 24: 3}[mul]
    out = []
    for word in stored:
        out += [(word >> (8 * k)) & 0xFF for k in range(4)]
    out += [(w >> (8 * k)) & 0xFF for k in range(n)]
    return out


@pytest.mark.parametrize("seed", range(6))
def test_pending_word_loop_stores_the_exponents_in_order(seed):
    rng = random.Random(seed)
    for _ in range(3000):
        codes = []
        for _ in range(rng.randint(0, 14)):
            if rng.random() < 0.2:
                codes.append(('l', rng.choice([0, 1, 0x80, 0xFF, rng.randint(0, 255)])))
            else:
                c = rng.randint(1, 3)
                codes.append(('t', [rng.choice([0, 1, 0xFF, rng.randint(0, 255)]) for _ in range(c)]))
        want = []
        for kind, v in codes:
            want += v if kind == 't' else [v]
        assert decode_chain(codes, rng) == want


def test_long_code_in_either_pass_at_every_byte_position():
    # a long code met in the first or the second pass of a trip, with 0..3
    # bytes pending: the bit-count drop tells the pass and the w repair
    # removes the entry's 2^24 x mul
    rng = random.Random(7)
    for lead in range(0, 8):
        for n_bytes in range(1, 4):
            codes = [('t', [0] * n_bytes)] * lead + [('l', 1), ('t', [1, 0, 0])]
            want = [0] * (n_bytes * lead) + [1, 1, 0, 0]
            assert decode_chain(codes, rng) == want


def test_registers_stay_ordered_without_long_codes():
    # w < mul after every pass: what lets chain_roles take the larger as mul
    rng = random.Random(8)
    for _ in range(2000):
        entries = [table_word(c, c, rng.randint(0, (1 << (8 * c)) - 1))
                   for c in [rng.randint(1, 3) for _ in range(rng.randint(1, 12))]]
        rem = sum((e >> 2) & 31 for e in entries)
        _, rem, regs, _ = run_loop(entries, rem, [1, 0])
        assert min(regs) < max(regs)
