"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks one oracle step against something the DFloat11 page or the
mathematics fixes: IEEE/BF16 field layout read back through numpy's float32,
brute-force optimality of code lengths on tiny alphabets, Kraft equality,
the Shannon bound, a printed canonical-code example (RFC 1951), a DF11 example
worked by hand, bit strings built symbol by symbol, LUT entries matched as bit
strings, exhaustive round trips, and the closed-form exponent entropy of a
Gaussian.  No expected value here is produced by the CUDA library.
"""
import itertools
import math
import os

import numpy as np
import pytest

from huffman_decode_03_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# helpers written from the definitions, as bit strings
# --------------------------------------------------------------------------
def code_strings(lens, codes):
    return {s: format(int(codes[s]), "0{}b".format(int(lens[s]))) for s in range(256) if lens[s] > 0}


def stream_string(stream, total_bits):
    bits = "".join(format(int(b), "08b") for b in np.asarray(stream, np.uint8))
    return bits[:total_bits]


def brute_force_min_cost(weights, cap):
    """Minimum sum w*l over all length vectors with l in 1..cap and Kraft <= 1."""
    k = len(weights)
    best = None
    for ls in itertools.product(range(1, cap + 1), repeat=k):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            c = sum(w * l for w, l in zip(weights, ls))
            if best is None or c < best:
                best = c
    return best


def entropy_bits(hist):
    h = np.asarray(hist, np.float64)
    p = h[h > 0] / h.sum()
    return float(-(p * np.log2(p)).sum())


# --------------------------------------------------------------------------
# BF16 field split ("Ruang kompresi": 1 sign, 8 exponent, 7 mantissa bits)
# --------------------------------------------------------------------------
def test_split_matches_ieee_layout(oracle_mod):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    exponent_field = (allbits >> 7) & 0xFF
    ok = allbits[exponent_field < 240]
    assert ok.size == 61440
    exps, sm = oracle_mod.split(ok)
    f = (ok.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # sign from the float's sign bit
    assert np.array_equal((sm >> 7).astype(bool), np.signbit(f))
    # exponent: zero/subnormal -> 0, normal x = m * 2^e (0.5 <= m < 1) -> e + 126
    mant, e = np.frexp(np.abs(f))
    normal = np.abs(f) >= 2.0 ** -126
    assert np.all(exps[~normal] == 0)
    assert np.array_equal(exps[normal].astype(np.int64), e[normal].astype(np.int64) + 126)
    # mantissa: 7 fraction bits
    frac = np.where(normal, (2 * mant - 1) * 128, np.abs(f) / 2.0 ** -133)
    assert np.array_equal((sm & 0x7F).astype(np.int64), np.round(frac).astype(np.int64))


def test_split_textbook_values(oracle_mod):
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x8000, 0x3F00, 0x7780], np.uint16)
    exps, sm = oracle_mod.split(bits)
    assert exps.tolist() == [127, 128, 0, 0, 126, 239]
    assert sm.tolist() == [0x00, 0x80, 0x01, 0x80, 0x00, 0x00]


@pytest.mark.parametrize("bits", [0x7800, 0x7F7F, 0x7F80, 0xFFC0, 0xF800])
def test_split_rejects_pointer_exponents(oracle_mod, bits):
    # exponents 240..255 (huge magnitudes, Inf, NaN) are reserved as pointers
    with pytest.raises(oracle_mod.UnsupportedExponent):
        oracle_mod.split(np.array([0x3F80, bits], np.uint16))


def test_histogram_counts(oracle_mod):
    x = np.random.default_rng(1).integers(0, 240, 10000).astype(np.uint8)
    assert np.array_equal(oracle_mod.histogram(x), np.bincount(x, minlength=256).astype(np.uint64))


# --------------------------------------------------------------------------
# Code lengths ("Format DFloat11": Huffman over the exponent distribution)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(40))
def test_huffman_is_optimal_brute_force(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    k = int(rng.integers(2, 7))
    syms = rng.choice(240, k, replace=False)
    hist = np.zeros(256, np.uint64)
    w = rng.integers(1, 50, k)
    if seed % 4 == 0:
        w[:] = w[0]  # all ties
    hist[syms] = w
    lens = oracle_mod.huffman_lengths(hist)
    cost = int((hist * lens).sum())
    assert cost == brute_force_min_cost([int(x) for x in w], k - 1)
    assert sum(2.0 ** -int(lens[s]) for s in syms) == 1.0  # Kraft equality
    assert np.all(lens[hist == 0] == 0)


@pytest.mark.parametrize("seed", range(30))
def test_package_merge_is_optimal_under_cap(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    k = int(rng.integers(3, 8))
    cap = int(rng.integers(max(2, math.ceil(math.log2(k))), 5))
    syms = rng.choice(240, k, replace=False)
    hist = np.zeros(256, np.uint64)
    w = (2 ** rng.integers(0, 8, k)) + rng.integers(0, 3, k)  # skewed, forces deep trees
    hist[syms] = w
    lens = oracle_mod.package_merge(hist, cap)
    assert int(lens.max()) <= cap
    assert int((hist * lens).sum()) == brute_force_min_cost([int(x) for x in w], cap)
    assert sum(2.0 ** -int(lens[s]) for s in syms) == 1.0


def test_package_merge_without_binding_cap_equals_huffman_cost(oracle_mod):
    rng = np.random.default_rng(7)
    for _ in range(20):
        hist = np.zeros(256, np.uint64)
        k = int(rng.integers(2, 60))
        hist[rng.choice(240, k, replace=False)] = rng.integers(1, 1000, k)
        h = oracle_mod.huffman_lengths(hist)
        p = oracle_mod.package_merge(hist, 32)
        assert int((hist * h).sum()) == int((hist * p).sum())


def test_package_merge_infeasible_cap(oracle_mod):
    hist = np.zeros(256, np.uint64)
    hist[:5] = 1
    with pytest.raises(ValueError):
        oracle_mod.package_merge(hist, 2)  # 5 symbols need a length-3 code


def fibonacci_hist(k):
    f = [1, 1]
    while len(f) < k:
        f.append(f[-1] + f[-2])
    hist = np.zeros(256, np.uint64)
    hist[:k] = f[:k]
    return hist


def test_fibonacci_weights_force_length_limit(oracle_mod):
    # Fibonacci weights give the most skewed Huffman tree: depth k - 1.
    hist = fibonacci_hist(40)
    plain = oracle_mod.huffman_lengths(hist)
    assert int(plain.max()) == 39
    capped = oracle_mod.code_lengths(hist, 32)
    assert int(capped.max()) == 32
    assert sum(2.0 ** -int(capped[s]) for s in range(40)) == 1.0
    # the cap costs bits, but never below the unconstrained optimum
    assert int((hist * capped).sum()) >= int((hist * plain).sum())


def test_single_and_empty_alphabets(oracle_mod):
    hist = np.zeros(256, np.uint64)
    assert oracle_mod.huffman_lengths(hist).max() == 0
    hist[77] = 5
    lens = oracle_mod.code_lengths(hist)
    assert lens[77] == 1 and lens.sum() == 1


@pytest.mark.parametrize("seed", range(10))
def test_shannon_bound(oracle_mod, seed):
    rng = np.random.default_rng(200 + seed)
    hist = np.zeros(256, np.uint64)
    k = int(rng.integers(2, 80))
    hist[rng.choice(240, k, replace=False)] = rng.geometric(0.05, k) ** 2
    lens = oracle_mod.code_lengths(hist)
    H = entropy_bits(hist)
    avg = float((hist * lens).sum()) / float(hist.sum())
    assert H - 1e-12 <= avg < H + 1


# --------------------------------------------------------------------------
# Canonical codes
# --------------------------------------------------------------------------
def test_canonical_codes_rfc1951_example(oracle_mod):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "rfc1951_canonical.txt")) if l.strip() and not l.startswith("#")]
    lens = np.zeros(256, np.uint8)
    for sym, l, _ in rows:
        lens[int(sym)] = int(l)
    codes = oracle_mod.canonical_codes(lens)
    got = code_strings(lens, codes)
    for sym, _, code in rows:
        assert got[int(sym)] == code


@pytest.mark.parametrize("seed", range(10))
def test_canonical_codes_prefix_free_and_ordered(oracle_mod, seed):
    rng = np.random.default_rng(300 + seed)
    hist = np.zeros(256, np.uint64)
    k = int(rng.integers(2, 50))
    hist[rng.choice(240, k, replace=False)] = rng.integers(1, 10 ** 6, k)
    lens = oracle_mod.code_lengths(hist)
    cs = code_strings(lens, oracle_mod.canonical_codes(lens))
    strs = list(cs.values())
    for a in strs:
        for b in strs:
            if a is not b:
                assert not b.startswith(a)
    order = sorted(cs, key=lambda s: (len(cs[s]), s))
    vals = [int(cs[s], 2) << (64 - len(cs[s])) for s in order]
    assert vals == sorted(vals) and len(set(vals)) == len(vals)


# --------------------------------------------------------------------------
# The hand-worked DF11 example
# --------------------------------------------------------------------------
def _golden_example():
    d = {}
    for line in open(os.path.join(GOLDEN, "df11_hand_example.txt")):
        if line.strip() and not line.startswith("#"):
            key, *vals = line.split()
            d[key] = vals
    return d


def test_hand_worked_example(oracle_mod):
    g = _golden_example()
    w = np.array([int(x, 16) for x in g["bits"]], np.uint16)
    f = oracle_mod.build_format(w, threads_per_block=256)
    exps, sm = oracle_mod.split(w)
    assert exps.tolist() == [int(x) for x in g["exps"]]
    assert sm.tolist() == [int(x, 16) for x in g["sm"]]
    for item in g["lengths"]:
        s, l = item.split(":")
        assert int(f["code_lengths"][int(s)]) == int(l)
    cs = code_strings(f["code_lengths"], f["codes"])
    for item in g["codes"]:
        s, c = item.split(":")
        assert cs[int(s)] == c
    assert f["encoded_exponent"].tolist() == [int(x, 16) for x in g["stream"]]
    assert f["total_bits"] == int(g["total_bits"][0])
    assert f["gaps"].tolist() == [int(x) for x in g["gaps"]]
    assert f["block_offset"].tolist() == [int(x) for x in g["block_offset"]]
    lut0 = f["luts"][0]
    for item in g["lut0"]:
        rng_, s = item.split(":")
        lo, hi = (int(x) for x in rng_.split("-"))
        assert np.all(lut0[lo:hi + 1] == int(s))
    assert f["luts"].shape[0] == 1
    assert np.array_equal(oracle_mod.decode_format(f), w)


# --------------------------------------------------------------------------
# Encoding, metadata and LUTs against bit-string constructions
# --------------------------------------------------------------------------
def _tiny_sequences():
    for alpha in (1, 2, 3):
        for length in range(1, 6):
            for seq in itertools.product(range(alpha), repeat=length):
                yield alpha, seq


def test_encode_exhaustive_tiny(oracle_mod):
    base = 100  # exponents 100, 101, 102
    for alpha, seq in _tiny_sequences():
        exps = np.array([base + s for s in seq], np.uint8)
        hist = oracle_mod.histogram(exps)
        lens = oracle_mod.code_lengths(hist)
        codes = oracle_mod.canonical_codes(lens)
        stream, total = oracle_mod.encode(exps, lens, codes)
        cs = code_strings(lens, codes)
        expect = "".join(cs[int(e)] for e in exps)
        assert total == len(expect)
        assert stream_string(stream, total) == expect
        # padding bits are zero
        assert stream_string(stream, len(stream) * 8)[total:] == "0" * (len(stream) * 8 - total)


def _metadata_from_strings(code_lens, total, T):
    starts = np.concatenate([[0], np.cumsum(code_lens)[:-1]]).astype(np.int64) if len(code_lens) else np.zeros(0, np.int64)
    nseg = (total + 63) // 64
    nblocks = (nseg + T - 1) // T
    gaps = []
    for s in range(nseg):
        later = starts[starts >= 64 * s]
        first = int(later[0]) if later.size else total
        gaps.append(first - 64 * s)
    offs = [int(np.sum(starts < 64 * T * b)) for b in range(nblocks)] + [len(code_lens)]
    return gaps, offs


@pytest.mark.parametrize("T", [1, 2, 3, 32])
@pytest.mark.parametrize("seed", range(6))
def test_metadata_definition(oracle_mod, T, seed):
    rng = np.random.default_rng(400 + seed)
    n = int(rng.integers(1, 3000))
    w = inputs.to_bf16_bits((rng.standard_t(3, n) * 0.02).astype(np.float32))
    f = oracle_mod.build_format(w, threads_per_block=T)
    code_lens = f["code_lengths"][oracle_mod.split(w)[0]].astype(np.int64)
    gaps, offs = _metadata_from_strings(code_lens, f["total_bits"], T)
    assert f["gaps"].tolist() == gaps
    assert f["block_offset"].tolist() == offs
    assert max(gaps) <= 31
    # packed 5-bit fields, LSB-first
    words = f["gaps_packed"]
    bitstr = "".join(format(int(x), "064b")[::-1] for x in words)
    for s, g in enumerate(gaps):
        assert int(bitstr[5 * s:5 * s + 5][::-1], 2) == g


def _lut_expectation(cs):
    """Expected LUTs from the code strings: child LUT prefixes numbered level by
    level in increasing prefix order; pointer to child j is 256 - j."""
    longest = max(len(c) for c in cs.values())
    prefixes = [""]
    for m in range(1, (longest + 7) // 8):
        lvl = sorted({c[: 8 * m] for c in cs.values() if len(c) > 8 * m})
        prefixes += lvl
    ptr = {p: 256 - j for j, p in enumerate(prefixes) if j > 0}
    luts = []
    for p in prefixes:
        row = []
        for i in range(256):
            s = p + format(i, "08b")
            hit = [sym for sym, c in cs.items() if s.startswith(c)]
            if hit:
                row.append(hit[0])
            else:
                row.append(ptr[s])
        luts.append(row)
    return luts


@pytest.mark.parametrize("seed", range(8))
def test_luts_match_bit_strings(oracle_mod, seed):
    rng = np.random.default_rng(500 + seed)
    hist = np.zeros(256, np.uint64)
    k = int(rng.integers(2, 60))
    syms = rng.choice(240, k, replace=False)
    hist[syms] = (2.0 ** rng.uniform(0, 26, k)).astype(np.uint64) + 1  # wide spread -> long codes
    lens = oracle_mod.code_lengths(hist)
    codes = oracle_mod.canonical_codes(lens)
    luts = oracle_mod.build_luts(lens, codes)
    expect = _lut_expectation(code_strings(lens, codes))
    assert luts.shape[0] == len(expect)
    assert luts.tolist() == expect


def test_luts_fibonacci_depth32(oracle_mod):
    hist = fibonacci_hist(34)
    lens = oracle_mod.code_lengths(hist)
    assert int(oracle_mod.huffman_lengths(hist).max()) == 33
    assert int(lens.max()) == 32
    codes = oracle_mod.canonical_codes(lens)
    luts = oracle_mod.build_luts(lens, codes)
    assert luts.tolist() == _lut_expectation(code_strings(lens, codes))
    assert 2 <= luts.shape[0] <= 17


def test_luts_single_symbol_fill(oracle_mod):
    hist = np.zeros(256, np.uint64)
    hist[126] = 9
    lens = oracle_mod.code_lengths(hist)
    luts = oracle_mod.build_luts(lens, oracle_mod.canonical_codes(lens))
    assert luts.shape == (1, 256) and np.all(luts == 126)


@pytest.mark.parametrize("heavy,children", [(4, 32), (8, 16)])
def test_child_lut_limit(oracle_mod, heavy, children):
    # 239 symbols, a few heavy ones: the rare symbols get 9..13-bit codes under
    # many different 8-bit prefixes.  Pointer values 240..255 name at most 16
    # children ("Decoding berbasis LUT hierarkis").
    hist = np.zeros(256, np.uint64)
    hist[:239] = 1
    hist[:heavy] = 1000
    lens = oracle_mod.code_lengths(hist)
    codes = oracle_mod.canonical_codes(lens)
    cs = code_strings(lens, codes)
    assert len({c[:8] for c in cs.values() if len(c) > 8}) == children
    if children > 16:
        with pytest.raises(ValueError):
            oracle_mod.build_luts(lens, codes)
    else:
        luts = oracle_mod.build_luts(lens, codes)
        assert luts.shape[0] == 17
        assert luts.tolist() == _lut_expectation(cs)


# --------------------------------------------------------------------------
# Round trips (the losslessness claim of the page: bit-identical BF16)
# --------------------------------------------------------------------------
def test_round_trip_every_bf16_pattern(oracle_mod):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ok = allbits[((allbits >> 7) & 0xFF) < 240]
    for seed in range(3):
        w = np.random.default_rng(seed).permutation(ok) if seed else ok
        f = oracle_mod.build_format(w)
        assert np.array_equal(oracle_mod.decode_format(f), w)


def test_round_trip_tiny_exhaustive(oracle_mod):
    for alpha, seq in _tiny_sequences():
        w = np.array([(0x3F80 - 0x80 * s) ^ (0x8000 * (s == 1)) for s in seq], np.uint16)
        f = oracle_mod.build_format(w, threads_per_block=1)
        assert np.array_equal(oracle_mod.decode_format(f), w)


@pytest.mark.parametrize("n", [0, 1, 2, 63, 64, 65, 256 * 25 - 1, 256 * 25 + 1])
def test_round_trip_sizes(oracle_mod, n):
    w = inputs.gaussian(n, [9, n])
    f = oracle_mod.build_format(w)
    assert np.array_equal(oracle_mod.decode_format(f), w)
    assert f["block_offset"][-1] == n


def test_round_trip_length_limited(oracle_mod):
    # 34 exponents with Fibonacci counts (14.9 M elements): plain Huffman
    # would need a 33-bit code, so the 32-bit cap must act.
    hist = fibonacci_hist(34)
    exps = np.repeat(np.arange(34, dtype=np.uint16) + 60, hist[:34].astype(np.int64))
    exps = np.random.default_rng(5).permutation(exps)
    w = (exps << 7).astype(np.uint16) | np.uint16(0x8000)
    f = oracle_mod.build_format(w)
    assert int(oracle_mod.huffman_lengths(f["hist"]).max()) == 33
    assert int(f["code_lengths"].max()) == 32
    assert np.array_equal(oracle_mod.decode_format(f), w)


def test_decode_rejects_truncated_stream(oracle_mod):
    w = inputs.gaussian(1000, [9, 1000])
    f = oracle_mod.build_format(w)
    with pytest.raises(ValueError):
        oracle_mod.decode(f["encoded_exponent"], f["total_bits"] - 40, f["code_lengths"], f["codes"],
                          f["packed_sign_mantissa"], f["n"])


def test_decode_range_partitions_stream(oracle_mod):
    w = inputs.gaussian(5000, [9, 5000])
    f = oracle_mod.build_format(w, threads_per_block=4)
    exps, _ = oracle_mod.split(w)
    parts = []
    nseg = len(f["gaps"])
    for s in range(nseg):
        a = 64 * s + int(f["gaps"][s])
        b = 64 * (s + 1) + int(f["gaps"][s + 1]) if s + 1 < nseg else f["total_bits"]
        parts.append(oracle_mod.decode_range(f["encoded_exponent"], f["total_bits"], a, b,
                                             f["code_lengths"], f["codes"]))
    assert np.array_equal(np.concatenate(parts), exps)


# --------------------------------------------------------------------------
# Closed form: exponent entropy of N(0, sigma) rounded to BF16
# ("Ruang kompresi": the exponent carries about 2.6 of its 8 bits)
# --------------------------------------------------------------------------
def gaussian_exponent_entropy(sigma):
    # bf16 exponent e covers |x| in [2^(e-127), 2^(e-126)); round-to-nearest-even
    # moves each boundary down to 2^k (1 - 2^-9).
    def cdf_abs(a):
        return math.erf(a / (sigma * math.sqrt(2)))

    probs = []
    for e in range(1, 240):
        lo = 2.0 ** (e - 127) * (1 - 2 ** -9)
        hi = 2.0 ** (e - 126) * (1 - 2 ** -9)
        probs.append(cdf_abs(hi) - cdf_abs(lo))
    p = np.array([x for x in probs if x > 0])
    p0 = 1 - p.sum()
    if p0 > 0:
        p = np.append(p, p0)
    return float(-(p * np.log2(p)).sum())


def test_gaussian_exponent_entropy_closed_form(oracle_mod):
    H_closed = gaussian_exponent_entropy(0.02)
    assert abs(H_closed - 2.546) < 0.01
    w = inputs.single_matrix()
    exps, _ = oracle_mod.split(w)
    hist = oracle_mod.histogram(exps)
    assert abs(entropy_bits(hist) - H_closed) < 0.005
    f = oracle_mod.build_format(w)
    avg = f["total_bits"] / f["n"]
    assert entropy_bits(hist) <= avg < entropy_bits(hist) + 0.1
    # DF11 size on this input: 8 sign/mantissa bits + ~2.6 exponent bits per
    # weight, about 2/3 of BF16 ("Format DFloat11": ~11 bits per weight)
    assert 0.6 < (8 + avg) / 16 < 0.72
