"""The library's host-side format builder against the CPU oracle (no GPU).

Both sides compress the same seeded inputs independently; every array of the
format must agree byte for byte: CodeLengths, EncodedExponent (with its zero
padding), PackedSignMantissa, the packed 5-bit Gaps, BlockOffset and the
hierarchical LUTs.  Also checks the exported C ABI and its error codes.
"""
import ctypes

import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs


def compare(fmt, ref):
    a = fmt.arrays()
    s = fmt.scalars()
    n = ref["n"]
    assert s["n"] == n
    assert s["total_bits"] == ref["total_bits"]
    assert np.array_equal(a["code_lengths"], ref["code_lengths"])
    nbytes = (ref["total_bits"] + 7) // 8
    assert np.array_equal(a["encoded_exponent"][:nbytes], ref["encoded_exponent"])
    assert not a["encoded_exponent"][nbytes:].any()
    T = s["threads_per_block"]
    assert a["encoded_exponent"].size == s["num_blocks"] * T * 8 + 16
    assert np.array_equal(a["packed_sign_mantissa"][:n], ref["packed_sign_mantissa"])
    assert not a["packed_sign_mantissa"][n:].any()
    g_ref = ref["gaps_packed"]
    g = a["gaps"]
    m = min(g.size, g_ref.size)
    assert np.array_equal(g[:m], g_ref[:m])
    assert not g[m:].any() and not g_ref[m:].any()
    assert np.array_equal(a["block_offset"], ref["block_offset"])
    assert np.array_equal(a["luts"], ref["luts"])
    assert s["num_segments"] == len(ref["gaps"])
    assert s["max_code_len"] == int(ref["code_lengths"].max()) if n else True
    used = ref["code_lengths"][ref["code_lengths"] > 0]
    assert s["min_code_len"] == (int(used.min()) if used.size else 0)
    offs = ref["block_offset"].astype(np.int64)
    assert s["max_block_elems"] == (int(np.diff(offs).max()) if offs.size > 1 else 0)


@pytest.mark.parametrize("n", [0, 1, 2, 7, 63, 64, 65, 1000, 32 * 25 - 1, 32 * 25, 32 * 25 + 1, 256 * 25 + 1, 100_003])
def test_gaussian_sizes(oracle_mod, n):
    w = inputs.gaussian(n, [11, n])
    compare(df11.build_format(w), oracle_mod.build_format(w, 64))


@pytest.mark.parametrize("T", [32, 64, 128, 256, 512, 1024])
def test_threads_per_block(oracle_mod, T):
    w = inputs.gaussian(50_000, [12, T])
    compare(df11.build_format(w, T), oracle_mod.build_format(w, T))


def test_stress_distribution(oracle_mod):
    w = inputs.stress(1 << 20, key=(3, 9, 9))
    fmt = df11.build_format(w)
    compare(fmt, oracle_mod.build_format(w, 64))
    info = fmt.info()
    assert info["max_code_len"] >= 18 and info["num_luts"] >= 3


def test_chunk_boundaries_many_threads(oracle_mod):
    # > 4 Mi elements: the encoder splits work into several chunks whose
    # boundary bytes are shared
    w = inputs.gaussian((1 << 22) * 2 + 12345, [13, 0])
    compare(df11.build_format(w), oracle_mod.build_format(w, 64))


def test_every_bf16_pattern(oracle_mod):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ok = allbits[((allbits >> 7) & 0xFF) < 240]
    w = np.random.default_rng(3).permutation(ok)
    compare(df11.build_format(w), oracle_mod.build_format(w, 64))


def test_single_symbol(oracle_mod):
    w = np.full(5000, 0x3F80, np.uint16)
    w[::7] = 0xBF80  # sign differs, exponent the same
    fmt = df11.build_format(w)
    compare(fmt, oracle_mod.build_format(w, 64))
    assert fmt.info()["max_code_len"] == 1


def test_length_limited_code(oracle_mod):
    f = [1, 1]
    while len(f) < 34:
        f.append(f[-1] + f[-2])
    exps = np.repeat(np.arange(34, dtype=np.uint16) + 60, f)
    exps = np.random.default_rng(5).permutation(exps)
    w = (exps << 7).astype(np.uint16)
    fmt = df11.build_format(w)
    ref = oracle_mod.build_format(w, 64)
    compare(fmt, ref)
    assert fmt.info()["max_code_len"] == 32


def test_multi_matrix_equals_concatenation(oracle_mod):
    mats = [inputs.gaussian(n, [14, n]) for n in (1000, 0, 4097, 33)]
    fmt = df11.build_format(mats)
    compare(fmt, oracle_mod.build_format(np.concatenate(mats), 64))


def test_info_statistics(oracle_mod):
    w = inputs.single_matrix()
    info = df11.build_format(w).info()
    h = info["histogram"].astype(np.float64)
    p = h[h > 0] / h.sum()
    assert abs(info["entropy_bits"] - float(-(p * np.log2(p)).sum())) < 1e-9
    assert info["distinct_exponents"] == int((h > 0).sum())
    assert info["entropy_bits"] <= info["avg_code_len"] < info["entropy_bits"] + 1


# ------------------------------------------------------------------ errors
def test_rejects_pointer_exponents():
    w = inputs.gaussian(100, [15])
    w[50] = 0x7F80  # +Inf, exponent 255
    with pytest.raises(df11.Df11Error) as e:
        df11.build_format(w)
    assert e.value.status == 2


@pytest.mark.parametrize("T", [1, 31, 48, 2048])
def test_rejects_bad_threads_per_block(T):
    with pytest.raises(df11.Df11Error) as e:
        df11.build_format(inputs.gaussian(100, [16]), T)
    assert e.value.status == 1


def test_rejects_too_many_luts():
    exps = np.arange(239, dtype=np.uint16)
    counts = np.ones(239, np.int64)
    counts[:4] = 1000
    w = (np.repeat(exps, counts) << 7).astype(np.uint16)
    with pytest.raises(df11.Df11Error) as e:
        df11.build_format(w)
    assert e.value.status == 4


def test_null_arguments():
    lib = df11.load_library()
    out = ctypes.c_void_p()
    assert lib.df11_build_format(None, None, 1, 256, ctypes.byref(out)) == 1
    assert lib.df11_build_format(None, None, 0, 256, None) == 1
    assert lib.df11_format_arrays(None, None) == 1
    lib.df11_free(None)


@pytest.mark.parametrize("case", ["gauss", "stress", "one_symbol", "two_symbols"])
def test_symbol_table_against_the_oracle_code(oracle_mod, case):
    # the decoders' derived table that df11_build_format stores with a stream:
    # for every 12-bit window, the first up to three whole codes inside it
    # (exponents rotated right by one bit), their count and total length --
    # checked by prefix matching against the oracle's canonical code
    w = {"gauss": lambda: inputs.gaussian(200_000, [120]),
         "stress": lambda: inputs.stress(200_000, key=(121, 0)),
         "one_symbol": lambda: np.full(5000, 0x3F80, np.uint16),
         "two_symbols": lambda: np.array([0x3F80, 0x4000] * 2500, np.uint16)}[case]()
    fmt = df11.build_format(w)
    a = fmt.arrays()
    tab = a["symbol_table"]
    assert tab.size == 4096
    lens = a["code_lengths"].astype(np.int64)
    codes = oracle_mod.canonical_codes(a["code_lengths"]).astype(np.int64)
    syms = [s for s in range(256) if lens[s]]
    complete = sum(2.0 ** -lens[s] for s in syms) == 1.0
    for i in range(4096):
        if not complete and i != 0:
            # an incomplete code (one exponent: the code 0, Kraft sum 1/2):
            # a valid stream is all zeros; the unused LUT entries repeat the
            # symbol, so other windows are never decoded
            continue
        bits, found = 0, []
        while len(found) < 3:
            hit = [s for s in syms if bits + lens[s] <= 12
                   and (i >> (12 - bits - lens[s])) & ((1 << lens[s]) - 1) == codes[s]]
            if not hit:
                break
            assert len(hit) == 1  # prefix code
            found.append(hit[0])
            bits += lens[hit[0]]
        e = int(tab[i])
        assert e >> 29 == len(found) and (e >> 24) & 31 == bits, i
        for j, s in enumerate(found):
            assert (e >> (8 * j)) & 0xFF == ((s >> 1) | (s << 7)) & 0xFF, (i, j)
        assert e & (0xFFFFFF >> (8 * (3 - len(found)))) == e & 0xFFFFFF  # unused bytes are zero
    # the exported function gives the same table
    out = np.zeros(4096, np.uint32)
    lib = df11.load_library()
    assert lib.df11_symbol_table(a["luts"].ctypes.data, a["code_lengths"].ctypes.data,
                                 fmt.scalars()["num_luts"], out.ctypes.data) == 0
    assert np.array_equal(out, tab)
    assert lib.df11_symbol_table(None, a["code_lengths"].ctypes.data, 1, out.ctypes.data) == 1
