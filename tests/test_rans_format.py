"""The library's host builder of the rANS variant against the oracle (no GPU).

Both sides quantise the model and encode the same seeded inputs
independently (library: df11_rans_format.cpp, oracle: df11_oracle.c); every
array must agree element for element: frequencies, block word offsets, start
states, lane counts, the word sequence (each lane's stream in turn; the
library pads it with 8 zero words) and the sign/mantissa bytes.
"""
import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs


def compare(w, chunks, oracle_mod):
    fmt = df11.rans_build_format(w, chunks)
    ref = oracle_mod.rans_build_format(w, 12, chunks)
    a, s = fmt.arrays(), fmt.scalars()
    n = ref["n"]
    assert s["n"] == n and s["prob_bits"] == 12 and s["chunks"] == chunks
    if n == 0:
        assert s["num_blocks"] == 0 and s["num_words"] == 0
        return fmt
    assert np.array_equal(a["freq"].astype(np.uint32), ref["freq"])
    assert np.array_equal(a["block_word"].astype(np.uint64), ref["offsets"])
    assert np.array_equal(a["states"].reshape(-1, 32), ref["states"])
    assert np.array_equal(a["lane_words"].reshape(-1, 32), ref["lane_words"])
    nw = ref["words"].size
    assert s["num_words"] == nw
    assert np.array_equal(a["words"][:nw], ref["words"]) and not a["words"][nw:].any()
    assert np.array_equal(a["packed_sign_mantissa"][:n], ref["packed_sign_mantissa"])
    assert not a["packed_sign_mantissa"][n:].any()
    assert s["max_block_words"] == int(np.diff(ref["offsets"].astype(np.int64)).max())
    return fmt


@pytest.mark.parametrize("n", [0, 1, 15, 16, 511, 512, 4095, 4096, 4097, 3 * 4096 + 100, 100_003])
def test_gaussian_sizes(oracle_mod, n):
    w = inputs.gaussian(n, [60, n]) if n else np.zeros(0, np.uint16)
    compare(w, 8, oracle_mod)


@pytest.mark.parametrize("chunks", [1, 2, 8, 15])
def test_chunks(oracle_mod, chunks):
    compare(inputs.stress(70_001, key=(61, chunks)), chunks, oracle_mod)


def test_every_pattern_and_one_symbol(oracle_mod):
    rng = np.random.default_rng(62)
    allp = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    rng.shuffle(allp)
    compare(allp, 8, oracle_mod)  # exponents 240..255 included
    compare(np.full(20_000, 0x4011, np.uint16), 8, oracle_mod)


def test_multi_matrix_equals_concatenation(oracle_mod):
    a, b = inputs.gaussian(5000, [63]), inputs.stress(7001, key=(64, 0))
    one = df11.rans_build_format(np.concatenate([a, b]))
    two = df11.rans_build_format([a, b])
    for k in one.arrays():
        assert np.array_equal(one.arrays()[k], two.arrays()[k])


def test_rejects_bad_arguments():
    import ctypes

    lib = df11.load_library()
    h = ctypes.c_void_p()
    w = np.zeros(10, np.uint16)
    ptrs = (ctypes.c_void_p * 1)(w.ctypes.data)
    counts = (ctypes.c_uint64 * 1)(10)
    assert lib.df11_rans_build(ptrs, counts, 1, 16, ctypes.byref(h)) == 1  # chunks > 15
    assert lib.df11_rans_build(ptrs, counts, 1, 8, None) == 1
    assert lib.df11_rans_decompress(None, None, None, None) == 1
