"""ctypes front end of the CPU oracle (``df11_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product package never
imports this module, and this module never imports the product package.

The steps follow "DFloat11: Kompresi inferensi GPU lossless ..."
(id.news.hada.io/topic?id=20542); each C function names the section it
restates.  ``build_format`` chains them in the page's order: split the BF16
fields, histogram the exponents, Huffman code lengths (capped at 32 bits),
canonical codes, bit-pack EncodedExponent, then the decoder metadata (Gaps,
BlockOffset) and the hierarchical LUTs.

``rans_build_format`` / ``rans_decode_format`` are the rANS variant of the
exponent coder that the page's discussion proposes (range asymmetric numeral
systems from their published definition: quantised frequencies, one 32-bit
state per lane, 16-bit words, each lane its own word stream, blocks of 512 J
elements decoded by 32 lanes in step); sign and mantissa stay verbatim as in
DF11.  Pinned in
``tests/test_rans_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "df11_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdf11_oracle.so")
_lock = threading.Lock()
_lib = None

MAX_CODE_LEN = 32  # "Kernel GPU 2 tahap": the longest code is 32 bits
SEGMENT_BITS = 64  # "Kernel GPU 2 tahap": n = 8 bytes per thread


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc into a shared object next to its source."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-Wall", "-o", tmp, _SRC],
            check=True,
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        U64 = ctypes.c_uint64
        lib.df11o_split.argtypes = [P, U64, P, P]
        lib.df11o_split.restype = ctypes.c_int64
        lib.df11o_histogram.argtypes = [P, U64, P]
        lib.df11o_histogram.restype = None
        lib.df11o_huffman_lengths.argtypes = [P, P]
        lib.df11o_huffman_lengths.restype = ctypes.c_int
        lib.df11o_package_merge.argtypes = [P, ctypes.c_int, P]
        lib.df11o_package_merge.restype = ctypes.c_int
        lib.df11o_code_lengths.argtypes = [P, ctypes.c_int, P]
        lib.df11o_code_lengths.restype = ctypes.c_int
        lib.df11o_canonical_codes.argtypes = [P, P]
        lib.df11o_canonical_codes.restype = None
        lib.df11o_encode.argtypes = [P, U64, P, P, P]
        lib.df11o_encode.restype = U64
        lib.df11o_metadata.argtypes = [P, U64, P, U64, ctypes.c_uint32, P, P]
        lib.df11o_metadata.restype = ctypes.c_int
        lib.df11o_pack_gaps.argtypes = [P, U64, P]
        lib.df11o_pack_gaps.restype = None
        lib.df11o_build_luts.argtypes = [P, P, P, ctypes.POINTER(ctypes.c_int)]
        lib.df11o_build_luts.restype = ctypes.c_int
        lib.df11o_decode.argtypes = [P, U64, P, P, P, U64, P]
        lib.df11o_decode.restype = ctypes.c_int
        lib.df11o_decode_range.argtypes = [P, U64, U64, U64, P, P, P, U64]
        lib.df11o_decode_range.restype = ctypes.c_int64
        lib.df11o_split_all.argtypes = [P, U64, P, P]
        lib.df11o_split_all.restype = None
        lib.df11o_rans_freqs.argtypes = [P, ctypes.c_int, P]
        lib.df11o_rans_freqs.restype = ctypes.c_int
        lib.df11o_rans_encode.argtypes = [P, U64, P, ctypes.c_int, ctypes.c_int, P, U64, P, P, P]
        lib.df11o_rans_encode.restype = ctypes.c_int64
        lib.df11o_rans_decode.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int, U64, P, P]
        lib.df11o_rans_decode.restype = ctypes.c_int
        lib.df11o_rans_step_encode.argtypes = [U64, ctypes.c_int, P, ctypes.c_int, P, P]
        lib.df11o_rans_step_encode.restype = U64
        _lib = lib
        return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


class UnsupportedExponent(ValueError):
    """An element has an exponent in 240..255, the range reserved for LUT
    pointers ("Decoding berbasis LUT hierarkis")."""


def split(w: np.ndarray):
    """BF16 bits -> (exponent bytes, sign/mantissa bytes)."""
    w = np.ascontiguousarray(w, dtype=np.uint16).ravel()
    exps = np.empty(w.size, np.uint8)
    sm = np.empty(w.size, np.uint8)
    bad = _load().df11o_split(_ptr(w), w.size, _ptr(exps), _ptr(sm))
    if bad >= 0:
        raise UnsupportedExponent(f"element {bad} has exponent >= 240")
    return exps, sm


def histogram(exps: np.ndarray) -> np.ndarray:
    exps = np.ascontiguousarray(exps, dtype=np.uint8)
    hist = np.zeros(256, np.uint64)
    _load().df11o_histogram(_ptr(exps), exps.size, _ptr(hist))
    return hist


def huffman_lengths(hist) -> np.ndarray:
    """Plain (uncapped) Huffman code lengths."""
    hist = np.ascontiguousarray(hist, dtype=np.uint64)
    lens = np.zeros(256, np.uint8)
    _load().df11o_huffman_lengths(_ptr(hist), _ptr(lens))
    return lens


def package_merge(hist, max_len: int) -> np.ndarray:
    """Optimal code lengths with every length <= max_len."""
    hist = np.ascontiguousarray(hist, dtype=np.uint64)
    lens = np.zeros(256, np.uint8)
    if _load().df11o_package_merge(_ptr(hist), int(max_len), _ptr(lens)) != 0:
        raise ValueError("no prefix code with this length cap")
    return lens


def code_lengths(hist, max_len: int = MAX_CODE_LEN) -> np.ndarray:
    """The format's code lengths: Huffman, else package-merge at the cap."""
    hist = np.ascontiguousarray(hist, dtype=np.uint64)
    lens = np.zeros(256, np.uint8)
    if _load().df11o_code_lengths(_ptr(hist), int(max_len), _ptr(lens)) < 0:
        raise ValueError("no prefix code with this length cap")
    return lens


def canonical_codes(lens) -> np.ndarray:
    lens = np.ascontiguousarray(lens, dtype=np.uint8)
    codes = np.zeros(256, np.uint32)
    _load().df11o_canonical_codes(_ptr(lens), _ptr(codes))
    return codes


def encode(exps, lens, codes):
    """Returns (stream bytes, total bits); the stream has ceil(bits/8) bytes."""
    exps = np.ascontiguousarray(exps, dtype=np.uint8)
    lens = np.ascontiguousarray(lens, dtype=np.uint8)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    total = int(np.sum(lens[exps].astype(np.uint64))) if exps.size else 0
    stream = np.zeros(max((total + 7) // 8, 1), np.uint8)
    bits = _load().df11o_encode(_ptr(exps), exps.size, _ptr(lens), _ptr(codes), _ptr(stream))
    assert bits == total
    return stream[: (total + 7) // 8], int(bits)


def metadata(exps, lens, total_bits: int, threads_per_block: int):
    """Returns (gaps: one uint8 per segment, block_offset: uint32[nblocks+1])."""
    exps = np.ascontiguousarray(exps, dtype=np.uint8)
    lens = np.ascontiguousarray(lens, dtype=np.uint8)
    nseg = (total_bits + SEGMENT_BITS - 1) // SEGMENT_BITS
    nblocks = (nseg + threads_per_block - 1) // threads_per_block
    gaps = np.zeros(max(nseg, 1), np.uint8)
    offs = np.zeros(nblocks + 1, np.uint32)
    rc = _load().df11o_metadata(
        _ptr(exps), exps.size, _ptr(lens), total_bits, threads_per_block, _ptr(gaps), _ptr(offs)
    )
    if rc != 0:
        raise ValueError("a gap exceeds 31 bits")
    return gaps[:nseg], offs


def pack_gaps(gaps) -> np.ndarray:
    """5-bit fields, LSB-first, into uint64 words (one spare word at the end)."""
    gaps = np.ascontiguousarray(gaps, dtype=np.uint8)
    words = np.zeros((5 * gaps.size + 63) // 64 + 1, np.uint64)
    _load().df11o_pack_gaps(_ptr(gaps), gaps.size, _ptr(words))
    return words


def build_luts(lens, codes):
    """Returns the k x 256 uint8 hierarchical LUTs."""
    lens = np.ascontiguousarray(lens, dtype=np.uint8)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    luts = np.zeros(17 * 256, np.uint8)
    k = ctypes.c_int(0)
    rc = _load().df11o_build_luts(_ptr(lens), _ptr(codes), _ptr(luts), ctypes.byref(k))
    if rc == -2:
        raise ValueError("more than 16 child LUTs")
    if rc != 0:
        raise ValueError("code lengths do not form a prefix code")
    return luts[: k.value * 256].reshape(k.value, 256).copy()


def decode(stream, total_bits: int, lens, codes, sm, n: int) -> np.ndarray:
    """Bit-by-bit tree-walk decode back to BF16 bits (uint16)."""
    stream = np.ascontiguousarray(stream, dtype=np.uint8)
    if stream.size == 0:
        stream = np.zeros(1, np.uint8)
    lens = np.ascontiguousarray(lens, dtype=np.uint8)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    sm = np.ascontiguousarray(sm, dtype=np.uint8)
    if sm.size == 0:
        sm = np.zeros(1, np.uint8)
    out = np.empty(max(n, 1), np.uint16)
    rc = _load().df11o_decode(
        _ptr(stream), total_bits, _ptr(lens), _ptr(codes), _ptr(sm), n, _ptr(out)
    )
    if rc != 0:
        raise ValueError("stream is inconsistent with the code")
    return out[:n]


def decode_range(stream, stream_bits: int, start_bit: int, end_bit: int, lens, codes) -> np.ndarray:
    """Exponents of the codes that start in [start_bit, end_bit)."""
    stream = np.ascontiguousarray(stream, dtype=np.uint8)
    lens = np.ascontiguousarray(lens, dtype=np.uint8)
    codes = np.ascontiguousarray(codes, dtype=np.uint32)
    cap = max(end_bit - start_bit, 1)
    out = np.empty(cap, np.uint8)
    cnt = _load().df11o_decode_range(
        _ptr(stream), stream_bits, start_bit, end_bit, _ptr(lens), _ptr(codes), _ptr(out), cap
    )
    if cnt < 0:
        raise ValueError("stream is inconsistent with the code")
    return out[:cnt].copy()


def build_format(w: np.ndarray, threads_per_block: int = 64, max_len: int = MAX_CODE_LEN) -> dict:
    """All DF11 arrays for one stream of BF16 bits, built step by step."""
    exps, sm = split(w)
    hist = histogram(exps)
    lens = code_lengths(hist, max_len)
    codes = canonical_codes(lens)
    stream, total_bits = encode(exps, lens, codes)
    gaps, offs = metadata(exps, lens, total_bits, threads_per_block)
    luts = build_luts(lens, codes)
    return {
        "n": int(exps.size),
        "hist": hist,
        "code_lengths": lens,
        "codes": codes,
        "encoded_exponent": stream,
        "total_bits": total_bits,
        "packed_sign_mantissa": sm,
        "gaps": gaps,
        "gaps_packed": pack_gaps(gaps),
        "block_offset": offs,
        "luts": luts,
        "threads_per_block": threads_per_block,
    }


def decode_format(fmt: dict) -> np.ndarray:
    return decode(
        fmt["encoded_exponent"], fmt["total_bits"], fmt["code_lengths"], fmt["codes"],
        fmt["packed_sign_mantissa"], fmt["n"],
    )


# ------------------------------------------------------------------ rANS
# The rANS variant of the exponent coder (the page's discussion proposes rANS
# as the SIMD-friendlier entropy coder); the C side states the model and the
# layout.
RANS_PROB_BITS = 12
RANS_CHUNKS = 10  # J: chunks of 16 elements per lane and block (5120 elements per block)
RANS_L = 1 << 16


def rans_freqs(hist, prob_bits: int = RANS_PROB_BITS) -> np.ndarray:
    hist = np.ascontiguousarray(hist, dtype=np.uint64)
    freq = np.zeros(256, np.uint32)
    if _load().df11o_rans_freqs(_ptr(hist), prob_bits, _ptr(freq)) != 0:
        raise ValueError("no symbol, or more symbols than the precision allows")
    return freq


def rans_encode(exps, freq, prob_bits: int = RANS_PROB_BITS, chunks: int = RANS_CHUNKS):
    """-> (words uint16, states uint32 [nblocks, 32], offsets uint64 [nblocks + 1],
    lane_words uint8 [nblocks, 32]); words of a block: lane 0's stream, then
    lane 1's, ..."""
    exps = np.ascontiguousarray(exps, dtype=np.uint8)
    freq = np.ascontiguousarray(freq, dtype=np.uint32)
    n = exps.size
    B = 512 * chunks
    nblocks = (n + B - 1) // B
    words = np.zeros(max(n, 1), np.uint16)
    states = np.zeros(max(32 * nblocks, 1), np.uint32)
    offsets = np.zeros(nblocks + 1, np.uint64)
    lane_words = np.zeros(max(32 * nblocks, 1), np.uint8)
    src = exps if n else np.zeros(1, np.uint8)
    got = _load().df11o_rans_encode(_ptr(src), n, _ptr(freq), prob_bits, chunks, _ptr(words), words.size,
                                    _ptr(states), _ptr(offsets), _ptr(lane_words))
    if got < 0:
        raise ValueError("rANS encode failed")
    return (words[:got].copy(), states[: 32 * nblocks].reshape(nblocks, 32).copy(), offsets,
            lane_words[: 32 * nblocks].reshape(nblocks, 32).copy())


def rans_decode(words, states, offsets, lane_words, freq, sm, n: int, prob_bits: int = RANS_PROB_BITS,
                chunks: int = RANS_CHUNKS) -> np.ndarray:
    words = np.ascontiguousarray(words, dtype=np.uint16)
    if words.size == 0:
        words = np.zeros(1, np.uint16)
    states = np.ascontiguousarray(states, dtype=np.uint32).reshape(-1)
    if states.size == 0:
        states = np.zeros(1, np.uint32)
    offsets = np.ascontiguousarray(offsets, dtype=np.uint64)
    lane_words = np.ascontiguousarray(lane_words, dtype=np.uint8).reshape(-1)
    if lane_words.size == 0:
        lane_words = np.zeros(1, np.uint8)
    freq = np.ascontiguousarray(freq, dtype=np.uint32)
    sm = np.ascontiguousarray(sm, dtype=np.uint8)
    if sm.size == 0:
        sm = np.zeros(1, np.uint8)
    out = np.empty(max(n, 1), np.uint16)
    rc = _load().df11o_rans_decode(_ptr(words), _ptr(states), _ptr(offsets), _ptr(lane_words), _ptr(freq),
                                   prob_bits, chunks, n, _ptr(sm), _ptr(out))
    if rc != 0:
        raise ValueError("rANS data inconsistent")
    return out[:n]


def rans_step_encode(x: int, s: int, freq, prob_bits: int):
    """One encode step of one state -> (new state, emitted word or None)."""
    freq = np.ascontiguousarray(freq, dtype=np.uint32)
    word = ctypes.c_uint32(0)
    emitted = ctypes.c_int(0)
    y = _load().df11o_rans_step_encode(x, s, _ptr(freq), prob_bits, ctypes.byref(word), ctypes.byref(emitted))
    return int(y), (int(word.value) if emitted.value else None)


def split_all(w: np.ndarray):
    """BF16 bits -> (exponent bytes, sign/mantissa bytes), every exponent
    allowed (the rANS variant needs no pointer values)."""
    w = np.ascontiguousarray(w, dtype=np.uint16).ravel()
    exps = np.empty(w.size, np.uint8)
    sm = np.empty(w.size, np.uint8)
    if w.size:
        _load().df11o_split_all(_ptr(w), w.size, _ptr(exps), _ptr(sm))
    return exps, sm


def rans_build_format(w: np.ndarray, prob_bits: int = RANS_PROB_BITS, chunks: int = RANS_CHUNKS) -> dict:
    """All arrays of the rANS variant for one stream of BF16 bits."""
    exps, sm = split_all(w)
    hist = histogram(exps)
    freq = rans_freqs(hist, prob_bits) if exps.size else np.zeros(256, np.uint32)
    words, states, offsets, lane_words = rans_encode(exps, freq, prob_bits, chunks) if exps.size else (
        np.zeros(0, np.uint16), np.zeros((0, 32), np.uint32), np.zeros(1, np.uint64), np.zeros((0, 32), np.uint8))
    return {"n": int(exps.size), "hist": hist, "freq": freq, "words": words, "states": states,
            "offsets": offsets, "lane_words": lane_words, "packed_sign_mantissa": sm, "prob_bits": prob_bits,
            "chunks": chunks}


def rans_decode_format(fmt: dict) -> np.ndarray:
    if fmt["n"] == 0:
        return np.zeros(0, np.uint16)
    return rans_decode(fmt["words"], fmt["states"], fmt["offsets"], fmt["lane_words"], fmt["freq"],
                       fmt["packed_sign_mantissa"], fmt["n"], fmt["prob_bits"], fmt["chunks"])
