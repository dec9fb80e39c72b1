"""Compression of device-resident weights (df11_device_histogram,
df11_plan_from_histogram, df11_device_encode) must produce exactly the stream
df11_build_format builds on the host from the same elements: same code,
same bytes in every array ("Format DFloat11", "Kernel GPU 2 tahap dan
metadata bantu").  The host builder itself is checked byte for byte against
the oracle in test_host_format.py."""
import ctypes

import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs


def _hist(w):
    return np.bincount((np.asarray(w, np.uint16) >> 7) & 0xFF, minlength=256).astype(np.uint64)


def _plan(hist, T=64):
    lib = df11.load_library()
    h = ctypes.c_void_p()
    st = lib.df11_plan_from_histogram(np.ascontiguousarray(hist, np.uint64).ctypes.data, T, ctypes.byref(h))
    if st:
        raise df11.Df11Error(st, "df11_plan_from_histogram")
    return df11.Format(h.value, lib)


def _fibonacci_bits(k=34, seed=5):
    # exponent s appears F(s+1) times: the plain Huffman tree is k-1 deep, so
    # the code is length-limited to 32 by package-merge
    f = [1, 1]
    while len(f) < k:
        f.append(f[-1] + f[-2])
    e = np.repeat(np.arange(k, dtype=np.uint16), f[:k])
    rng = np.random.default_rng(seed)
    rng.shuffle(e)
    return (e << 7) | rng.integers(0, 128, e.size, dtype=np.uint16) | (rng.integers(0, 2, e.size, dtype=np.uint16) << 15)


CASES = {
    "gauss_100003": lambda: inputs.gaussian(100_003, [80]),
    "gauss_1Mi": lambda: inputs.gaussian(1 << 20, [81]),
    "stress_3M": lambda: inputs.stress(3_000_017, key=(82, 0, 0)),
    "single_symbol": lambda: np.full(50_001, 0x3F80, np.uint16),
    "all_patterns": lambda: np.random.default_rng(83).permutation(
        np.array([v for v in range(1 << 16) if ((v >> 7) & 0xFF) < 240], np.uint16)),
}


# ------------------------------------------------------------------- host
@pytest.mark.parametrize("name", ["gauss_100003", "stress_3M", "single_symbol", "all_patterns"])
@pytest.mark.parametrize("T", [32, 64, 256])
def test_plan_matches_builder(name, T):
    w = CASES[name]()
    fmt = df11.build_format(w, T)
    plan = _plan(_hist(w), T)
    a, b = fmt.arrays(), plan.arrays()
    assert np.array_equal(a["code_lengths"], b["code_lengths"])
    assert np.array_equal(a["luts"], b["luts"])
    sa, sb = fmt.scalars(), plan.scalars()
    for k in ("n", "total_bits", "num_segments", "threads_per_block", "num_blocks", "num_luts", "max_code_len"):
        assert sa[k] == sb[k], k
    assert sb["max_block_elems"] == 0
    pa, pb = fmt.c_arrays, plan.c_arrays
    assert pa.encoded_exponent_bytes == pb.encoded_exponent_bytes
    assert pa.packed_sign_mantissa_bytes == pb.packed_sign_mantissa_bytes
    assert pa.gaps_words == pb.gaps_words
    assert b["encoded_exponent"].size == 0 and b["gaps"].size == 0  # a plan holds no element arrays


def test_plan_of_fibonacci_counts_is_length_limited():
    w = _fibonacci_bits()
    plan = _plan(_hist(w))
    assert plan.scalars()["max_code_len"] == 32
    assert np.array_equal(plan.arrays()["code_lengths"], df11.build_format(w).arrays()["code_lengths"])


def test_plan_errors():
    hist = np.zeros(256, np.uint64)
    hist[240] = 1
    with pytest.raises(df11.Df11Error) as e:
        _plan(hist)
    assert e.value.status == 2  # DF11_ERR_UNSUPPORTED_EXPONENT
    hist = np.zeros(256, np.uint64)
    hist[120] = 1 << 32
    with pytest.raises(df11.Df11Error) as e:
        _plan(hist)
    assert e.value.status == 3  # DF11_ERR_TOO_LARGE
    with pytest.raises(df11.Df11Error):
        _plan(np.ones(256, np.uint64) * (np.arange(256) < 200), T=48)


def test_scratch_words():
    lib = df11.load_library()
    assert lib.df11_device_encode_scratch_words(0) == 1
    assert lib.df11_device_encode_scratch_words(1) == 2
    assert lib.df11_device_encode_scratch_words(8192) == 2
    assert lib.df11_device_encode_scratch_words(8193) == 3


# ------------------------------------------------------------------- device
def _torch():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _device_vs_host(w, T=64):
    torch = _torch()
    wt = torch.from_numpy(np.ascontiguousarray(w, np.uint16).view(np.int16)).cuda()
    devfmt, plan = df11.encode_device(wt, T)
    fmt = df11.build_format(w, T)
    ref = fmt.arrays()
    for name, t in devfmt.tensors.items():
        got = t.cpu().numpy()
        want = np.ascontiguousarray(ref[name]).reshape(-1).view(np.uint8)
        assert got.size == want.size, name
        assert np.array_equal(got, want), name
    assert devfmt.scalars == fmt.scalars()
    return devfmt


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 2, 31, 32, 33, 63, 64, 65, 1000, 8191, 8192, 8193, 16384 + 5, 77_777])
def test_device_encode_small_sizes(n):
    _device_vs_host(inputs.gaussian(n, [84, n]))


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("T", [32, 64])
def test_device_encode_matches_host(name, T):
    _device_vs_host(CASES[name](), T)


@pytest.mark.gpu
@pytest.mark.parametrize("T", [96, 128, 256, 1024])
def test_device_encode_other_block_sizes(T):
    # the format allows any multiple of 32 (the decoder takes 32 or 64): the
    # BlockOffset of every T-th segment must still land where the host puts it
    _device_vs_host(inputs.gaussian(1_000_003, [88, T]), T)


@pytest.mark.gpu
def test_device_encode_length_limited_code():
    _device_vs_host(_fibonacci_bits())


@pytest.mark.gpu
def test_device_encoded_stream_decodes():
    torch = _torch()
    w = inputs.gaussian(2_000_003, [85])
    devfmt = _device_vs_host(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = df11.decompress(devfmt, None, status)
    assert df11.read_status(status) == 0
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), w)


@pytest.mark.gpu
def test_device_encode_empty():
    torch = _torch()
    devfmt, plan = df11.encode_device(torch.zeros(0, dtype=torch.int16, device="cuda"))
    assert devfmt.n == 0 and plan.scalars()["total_bits"] == 0


@pytest.mark.gpu
def test_device_encode_reports_elements_that_do_not_match_the_plan():
    # a plan from one array's counts, elements of another: exponents without
    # a code and another total bit count are reported, nothing is written
    # out of bounds
    torch = _torch()
    lib = df11.load_library()
    a = inputs.gaussian(50_000, [86])
    b = a.copy()
    b[::7] = 0x4F00  # exponent 158: absent from a
    plan = _plan(_hist(a))
    pa = plan.c_arrays
    wt = torch.from_numpy(b.view(np.int16)).cuda()
    bufs = {
        "encoded_exponent": torch.zeros(pa.encoded_exponent_bytes, dtype=torch.uint8, device="cuda"),
        "packed_sign_mantissa": torch.zeros(pa.packed_sign_mantissa_bytes, dtype=torch.uint8, device="cuda"),
        "gaps": torch.zeros(pa.gaps_words * 8, dtype=torch.uint8, device="cuda"),
        "block_offset": torch.zeros(4 * (pa.num_blocks + 1), dtype=torch.uint8, device="cuda"),
        "luts": torch.zeros(256 * pa.num_luts, dtype=torch.uint8, device="cuda"),
        "code_lengths": torch.zeros(256, dtype=torch.uint8, device="cuda"),
    }
    dst = df11.df11_arrays()
    dst.encoded_exponent = bufs["encoded_exponent"].data_ptr()
    dst.encoded_exponent_bytes = pa.encoded_exponent_bytes
    dst.packed_sign_mantissa = bufs["packed_sign_mantissa"].data_ptr()
    dst.packed_sign_mantissa_bytes = pa.packed_sign_mantissa_bytes
    dst.gaps = bufs["gaps"].data_ptr()
    dst.gaps_words = pa.gaps_words
    dst.block_offset = bufs["block_offset"].data_ptr()
    dst.luts = bufs["luts"].data_ptr()
    dst.code_lengths = bufs["code_lengths"].data_ptr()
    words = lib.df11_device_encode_scratch_words(b.size)
    scratch = torch.empty(words, dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    maxb = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    st = lib.df11_device_encode(plan._h, ctypes.c_void_p(wt.data_ptr()), ctypes.byref(dst),
                                ctypes.c_void_p(scratch.data_ptr()), words, ctypes.c_void_p(maxb.data_ptr()),
                                ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(s.cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert int(status.item()) != 0
    # too little scratch is refused before anything runs
    st = lib.df11_device_encode(plan._h, ctypes.c_void_p(wt.data_ptr()), ctypes.byref(dst),
                                ctypes.c_void_p(scratch.data_ptr()), words - 1, ctypes.c_void_p(maxb.data_ptr()),
                                ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(s.cuda_stream))
    assert st == 1  # DF11_ERR_INVALID_ARG
