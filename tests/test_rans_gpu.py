"""GPU decoder of the rANS variant (df11_rans_decompress) against the
original bits and the CPU oracle's decode, through the C ABI."""
import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs

pytestmark = pytest.mark.gpu


def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def gpu_decode(w, chunks=10, out=None):
    torch = torch_cuda()
    fmt = df11.rans_build_format(w, chunks)
    dev = df11.RansDeviceFormat(fmt, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = df11.rans_decompress(dev, out, status)
    assert df11.read_status(status) == 0
    return got[: w.size].view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("n", [1, 15, 16, 17, 511, 512, 4095, 4096, 4097, 3 * 4096 + 100, 1_000_003])
def test_round_trip_against_the_oracle(oracle_mod, n):
    w = inputs.gaussian(n, [100, n])
    got = gpu_decode(w)
    assert np.array_equal(got, w)
    ref = oracle_mod.rans_decode_format(oracle_mod.rans_build_format(w))
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("chunks", [1, 2, 8, 15])
def test_chunks(chunks):
    w = inputs.stress(300_007, key=(101, chunks))
    assert np.array_equal(gpu_decode(w, chunks), w)


def test_every_pattern_and_one_symbol():
    rng = np.random.default_rng(102)
    allp = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    rng.shuffle(allp)
    assert np.array_equal(gpu_decode(np.tile(allp, 5)), np.tile(allp, 5))
    one = np.full(50_001, 0xBF80, np.uint16)
    assert np.array_equal(gpu_decode(one), one)


def test_output_alignment_and_neighbours():
    torch = torch_cuda()
    w = inputs.gaussian(70_011, [103])
    for shift in (0, 8):  # 32-byte and 16-byte aligned outputs
        buf = torch.full((w.size + 64,), -1, dtype=torch.int16, device="cuda")
        out = buf[shift: shift + w.size].view(torch.bfloat16)
        gpu_decode(w, 8, out)
        host = buf.cpu().numpy().view(np.uint16)
        assert np.array_equal(host[shift: shift + w.size], w)
        assert np.all(host[:shift] == 0xFFFF) and np.all(host[shift + w.size:] == 0xFFFF)


@pytest.mark.parametrize("workload", [2, 3])
def test_workloads(workload):
    mats = [m for _, _, m in inputs.workload_arrays(workload, 0)]
    w = np.concatenate(mats) if len(mats) > 1 else mats[0]
    assert np.array_equal(gpu_decode(w), w)


def test_corruption_is_reported():
    torch = torch_cuda()
    w = inputs.gaussian(200_000, [104])
    fmt = df11.rans_build_format(w)
    for name, edit in (("states", lambda t: t.view(torch.int32).__setitem__(5, 12345)),
                       ("block_word", lambda t: t.view(torch.int32).__setitem__(3, int(t.view(torch.int32)[3]) + 1)),
                       ("freq", lambda t: t.view(torch.int16).__setitem__(120, 7))):
        dev = df11.RansDeviceFormat(fmt, "cuda")
        edit(dev.tensors[name])
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.rans_decompress(dev, None, status)
        assert df11.read_status(status) != 0, name


def test_inconsistent_offsets_and_states_stay_in_bounds():
    # offsets far past the word array or going backwards, states of 0 (every
    # step then takes a word), lane counts that do not match the streams: the
    # copies are clamped to the array and the buffer, each lane's start to the
    # copied words (a block reads at most 240 more words per lane, inside the
    # buffer's slack), and the launch reports the block as corrupt
    torch = torch_cuda()
    w = inputs.gaussian(20 * 4096 + 77, [106])
    fmt = df11.rans_build_format(w)

    def far(t):
        t.view(torch.int32)[3] = 0x7FFFFFF0

    def backwards(t):
        t.view(torch.int32)[4] = 0

    def zero_states(t):
        t.view(torch.int32)[64:96] = 0
        t.view(torch.int32)[-32:] = 0  # the partial last block too

    def lane_counts_off(t):
        t[64] = 255  # lane 0 of block 2: a stream that runs past the block's words
        t[97] = 0  # lane 1 of block 3: a stream cut short

    for name, edit in (("block_word", far), ("block_word", backwards), ("states", zero_states),
                       ("lane_words", lane_counts_off)):
        dev = df11.RansDeviceFormat(fmt, "cuda")
        edit(dev.tensors[name])
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = df11.rans_decompress(dev, None, status)
        torch.cuda.synchronize()
        assert df11.read_status(status) != 0, name
        # blocks that were not touched still decode
        got = out.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got[:2 * 4096], w[:2 * 4096])


def _with_high_entropy_runs(seed):
    # Gaussian weights with runs of uniformly random bit patterns (every
    # exponent about equally likely, ~8 bits each): blocks of those runs need
    # ~2,600 words, more than a warp buffer holds at 32 warps per CTA, and
    # take the decoder's global-memory path; the stream ends inside such a run
    rng = np.random.default_rng(seed)
    parts = [inputs.gaussian(100_000, [seed, 1]), rng.integers(0, 1 << 16, 30_000, dtype=np.uint32).astype(np.uint16),
             inputs.gaussian(50_000, [seed, 2]), rng.integers(0, 1 << 16, 7_001, dtype=np.uint32).astype(np.uint16)]
    return np.concatenate(parts)


def test_blocks_larger_than_the_word_buffer():
    w = _with_high_entropy_runs(107)
    fmt = df11.rans_build_format(w)
    assert fmt.scalars()["max_block_words"] > 2400
    assert np.array_equal(gpu_decode(w), w)


def test_inconsistent_large_blocks_stay_in_bounds():
    # lane counts that do not match, on blocks read from global memory: each
    # lane's start is clamped so that its reads stay inside the word array,
    # and the launch reports the block as corrupt
    torch = torch_cuda()
    w = _with_high_entropy_runs(108)
    fmt = df11.rans_build_format(w)
    bw = np.diff(fmt.arrays()["block_word"].astype(np.int64))
    big = int(np.argmax(bw))
    assert bw[big] > 2400

    def lane_counts_off(t):
        t[32 * big] = 255
        t[32 * big + 1] = 0

    def states_off(t):
        t.view(torch.int32)[32 * big: 32 * big + 32] = 0

    for name, edit in (("lane_words", lane_counts_off), ("states", states_off)):
        dev = df11.RansDeviceFormat(fmt, "cuda")
        edit(dev.tensors[name])
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = df11.rans_decompress(dev, None, status)
        torch.cuda.synchronize()
        assert df11.read_status(status) != 0, name
        got = out.view(torch.int16).cpu().numpy().view(np.uint16)
        B = 5120
        assert np.array_equal(got[:B * big], w[:B * big])


def test_repeated_launches_are_identical():
    torch = torch_cuda()
    w = inputs.gaussian(1 << 20, [105])
    dev = df11.RansDeviceFormat(df11.rans_build_format(w), "cuda")
    a = df11.rans_decompress(dev)
    b = df11.rans_decompress(dev)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
