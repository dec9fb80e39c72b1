"""GPU parity: the sm_100a decoder, called through the C ABI, against the CPU
oracle and against the original BF16 bits (DF11 is lossless: "Format
DFloat11" / "Hasil evaluasi" -- outputs are bit-identical).

Small and mid-size cases compare every element with the oracle's own
tree-walk decode of its own format (built independently from the same seeded
input).  Full-size workloads compare every element with the original bits
and a sample of blocks with the oracle's decode of that block's bit range.
Corrupted inputs must raise the status word, never fault or hang: each
corruption below stays inside the bounds the kernel checks (5-bit gaps,
bounded loops, offset/capacity checks, LUT pointer range).
"""
import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs

pytestmark = pytest.mark.gpu


def torch_cuda():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def gpu_decode(mats, T=64, dev_fmt=None):
    torch = torch_cuda()
    fmt = df11.build_format(mats, T)
    dev = dev_fmt or df11.DeviceFormat(fmt, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((max(dev.n, 1),), float("nan"), dtype=torch.bfloat16, device="cuda")
    df11.decompress(dev, out, status)
    st = df11.read_status(status)
    got = out[: dev.n].view(torch.int16).cpu().numpy().view(np.uint16)
    return got, st, fmt


def check_against_oracle(oracle_mod, w, T=64):
    got, st, _ = gpu_decode(w, T)
    assert st == 0
    ref = oracle_mod.decode_format(oracle_mod.build_format(w, T))
    assert np.array_equal(ref, w)  # oracle round trip
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("n", [1, 2, 15, 16, 17, 63, 64, 65, 1000, 32 * 25 - 1, 32 * 25, 32 * 25 + 1,
                               256 * 25 + 1, 100_003, 1 << 20])
def test_sizes(oracle_mod, n):
    check_against_oracle(oracle_mod, inputs.gaussian(n, [21, n]))


@pytest.mark.parametrize("T", [32, 64])
@pytest.mark.parametrize("n", [1, 65, 32 * 64 + 1, 300_007])
def test_block_sizes(oracle_mod, T, n):
    # one warp decodes a block of T segments: T = 64 runs two chains per lane
    check_against_oracle(oracle_mod, inputs.gaussian(n, [31, T, n]), T)


@pytest.mark.parametrize("T", [96, 128, 256])
def test_other_block_sizes_are_rejected(T):
    # the decoder's thread block is one warp of one or two chains per lane:
    # other block sizes are refused on the host, nothing is launched
    torch = torch_cuda()
    fmt = df11.build_format(inputs.gaussian(10_000, [22, T]), T)
    dev = df11.DeviceFormat(fmt, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(df11.Df11Error) as e:
        df11.decompress(dev, None, status)
    assert e.value.status == 1


@pytest.mark.parametrize("T", [32, 64])
def test_many_blocks_per_warp(oracle_mod, T):
    # more blocks than resident warps: every warp walks several blocks
    check_against_oracle(oracle_mod, inputs.gaussian(6_000_011, [22, 1]), T)


def test_empty_stream():
    torch = torch_cuda()
    fmt = df11.build_format(np.zeros(0, np.uint16))
    dev = df11.DeviceFormat(fmt, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    df11.decompress(dev, out, status)
    assert df11.read_status(status) == 0


def test_every_bf16_pattern(oracle_mod):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ok = allbits[((allbits >> 7) & 0xFF) < 240]
    for seed in range(3):
        check_against_oracle(oracle_mod, np.random.default_rng(seed).permutation(ok))


def test_single_symbol(oracle_mod):
    w = np.full(100_000, 0x3F80, np.uint16)
    w[::3] |= 0x8000
    w[::5] |= 0x0055
    check_against_oracle(oracle_mod, w)


def test_length_limited_code(oracle_mod):
    f = [1, 1]
    while len(f) < 34:
        f.append(f[-1] + f[-2])
    exps = np.repeat(np.arange(34, dtype=np.uint16) + 60, f)
    exps = np.random.default_rng(5).permutation(exps)
    mant = np.random.default_rng(6).integers(0, 256, exps.size).astype(np.uint16)
    w = (exps << 7) | (mant & 0x7F) | ((mant & 0x80) << 8)
    got, st, fmt = gpu_decode(w)
    assert st == 0 and fmt.info()["max_code_len"] == 32
    assert np.array_equal(got, w)


@pytest.mark.parametrize("T", [32, 64])
def test_stress_small(oracle_mod, T):
    check_against_oracle(oracle_mod, inputs.stress(1 << 21, key=(3, 7, 7)), T)


def test_multi_matrix(oracle_mod):
    mats = [inputs.gaussian(n, [23, n]) for n in (4096 * 3 + 5, 17, 0, 70_000)]
    got, st, _ = gpu_decode(mats)
    assert st == 0
    ref = oracle_mod.decode_format(oracle_mod.build_format(np.concatenate(mats), 64))
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("offset", [8, 16])
def test_output_alignment_and_neighbours(offset):
    # decoding into the middle of a larger buffer writes exactly n elements;
    # offset 8 leaves the output 16-byte aligned only (16-byte stores),
    # offset 16 makes it 32-byte aligned (32-byte stores)
    torch = torch_cuda()
    w = inputs.gaussian(12_345, [24])
    fmt = df11.build_format(w)
    dev = df11.DeviceFormat(fmt, "cuda")
    buf = torch.full((12_345 + 64,), 7, dtype=torch.int16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress(dev, buf[offset:].view(torch.bfloat16), status)
    assert df11.read_status(status) == 0
    h = buf.cpu().numpy().view(np.uint16)
    assert np.all(h[:offset] == 7) and np.all(h[offset + 12_345:] == 7)
    assert np.array_equal(h[offset:offset + 12_345], w)


@pytest.mark.parametrize("max_sms", [1, 3, 17, 1000])
def test_sm_cap_gives_the_same_result(max_sms):
    # df11_decompress_sms: fewer persistent CTAs walk more blocks each
    torch = torch_cuda()
    w = inputs.gaussian(3_000_017, [26])
    dev = df11.DeviceFormat(df11.build_format(w), "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = df11.decompress(dev, None, status, max_sms=max_sms)
    assert df11.read_status(status) == 0
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), w)


@pytest.mark.parametrize("n,T,kind", [(1, 64, "g"), (100_003, 64, "g"), (20_000_011, 64, "g"),
                                      (20_000_011, 32, "g"), (9_000_001, 32, "stress")])
def test_host_buffers_round_trip(n, T, kind):
    # df11_decompress_host: pieces of whole blocks copied up, decoded and
    # copied down on separate streams (one piece below 8 Mi outputs, three
    # above 16 Mi); the device arrays start as garbage, so every byte the
    # decode reads must have been uploaded
    torch = torch_cuda()
    w = inputs.gaussian(n, [27, n, T]) if kind == "g" else inputs.stress(n, key=(27, n, T))
    dev = df11.DeviceFormat(df11.build_format(w, T), "cuda", pin_host=True)
    for t in dev.tensors.values():
        t.fill_(0xA5)
    out_dev = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    host_out = torch.empty(n, dtype=torch.int16).pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_host(dev, out_dev, host_out, status)
    assert df11.read_status(status) == 0
    assert np.array_equal(host_out.numpy().view(np.uint16), w)
    assert np.array_equal(out_dev.view(torch.int16).cpu().numpy().view(np.uint16), w)


def test_host_buffers_with_corrupt_offsets_stay_in_bounds():
    # a host BlockOffset entry past n: the kernel reports the block, and the
    # host-side copy ranges (taken from that array) stay inside the buffers
    torch = torch_cuda()
    n = 9_000_001
    w = inputs.gaussian(n, [28])
    dev = df11.DeviceFormat(df11.build_format(w), "cuda", pin_host=True)
    offs = dev.host_tensors["block_offset"].view(torch.int32)
    k = offs.numel() // 2
    offs[k] = n + 12_345
    guard = 64
    out_dev = torch.empty(n + guard, dtype=torch.bfloat16, device="cuda")
    host = torch.full((n + guard,), 0x5A5A, dtype=torch.int16).pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_host(dev, out_dev, host[:n], status)
    assert df11.read_status(status) != 0
    assert torch.all(host[n:] == 0x5A5A)  # nothing written past n


def test_repeated_launches_are_identical():
    torch = torch_cuda()
    w = inputs.gaussian(1 << 20, [25])
    fmt = df11.build_format(w)
    dev = df11.DeviceFormat(fmt, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = [df11.decompress(dev, None, status).view(torch.int16).clone() for _ in range(3)]
    assert df11.read_status(status) == 0
    for o in outs:
        assert torch.equal(o, outs[0])
    assert np.array_equal(outs[0].cpu().numpy().view(np.uint16), w)


# ----------------------------------------------------------------- corruption
def _corrupt_run(w, mutate):
    torch = torch_cuda()
    fmt = df11.build_format(w)
    dev = df11.DeviceFormat(fmt, "cuda")
    mutate(dev, torch)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(dev.n, dtype=torch.bfloat16, device="cuda")
    df11.decompress(dev, out, status)
    return df11.read_status(status)


def test_corrupt_block_offset_is_reported():
    def mutate(dev, torch):
        offs = dev.tensors["block_offset"].view(torch.int32)
        offs[3] += 5
    assert _corrupt_run(inputs.gaussian(200_000, [26]), mutate) == df11.DF11_ERR_CORRUPT


def test_corrupt_gaps_is_reported():
    def mutate(dev, torch):
        g = dev.tensors["gaps"]
        g[40:48] ^= 0x5A
    assert _corrupt_run(inputs.gaussian(200_000, [27]), mutate) == df11.DF11_ERR_CORRUPT


def test_corrupt_stream_is_reported():
    def mutate(dev, torch):
        s = dev.tensors["encoded_exponent"]
        s[1000:1400] = 0xFF
    assert _corrupt_run(inputs.gaussian(200_000, [28]), mutate) == df11.DF11_ERR_CORRUPT


def test_dangling_lut_pointer_is_reported():
    # long codes exist in the stress distribution: point one child entry past k
    w = inputs.stress(1 << 20, key=(3, 8, 8))
    fmt = df11.build_format(w)
    luts = fmt.arrays()["luts"]
    ptr_idx = int(np.nonzero(luts[0] >= 240)[0][0])

    def mutate(dev, torch):
        dev.tensors["luts"][ptr_idx] = 240  # child 16, beyond num_luts
        # without the stored table every code is looked up through the LUTs
        # (a stored table answers codes of up to 12 bits without them)
        dev.c_arrays.symbol_table = None
    assert _corrupt_run(w, mutate) == df11.DF11_ERR_CORRUPT


def test_impossible_symbol_table_entry_is_reported():
    # a stored table entry no code can produce (one code of 0 bits; 13 bits;
    # 4 codes) is refused before any block is decoded: the decode loop relies
    # on every code taking at least one bit
    for entry in (1 << 29, (1 << 29) | (13 << 24), (4 << 29) | (12 << 24)):
        def mutate(dev, torch, entry=entry):
            dev.tensors["symbol_table"].view(torch.int32)[77] = entry - (1 << 32 if entry >= 1 << 31 else 0)
        assert _corrupt_run(inputs.gaussian(200_000, [32]), mutate) == df11.DF11_ERR_CORRUPT


def _entry_i32(v):
    return v - (1 << 32) if v >= 1 << 31 else v


def test_symbol_table_entry_of_codes_shorter_than_the_slots_allow_is_reported():
    # a stream whose shortest code has 2 bits decodes through short staging
    # slots; a stored entry of two 1-bit codes would overrun them, so the
    # table is refused before any block is decoded
    w = inputs.gaussian(200_000, [32])
    assert df11.build_format(w).scalars()["min_code_len"] >= 2

    def mutate(dev, torch):
        dev.tensors["symbol_table"].view(torch.int32)[77] = _entry_i32((2 << 29) | (2 << 24) | 0x0101)
    assert _corrupt_run(w, mutate) == df11.DF11_ERR_CORRUPT


def test_symbol_table_bytes_past_the_count_are_ignored():
    # an entry's exponent bytes past its count carry no meaning: filled with
    # ones, the stream still decodes exactly
    torch = torch_cuda()
    w = inputs.gaussian(300_000, [30])
    fmt = df11.build_format(w)
    dev = df11.DeviceFormat(fmt, "cuda")
    t = dev.tensors["symbol_table"].view(torch.int32).cpu().numpy().view(np.uint32).copy()
    n = t >> 29
    keep = np.where(n >= 3, 0xFFFFFF, (np.uint32(1) << (8 * n).astype(np.uint32)) - 1).astype(np.uint32)
    filled = t | (np.uint32(0xFFFFFF) & ~keep)
    assert (filled != t).any()
    dev.tensors["symbol_table"].view(torch.int32).copy_(torch.from_numpy(filled.view(np.int32)))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(dev.n, dtype=torch.bfloat16, device="cuda")
    df11.decompress(dev, out, status)
    assert df11.read_status(status) == 0
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), w)


def test_symbol_table_that_leaves_short_codes_to_the_luts_is_reported():
    # an entry of 0 sends its window to the page's LUTs as a code longer than
    # 12 bits; the LUTs finding a shorter one there marks the table wrong
    def mutate(dev, torch):
        dev.tensors["symbol_table"].zero_()
    assert _corrupt_run(inputs.gaussian(200_000, [31]), mutate) == df11.DF11_ERR_CORRUPT


def test_understated_capacity_is_reported():
    def mutate(dev, torch):
        dev.c_arrays.max_block_elems = 100
    assert _corrupt_run(inputs.gaussian(200_000, [29]), mutate) == df11.DF11_ERR_CORRUPT


def test_bad_arguments_launch_nothing():
    torch = torch_cuda()
    fmt = df11.build_format(inputs.gaussian(1000, [30]))
    dev = df11.DeviceFormat(fmt, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(1000 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(df11.Df11Error) as e:
        df11.decompress(dev, out[1:], status)  # 2-byte aligned only
    assert e.value.status == 1
    dev.c_arrays.num_blocks += 1
    with pytest.raises(df11.Df11Error):
        df11.decompress(dev, out, status)


# ----------------------------------------------------------- full workloads
def _full_check(oracle_mod, workload, block_id=0, sample_blocks=200):
    torch = torch_cuda()
    mats = [m for _, _, m in inputs.workload_arrays(workload, block_id)]
    w = np.concatenate(mats) if len(mats) > 1 else mats[0]
    got, st, fmt = gpu_decode(mats, 64)
    assert st == 0
    assert np.array_equal(got, w)
    # oracle: its own format from the same input, then its tree walk over a
    # sample of blocks' bit ranges
    ref = oracle_mod.build_format(w, 64)
    offs = ref["block_offset"].astype(np.int64)
    nb = offs.size - 1
    rng = np.random.default_rng(workload)
    blocks = sorted(set([0, nb - 1] + rng.integers(0, nb, sample_blocks).tolist()))
    gaps = ref["gaps"]
    nseg = gaps.size
    for b in blocks:
        s0 = b * 64
        s1 = min((b + 1) * 64, nseg)
        a = 64 * s0 + int(gaps[s0])
        e = 64 * s1 + int(gaps[s1]) if s1 < nseg else ref["total_bits"]
        exps = oracle_mod.decode_range(ref["encoded_exponent"], ref["total_bits"], a, e,
                                       ref["code_lengths"], ref["codes"])
        sl = slice(int(offs[b]), int(offs[b + 1]))
        assert exps.size == sl.stop - sl.start
        assert np.array_equal((got[sl] >> 7) & 0xFF, exps)
    return fmt


def test_workload_single_matrix(oracle_mod):
    w = inputs.single_matrix()
    check_against_oracle(oracle_mod, w)


def test_workload_llama3_8b_block(oracle_mod):
    _full_check(oracle_mod, 2)


def test_workload_stress(oracle_mod):
    fmt = _full_check(oracle_mod, 3)
    info = fmt.info()
    assert info["max_code_len"] >= 24 and 4 <= info["num_luts"] <= 8


@pytest.mark.slow
def test_workload_llama3_70b_block(oracle_mod):
    _full_check(oracle_mod, 4, sample_blocks=100)


@pytest.mark.slow
def test_workload_stream_of_32_blocks():
    # 32 independent Llama-3-8B blocks, each with its own code, decoded back to
    # back into ONE reused BF16 buffer (the streaming launch configuration);
    # every block is checked against its original bits before the next
    # overwrites the buffer ("Dekompresi per transformer block").
    torch = torch_cuda()
    from concurrent.futures import ThreadPoolExecutor

    n = inputs.block_elements(5)
    out = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def prepare(b):
        mats = [m for _, _, m in inputs.workload_arrays(5, b)]
        return np.concatenate(mats), df11.build_format(mats)

    with ThreadPoolExecutor(1) as ex:
        nxt = ex.submit(prepare, 0)
        for b in range(32):
            w, fmt = nxt.result()
            if b + 1 < 32:
                nxt = ex.submit(prepare, b + 1)
            dev = df11.DeviceFormat(fmt, "cuda")
            fmt.free()
            df11.decompress(dev, out, status)
            ref = torch.from_numpy(w.view(np.int16)).to("cuda")
            assert torch.equal(out.view(torch.int16), ref), f"block {b}"
            del dev, ref
    assert df11.read_status(status) == 0


@pytest.mark.gpu
def test_stream_without_symbol_table_derives_it():
    # a stream whose arrays carry no derived table (symbol_table NULL): each
    # CTA derives it from the LUTs and CodeLengths, with the same result
    torch = torch_cuda()
    for w in (inputs.gaussian(3_000_017, [130]), inputs.stress(1_000_003, key=(131, 0))):
        dev = df11.DeviceFormat(df11.build_format(w), "cuda")
        assert dev.c_arrays.symbol_table
        dev.c_arrays.symbol_table = None
        out = torch.empty(w.size, dtype=torch.int16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        df11.decompress(dev, out, status)
        assert df11.read_status(status) == 0
        assert np.array_equal(out.cpu().numpy().view(np.uint16), w)
