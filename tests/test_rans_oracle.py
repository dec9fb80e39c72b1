"""Pins of the oracle's rANS variant of the exponent coder (no GPU).

The page's discussion proposes rANS (range asymmetric numeral systems) as an
entropy coder that suits SIMD hardware; the oracle restates its published
definition (one 32-bit state, L = 2^16, 16-bit renormalisation words,
probabilities quantised to M = 2^12).  Each test pins the oracle against
something other than itself: the decoding rule (an encode step must be
inverted by it, exhaustively on small models), information theory (the coded
size equals the information content of the quantised model up to rounding,
and is never below the entropy), and closed forms of special models (one
symbol costs nothing, two equally likely symbols cost one bit each).
"""
import numpy as np
import pytest

from huffman_decode_03_b200 import inputs

L = 1 << 16


def test_frequencies_sum_and_support(oracle_mod):
    rng = np.random.default_rng(0)
    for trial in range(200):
        k = int(rng.integers(1, 257))
        hist = np.zeros(256, np.uint64)
        syms = rng.choice(256, k, replace=False)
        hist[syms] = rng.integers(1, 1 << int(rng.integers(1, 40)), k).astype(np.uint64)
        for pb in (8, 12):
            if k > (1 << pb):
                continue
            f = oracle_mod.rans_freqs(hist, pb)
            assert int(f.sum()) == 1 << pb
            assert np.all((f > 0) == (hist > 0))
    with pytest.raises(ValueError):
        oracle_mod.rans_freqs(np.zeros(256, np.uint64), 12)
    with pytest.raises(ValueError):  # 256 symbols do not fit a 128-slot model
        oracle_mod.rans_freqs(np.ones(256, np.uint64), 7)


def test_frequencies_follow_the_counts(oracle_mod):
    # a frequency differs from the exact share h M / n by less than one slot,
    # except where the quantisation adds or removes the rounding remainder
    # (the largest counts); the adjusted total is exact
    hist = np.zeros(256, np.uint64)
    hist[[119, 120, 121, 122, 123, 124, 125, 126]] = [5, 400, 3000, 9000, 9000, 3000, 400, 5]
    f = oracle_mod.rans_freqs(hist, 12).astype(np.float64)
    share = hist.astype(np.float64) * 4096 / hist.sum()
    small = hist < 9000
    assert np.all(np.abs(f[small] - share[small]) < 1.0 + 1e-9)
    assert abs(f.sum() - 4096) < 1e-9


def _decode_step(y, freq, prob_bits, word):
    # the decoding rule, stated independently of the oracle's encoder
    M = 1 << prob_bits
    cum = np.concatenate([[0], np.cumsum(freq.astype(np.int64))])
    slot = y % M
    s = int(np.searchsorted(cum, slot, side="right") - 1)
    x = int(freq[s]) * (y // M) + slot - int(cum[s])
    if x < L:
        assert word is not None, "decoder needs a word the encoder did not emit"
        x = (x << 16) | word
    else:
        assert word is None, "encoder emitted a word the decoder does not read"
    return s, x


@pytest.mark.parametrize("freq", [
    [1, 15], [8, 8], [15, 1], [1, 1, 14], [3, 5, 7, 1], [2] * 8, [1] * 16,
])
def test_one_step_is_inverted_by_the_decoding_rule(oracle_mod, freq):
    # exhaustive over x in [L, L + 8192) and a band below 2^32, every symbol,
    # for a 4-bit model: the encoder keeps the state in [L, 2^32), emits a word
    # exactly when the decoder reads one, and decoding restores (s, x)
    pb = 4
    f = np.zeros(256, np.uint32)
    f[: len(freq)] = freq
    assert f.sum() == 1 << pb
    xs = list(range(L, L + 8192)) + list(range((1 << 32) - 4096, 1 << 32)) + list(range(1 << 31, (1 << 31) + 512))
    for s in range(len(freq)):
        for x in xs:
            y, word = oracle_mod.rans_step_encode(x, s, f, pb)
            assert L <= y < (1 << 32)
            assert _decode_step(y, f, pb, word) == (s, x)


def test_round_trips(oracle_mod):
    rng = np.random.default_rng(1)
    cases = [np.zeros(0, np.uint16), inputs.gaussian(1, [70]), inputs.gaussian(511, [71]),
             inputs.gaussian(4095, [72]), inputs.gaussian(4096, [73]), inputs.gaussian(4097, [74]),
             inputs.gaussian(3 * 4096 + 17, [75]), inputs.stress(50_000, key=(76, 0))]
    # every BF16 pattern, exponents 240..255 included (rANS needs no pointer values)
    allp = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    rng.shuffle(allp)
    cases.append(allp)
    cases.append(np.full(10_000, 0x3C00, np.uint16))  # one exponent only
    for w in cases:
        for chunks in (1, 8, 15):
            fmt = oracle_mod.rans_build_format(w, 12, chunks)
            assert np.array_equal(oracle_mod.rans_decode_format(fmt), w)
    # a lane reads at most one word per step and counts them in a byte: 16 J <= 240
    with pytest.raises(ValueError):
        oracle_mod.rans_build_format(inputs.gaussian(100, [77]), 12, 16)


def test_single_symbol_costs_nothing(oracle_mod):
    w = np.full(3 * 4096 + 5, 0x3C12, np.uint16)
    fmt = oracle_mod.rans_build_format(w)
    assert fmt["words"].size == 0 and np.all(fmt["states"] == L)


def test_two_equal_symbols_cost_one_bit_each(oracle_mod):
    # f = M/2 for both: every encode step adds exactly one bit to the state,
    # so a lane that codes k symbols from x = 2^16 emits floor(k / 16) words
    # (its stream's length) and ends with a state of 17 + k mod 16 bits
    rng = np.random.default_rng(2)
    for n in (4096, 4096 * 2 + 700, 123):
        exps = rng.integers(0, 2, n).astype(np.uint8)
        freq = np.zeros(256, np.uint32)
        freq[:2] = 2048
        words, states, offsets, lane_words = oracle_mod.rans_encode(exps, freq, 12, 8)
        for b in range(states.shape[0]):
            for lane in range(32):
                pos = b * 4096 + np.arange(8)[:, None] * 512 + 16 * lane + np.arange(16)[None, :]
                k = int((pos < n).sum())
                assert states[b, lane].item().bit_length() == 17 + k % 16
                assert int(lane_words[b, lane]) == k // 16
        per_lane = [int(((b * 4096 + np.arange(8)[:, None] * 512 + 16 * l + np.arange(16)[None, :]) < n).sum())
                    for b in range(states.shape[0]) for l in range(32)]
        assert words.size == sum(k // 16 for k in per_lane)


def test_size_is_the_information_content_of_the_model(oracle_mod):
    # 16 bits per word plus the bits the final states hold above their start
    # value L equal the model's information content sum_s h_s log2(M / f_s),
    # up to rANS rounding (well under a bit per lane); that content is at
    # least the entropy (Gibbs) and, for these counts, within 0.02 bit of it
    for w in (inputs.gaussian(1 << 20, [80]), inputs.stress(1 << 20, key=(81, 0))):
        fmt = oracle_mod.rans_build_format(w)
        hist = fmt["hist"].astype(np.float64)
        f = fmt["freq"].astype(np.float64)
        m = hist > 0
        content = float((hist[m] * np.log2(4096.0 / f[m])).sum())
        got = 16.0 * fmt["words"].size + float(np.log2(fmt["states"].astype(np.float64) / L).sum())
        lanes = fmt["states"].size
        assert abs(got - content) < lanes * 1.0
        n = hist.sum()
        p = hist[m] / n
        entropy = float(-(p * np.log2(p)).sum()) * n
        assert content >= entropy - 1e-6
        assert content <= entropy + 0.02 * n


def test_each_lane_stream_decodes_alone(oracle_mod):
    # every lane's stream, decoded on its own by the decoding rule (written
    # here independently of the oracle), gives back that lane's exponents in
    # the layout's order and ends at x = L with the stream used up
    w = inputs.stress(3 * 4096 + 1000, key=(78, 0))
    fmt = oracle_mod.rans_build_format(w, 12, 8)
    exps = ((w >> 7) & 0xFF).astype(np.int64)
    freq = fmt["freq"].astype(np.int64)
    cum = np.concatenate([[0], np.cumsum(freq)])
    n = w.size
    for b in range(fmt["states"].shape[0]):
        start = int(fmt["offsets"][b])
        for lane in range(32):
            cnt = int(fmt["lane_words"][b, lane])
            stream = fmt["words"][start: start + cnt]
            start += cnt
            x, k = int(fmt["states"][b, lane]), 0
            for t in range(16 * 8):
                pos = b * 4096 + 512 * (t // 16) + 16 * lane + t % 16
                if pos >= n:
                    continue
                slot = x % 4096
                s = int(np.searchsorted(cum, slot, side="right") - 1)
                assert s == exps[pos]
                x = int(freq[s]) * (x // 4096) + slot - int(cum[s])
                if x < L:
                    x = (x << 16) | int(stream[k])
                    k += 1
            assert x == L and k == cnt
        assert start == int(fmt["offsets"][b + 1])


def test_inconsistent_data_is_rejected(oracle_mod):
    w = inputs.gaussian(10_000, [90])
    fmt = oracle_mod.rans_build_format(w)
    moved = dict(fmt)  # one word moved from lane 3's stream to lane 4's
    moved["lane_words"] = fmt["lane_words"].copy()
    moved["lane_words"][0, 3] -= 1
    moved["lane_words"][0, 4] += 1
    with pytest.raises(ValueError):
        oracle_mod.rans_decode_format(moved)
    uncounted = dict(fmt)  # lane counts that do not add up to the block's words
    uncounted["lane_words"] = fmt["lane_words"].copy()
    uncounted["lane_words"][1, 0] += 1
    with pytest.raises(ValueError):
        oracle_mod.rans_decode_format(uncounted)
    short = dict(fmt)
    short["words"] = fmt["words"][:-1]
    short["offsets"] = fmt["offsets"].copy()
    short["offsets"][-1] -= 1
    with pytest.raises(ValueError):
        oracle_mod.rans_decode_format(short)
    bad_state = dict(fmt)
    bad_state["states"] = fmt["states"].copy()
    bad_state["states"][0, 0] ^= 1
    with pytest.raises(ValueError):
        oracle_mod.rans_decode_format(bad_state)


def test_split_all_is_the_ieee_field_split(oracle_mod):
    # every BF16 pattern against numpy's IEEE view of float32 (BF16 = top 16 bits)
    w = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exps, sm = oracle_mod.split_all(w)
    f = (w.astype(np.uint32) << 16).view(np.float32)
    bits = f.view(np.uint32)
    assert np.array_equal(exps, ((bits >> 23) & 0xFF).astype(np.uint8))
    assert np.array_equal(sm, (((bits >> 24) & 0x80) | ((bits >> 16) & 0x7F)).astype(np.uint8))
