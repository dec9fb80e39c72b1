"""Property test of the library's host format builder against the oracle on
random streams (no GPU): random sizes, block sizes T and exponent
distributions — from one dominant exponent (1-bit codes) through geometric
(a deep, skewed tree) to nearly uniform over up to 40 values — with random
sign and mantissa bits.  Every array must agree byte for byte with the
oracle's ("Format DFloat11", "Decoding berbasis LUT hierarkis", "Kernel GPU 2
tahap dan metadata bantu"), and the oracle's tree-walk decode of its own
format must return the input."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import huffman_decode_03_b200 as df11
from test_host_format import compare


@st.composite
def streams(draw):
    n = draw(st.integers(1, 4000))
    k = draw(st.integers(1, 40))
    values = draw(st.lists(st.integers(0, 239), min_size=k, max_size=k, unique=True))
    shape = draw(st.sampled_from(["geometric", "uniform", "one_heavy", "two_level"]))
    T = draw(st.sampled_from([32, 64, 96, 128, 1024]))
    seed = draw(st.integers(0, 2**32 - 1))
    rng = np.random.default_rng(seed)
    if shape == "geometric":
        p = 0.5 ** np.arange(k, dtype=np.float64)
    elif shape == "uniform":
        p = np.ones(k)
    elif shape == "one_heavy":
        p = np.full(k, 0.03 / max(k - 1, 1))
        p[0] = 0.97
    else:
        p = np.where(np.arange(k) < (k + 1) // 2, 1.0, 0.01)
    p = p / p.sum()
    e = rng.choice(np.array(values, np.uint16), size=n, p=p)
    sm = rng.integers(0, 256, n, dtype=np.uint16)
    w = ((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)
    return w.astype(np.uint16), T


@settings(max_examples=120, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(streams())
def test_library_format_equals_oracle_on_random_streams(oracle_mod, case):
    w, T = case
    ref = oracle_mod.build_format(w, T)
    compare(df11.build_format(w, T), ref)
    assert np.array_equal(oracle_mod.decode_format(ref), w)
