"""Seeded synthetic BF16 weights: the one module the tests, the oracle checks
and the benchmark all read their inputs from.

It holds no DF11 arithmetic (no field split, no code, no format): it only draws
numbers and rounds them to BF16 bits.  The DFloat11 page measures on trained
LLM and diffusion weights, which are not available here; these generators
stand in for them with the shapes of Llama-3-8B and Llama-3-70B transformer
blocks and LLM-like value distributions.

Recipe (numpy PCG64):
  * float32 samples -> BF16 by round-to-nearest-even on the top 16 bits;
  * a matrix is drawn in chunks of ``CHUNK`` elements, chunk j of matrix m of
    block b of workload c from ``SeedSequence([c, b, m, j])`` (so chunks can
    be drawn in parallel without changing a value);
  * ``single``   : 1024 x 1024, N(0, 0.02), ``default_rng(0)``;
  * ``llama3_8b``: q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096,
                   down 4096x14336, N(0, 0.02) per matrix;
  * ``stress``   : 64 Mi elements, Student-t (nu = 3) x 0.02, then 0.1% exact
                   zeros (half +0, half -0) and 0.05% subnormals (random sign,
                   exponent 0, mantissa 1..127) at random positions;
  * ``llama3_70b``: q/o 8192x8192, k/v 1024x8192, gate/up 28672x8192,
                   down 8192x28672, N(0, sigma_row) with sigma_row drawn
                   log-normal(ln 0.02, 0.5) once per row;
  * ``stream32`` : 32 independent ``llama3_8b`` blocks (workload id 5).
Matrices are row-major and a block concatenates q, k, v, o, gate, up, down.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

CHUNK = 1 << 24

LLAMA3_8B = [
    ("q", (4096, 4096)), ("k", (1024, 4096)), ("v", (1024, 4096)), ("o", (4096, 4096)),
    ("gate", (14336, 4096)), ("up", (14336, 4096)), ("down", (4096, 14336)),
]
LLAMA3_70B = [
    ("q", (8192, 8192)), ("k", (1024, 8192)), ("v", (1024, 8192)), ("o", (8192, 8192)),
    ("gate", (28672, 8192)), ("up", (28672, 8192)), ("down", (8192, 28672)),
]

WORKLOADS = {
    1: "single_1024x1024_gauss",
    2: "llama3_8b_block",
    3: "stress_t3_64Mi",
    4: "llama3_70b_block",
    5: "llama3_8b_x32_stream",
}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _chunked(n: int, fill, key) -> np.ndarray:
    """Draws n BF16 values chunk by chunk; fill(rng, lo, hi) -> float32."""
    out = np.empty(n, np.uint16)

    def work(j):
        lo = j * CHUNK
        hi = min(n, lo + CHUNK)
        rng = np.random.default_rng(np.random.SeedSequence(list(key) + [j]))
        out[lo:hi] = to_bf16_bits(fill(rng, lo, hi))

    nchunks = (n + CHUNK - 1) // CHUNK
    if nchunks <= 1:
        for j in range(nchunks):
            work(j)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(work, range(nchunks)))
    return out


def gaussian(n: int, key, sigma: float = 0.02) -> np.ndarray:
    """n BF16 values ~ N(0, sigma), drawn under the seed key (a list of ints)."""
    return _chunked(n, lambda rng, lo, hi: rng.standard_normal(hi - lo, dtype=np.float32) * np.float32(sigma), key)


def single_matrix() -> np.ndarray:
    """Workload 1: 1024 x 1024 N(0, 0.02), default_rng(0)."""
    rng = np.random.default_rng(0)
    return to_bf16_bits(rng.standard_normal(1 << 20, dtype=np.float32) * np.float32(0.02))


def stress(n: int = 64 << 20, key=(3, 0, 0)) -> np.ndarray:
    """Workload 3: heavy-tailed values plus exact zeros and subnormals."""
    key = list(key)

    def fill(rng, lo, hi):
        return (rng.standard_t(3, hi - lo) * 0.02).astype(np.float32)

    w = _chunked(n, fill, key)
    rng = np.random.default_rng(np.random.SeedSequence(key + [1 << 30]))
    u = rng.random(n, dtype=np.float32)
    zero = u < np.float32(0.001)
    sub = (u >= np.float32(0.001)) & (u < np.float32(0.0015))
    sign = (rng.integers(0, 2, n, dtype=np.uint16) << np.uint16(15)).astype(np.uint16)
    mant = rng.integers(1, 128, n, dtype=np.uint16)
    w[zero] = sign[zero]
    w[sub] = sign[sub] | mant[sub]
    # no exponent in 240..255 (t3 * 0.02 never gets near 2^113; kept as a guard)
    bad = ((w >> np.uint16(7)) & np.uint16(0xFF)) >= 240
    while bad.any():
        w[bad] = to_bf16_bits(rng.standard_normal(int(bad.sum()), dtype=np.float32) * np.float32(0.02))
        bad = ((w >> np.uint16(7)) & np.uint16(0xFF)) >= 240
    return w


def _row_lognormal(rows: int, cols: int, key) -> np.ndarray:
    key = list(key)
    srng = np.random.default_rng(np.random.SeedSequence(key + [1 << 30]))
    sigma = srng.lognormal(np.log(0.02), 0.5, rows).astype(np.float32)

    def fill(rng, lo, hi):
        z = rng.standard_normal(hi - lo, dtype=np.float32)
        row = np.arange(lo, hi, dtype=np.int64) // cols
        return z * sigma[row]

    return _chunked(rows * cols, fill, key)


def block(workload: int, block_id: int = 0):
    """One transformer block: list of (name, shape, uint16 bits)."""
    if workload in (2, 5):
        return [(name, shape, gaussian(shape[0] * shape[1], [workload, block_id, m]))
                for m, (name, shape) in enumerate(LLAMA3_8B)]
    if workload == 4:
        return [(name, shape, _row_lognormal(shape[0], shape[1], [workload, block_id, m]))
                for m, (name, shape) in enumerate(LLAMA3_70B)]
    raise ValueError(f"workload {workload} is not a transformer block")


def block_elements(workload: int) -> int:
    shapes = LLAMA3_70B if workload == 4 else LLAMA3_8B
    return sum(r * c for _, (r, c) in shapes)


def workload_arrays(workload: int, block_id: int = 0):
    """Matrices of one stream of a workload (one Huffman code per stream)."""
    if workload == 1:
        return [("w", (1024, 1024), single_matrix())]
    if workload == 3:
        return [("w", (64, 1 << 20), stress())]
    return block(workload, block_id)
