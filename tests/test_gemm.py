"""Fused decode + tensor-core GEMM (df11_decompress_gemm): Y_m += X_m W_m^T
with the BF16 weights decoded tile by tile into shared memory and never
stored ("Dekompresi yang disesuaikan untuk inferensi GPU": decompress right
before the matrix multiplication).  The stream holds each matrix in
tile-major order (df11_tile_major).

Reference: the product of the ORIGINAL row-major BF16 weights with the same
BF16 activations, in float64, so a wrong tile order, swizzle or operand
layout fails.  Tolerance: a BF16 x BF16 product is exact in float32 and each
output is a float32 sum of `cols` of them (tensor-core accumulation over K
chunks of 64, atomic adds over groups of 16 chunks) in some order and
rounding; with at most 2^-23 relative error per addition,
|y - y_ref| <= cols * 2^-23 * sum_k |w_k x_k|; the tests allow twice that.

Identity activations (x_n = e_{c0 + n}) turn the product into a copy of
columns c0 .. c0 + batch - 1 of W, which must come back exactly; on a
mismatch the message names where the wrong values came from."""
import ctypes

import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _ref_tile_major(w, rows, cols):
    # the order written out: row tiles, column tiles, rows of a tile
    return np.asarray(w, np.uint16).reshape(rows // 128, 128, cols // 64, 64).transpose(0, 2, 1, 3).reshape(-1)


# ------------------------------------------------------------------- host
@pytest.mark.parametrize("rows,cols", [(128, 64), (256, 128), (384, 1088)])
def test_tile_major_order(rows, cols):
    w = np.arange(rows * cols, dtype=np.uint32).astype(np.uint16)
    t = df11.tile_major(w, rows, cols)
    assert np.array_equal(t, _ref_tile_major(w, rows, cols))
    # element (r, c) sits at ((r // 128 * (cols // 64) + c // 64) * 128 + r % 128) * 64 + c % 64
    r, c = rows - 1, cols - 3
    i = ((r // 128 * (cols // 64) + c // 64) * 128 + r % 128) * 64 + c % 64
    assert t[i] == w[r * cols + c]


def test_tile_major_stream_has_the_same_code_and_size():
    # the element order is the compressor's choice: the histogram, and so the
    # code, the LUTs and the compressed size, do not depend on it
    shapes = [(256, 128), (128, 1088)]
    mats = [inputs.gaussian(r * c, [79, m]) for m, (r, c) in enumerate(shapes)]
    row = df11.build_format(mats)
    tiled = df11.build_format([df11.tile_major(w, r, c) for (r, c), w in zip(shapes, mats)])
    a, b = row.arrays(), tiled.arrays()
    assert np.array_equal(a["code_lengths"], b["code_lengths"])
    assert np.array_equal(a["luts"], b["luts"])
    assert row.scalars()["total_bits"] == tiled.scalars()["total_bits"]
    assert row.info()["compressed_bytes"] == tiled.info()["compressed_bytes"]
    assert not np.array_equal(a["encoded_exponent"], b["encoded_exponent"])


def test_tile_major_rejects_ragged_shapes():
    with pytest.raises(df11.Df11Error):
        df11.tile_major(np.zeros(100 * 64, np.uint16), 100, 64)
    with pytest.raises(df11.Df11Error):
        df11.tile_major(np.zeros(128 * 48, np.uint16), 128, 48)


def test_scratch_bytes():
    # packed X (batch * cols * 2 bytes per matrix) + 8 bytes per work unit
    # (one per 128 rows and 16 chunks of 64 columns)
    shapes = [(4096, 4096), (1024, 4096), (4096, 14336)]
    units = 32 * 4 + 8 * 4 + 32 * 14
    assert df11.gemm_scratch_bytes(shapes, 64) == 64 * 2 * (4096 + 4096 + 14336) + 8 * units
    assert df11.gemm_scratch_bytes([(128, 1088)], 16) == 16 * 2 * 1088 + 8 * 2
    assert df11.gemm_scratch_bytes([(100, 64)], 64) == 0
    assert df11.gemm_scratch_bytes([(128, 64)], 8) == 0
    assert df11.gemm_scratch_bytes([(128, 64)], 24) == 0
    assert df11.gemm_scratch_bytes([(128, 64)], 272) == 0


def test_gemm_argument_checks_run_before_any_launch():
    # refused on the host before any CUDA call (no GPU needed); the arrays
    # are the host copies, only checked
    lib = df11.load_library()
    shapes = [(128, 64), (256, 128)]
    w = np.concatenate([df11.tile_major(inputs.gaussian(r * c, [70, m]), r, c) for m, (r, c) in enumerate(shapes)])
    fmt = df11.build_format(w)
    a = fmt.c_arrays
    status = (ctypes.c_uint32 * 4)()
    buf = (ctypes.c_uint8 * (1 << 16))()
    base = (ctypes.addressof(buf) + 15) & ~15

    def call(shapes, batch=16, x=base, y=base, scratch=base, scratch_bytes=1 << 15):
        mats = (df11.df11_gemm_matrix * max(len(shapes), 1))()
        for m, (r, c) in enumerate(shapes):
            mats[m].rows, mats[m].cols, mats[m].x, mats[m].y = r, c, x, y
        return lib.df11_decompress_gemm(ctypes.byref(a), mats, len(shapes), batch, scratch, scratch_bytes,
                                        ctypes.addressof(status), None)

    assert call(shapes[:1]) == 1                         # rows*cols do not cover the stream
    assert call(shapes + [(128, 64)]) == 1               # more elements than the stream
    assert call([(64, 128), (256, 128)]) == 1            # rows not a multiple of 128
    assert call(shapes, batch=8) == 1                    # batch below 16
    assert call(shapes, batch=40) == 1                   # batch not a multiple of 16
    assert call(shapes, x=base + 2) == 1                 # x not 16-byte aligned
    assert call(shapes, scratch_bytes=100) == 1          # scratch too small
    assert call(shapes, scratch=base + 4) == 1           # scratch not 16-byte aligned
    assert call([]) == 1
    assert call([(128, 64)] * 17) == 1                   # more than 16 matrices


# ------------------------------------------------------------------- device
def _torch():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _run(shapes, mats, batch, T=64, xbits=None, seed=0, y0=None):
    """Runs the fused GEMM on tile-major streams of `mats` (row-major bits);
    returns (ys as float64 arrays, xs bits, status word)."""
    torch = _torch()
    stream = [df11.tile_major(W, r, c) for (r, c), W in zip(shapes, mats)]
    dev = df11.DeviceFormat(df11.build_format(stream, T), "cuda")
    if xbits is None:
        xbits = [inputs.gaussian(batch * c, [71, seed, m], sigma=1.0) for m, (r, c) in enumerate(shapes)]
    xs = [torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16).reshape(batch, c)
          for b, (r, c) in zip(xbits, shapes)]
    ys = [torch.zeros(batch, r, dtype=torch.float32, device="cuda") if y0 is None
          else torch.from_numpy(y0[m].astype(np.float32)).cuda() for m, (r, c) in enumerate(shapes)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_gemm(dev, shapes, xs, ys, status)
    torch.cuda.synchronize()
    word = int(status.item()) & 0xFFFFFFFF
    return [y.cpu().numpy().astype(np.float64) for y in ys], xbits, word


def _check(y, W_bits, x_bits, rows, cols, batch, y0=None, row_sample=None):
    W = _bf16_to_f64(W_bits).reshape(rows, cols)
    X = _bf16_to_f64(x_bits).reshape(batch, cols)
    rs = np.arange(rows) if row_sample is None else row_sample
    ref = X @ W[rs].T + (0 if y0 is None else y0[:, rs])
    bound = 2 * cols * 2.0 ** -23 * (np.abs(X) @ np.abs(W[rs]).T) + 1e-30
    err = np.abs(y[:, rs] - ref)
    assert np.all(err <= bound), f"worst error / bound {float((err / bound).max()):.3g}"


def _identity_bits(batch, cols, c0):
    x = np.zeros((batch, cols), np.uint16)
    x[np.arange(batch), c0 + np.arange(batch)] = 0x3F80  # 1.0
    return x.reshape(-1)


def _explain(got, W, c0):
    """Where the wrong values of a copied W block came from (first few)."""
    rows, cols = W.shape
    where = {}
    for r in range(rows):
        for c in range(cols):
            where.setdefault(float(W[r, c]), (r, c))
    lines = []
    batch = got.shape[0]
    for n in range(batch):
        for r in range(rows):
            want = W[r, c0 + n]
            if got[n, r] != want:
                lines.append(f"y[{n}][{r}] = W{where.get(float(got[n, r]), '(none)')} instead of W({r}, {c0 + n})")
                if len(lines) >= 12:
                    return "\n".join(lines)
    return "\n".join(lines)


@pytest.mark.gpu
@pytest.mark.parametrize("rows,cols,batch,c0", [(128, 64, 64, 0), (256, 192, 64, 64), (128, 1088, 128, 960)])
def test_gemm_identity_activations_copy_w(rows, cols, batch, c0):
    W_bits = inputs.gaussian(rows * cols, [72, rows, cols])
    ys, _, word = _run([(rows, cols)], [W_bits], batch, xbits=[_identity_bits(batch, cols, c0)])
    assert word == 0
    W = _bf16_to_f64(W_bits).reshape(rows, cols)
    got = ys[0]
    want = W[:, c0:c0 + batch].T
    assert np.array_equal(got, want), f"{int((got != want).sum())} of {got.size} differ:\n" + _explain(got, W, c0)


@pytest.mark.gpu
@pytest.mark.parametrize("T", [32, 64])
@pytest.mark.parametrize("batch", [16, 64, 128, 256])
def test_gemm_small_matrices(T, batch):
    shapes = [(128, 64), (256, 128), (384, 1088), (128, 2048)]
    mats = [inputs.gaussian(r * c, [73, m]) for m, (r, c) in enumerate(shapes)]
    ys, xb, word = _run(shapes, mats, batch, T)
    assert word == 0
    for m, (r, c) in enumerate(shapes):
        _check(ys[m], mats[m], xb[m], r, c, batch)


@pytest.mark.gpu
def test_gemm_accumulates_into_y():
    shapes = [(256, 1024), (128, 64)]
    batch = 32
    mats = [inputs.gaussian(r * c, [74, m]) for m, (r, c) in enumerate(shapes)]
    y0 = [np.random.default_rng(m).normal(size=(batch, r)) for m, (r, c) in enumerate(shapes)]
    ys, xb, word = _run(shapes, mats, batch, y0=y0)
    assert word == 0
    for m, (r, c) in enumerate(shapes):
        _check(ys[m], mats[m], xb[m], r, c, batch, y0=y0[m].astype(np.float32).astype(np.float64))


@pytest.mark.gpu
def test_gemm_stress_values():
    # exact zeros of both signs, subnormals, a long code: the products stay
    # within the bound (a subnormal weight may be flushed; its product is
    # below 2^-126 |x|)
    shapes = [(512, 1024), (1024, 512)]
    mats = [inputs.stress(r * c, key=(75, m, 0)) for m, (r, c) in enumerate(shapes)]
    ys, xb, word = _run(shapes, mats, 32, seed=1)
    assert word == 0
    for m, (r, c) in enumerate(shapes):
        _check(ys[m], mats[m], xb[m], r, c, 32)


@pytest.mark.gpu
@pytest.mark.slow
def test_gemm_llama3_8b_block():
    # the Llama-3-8B block at batch 64, checked on 64 sampled rows per matrix
    shapes = [s for _, s in inputs.LLAMA3_8B]
    mats = [m for _, _, m in inputs.block(2, 0)]
    batch = 64
    ys, xb, word = _run(shapes, mats, batch, seed=2)
    assert word == 0
    rng = np.random.default_rng(76)
    for m, (r, c) in enumerate(shapes):
        rs = np.sort(rng.choice(r, 64, replace=False))
        _check(ys[m], mats[m], xb[m], r, c, batch, row_sample=rs)


@pytest.mark.gpu
def test_gemm_reports_a_corrupt_block():
    torch = _torch()
    shapes = [(256, 1024), (128, 512)]
    mats = [df11.tile_major(inputs.gaussian(r * c, [77, m]), r, c) for m, (r, c) in enumerate(shapes)]
    dev = df11.DeviceFormat(df11.build_format(mats), "cuda")
    offs = dev.tensors["block_offset"].view(torch.int32)
    offs[5] = offs[5] + 1
    xs = [torch.ones(16, c, dtype=torch.bfloat16, device="cuda") for r, c in shapes]
    ys = [torch.zeros(16, r, dtype=torch.float32, device="cuda") for r, c in shapes]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_gemm(dev, shapes, xs, ys, status)
    torch.cuda.synchronize()
    word = int(status.item()) & 0xFFFFFFFF
    assert word != 0 and not (word & 0x80000000), hex(word)


@pytest.mark.gpu
def test_gemm_refuses_an_impossible_symbol_table():
    # a stored table entry no code can produce (one code of 0 bits) is
    # refused before any role runs: reported, no timeout, tensor memory freed
    torch = _torch()
    shapes = [(256, 1024)]
    mats = [df11.tile_major(inputs.gaussian(256 * 1024, [78]), 256, 1024)]
    dev = df11.DeviceFormat(df11.build_format(mats), "cuda")
    dev.tensors["symbol_table"].view(torch.int32)[300] = 1 << 29
    xs = [torch.ones(16, 1024, dtype=torch.bfloat16, device="cuda")]
    ys = [torch.zeros(16, 256, dtype=torch.float32, device="cuda")]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_gemm(dev, shapes, xs, ys, status)
    torch.cuda.synchronize()
    word = int(status.item()) & 0xFFFFFFFF
    assert word == df11.DF11_ERR_CORRUPT, hex(word)
    # the next launch on the same context works
    dev2 = df11.DeviceFormat(df11.build_format(mats), "cuda")
    status.zero_()
    df11.decompress_gemm(dev2, shapes, xs, ys, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
