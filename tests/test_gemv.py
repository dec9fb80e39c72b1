"""Fused decode + matrix-vector product (df11_decompress_gemv): y_m += W_m x_m
with the BF16 weights decoded on chip and never stored ("Dekompresi yang
disesuaikan untuk inferensi GPU": decompress right before the product).

Reference: the product of the ORIGINAL BF16 weights (bit-exact input of the
decode) with the same BF16 activations, in float64.  Tolerance: the kernel
forms each product exactly in float32 (a BF16 x BF16 product has 16
significant bits) and sums a row's `cols` products in float32 in some order
(per-lane fused multiply-adds, a warp tree, atomic adds), so
|y - y_ref| <= cols * 2^-24 * sum_c |w_c x_c|; the tests allow twice that."""
import ctypes

import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs

SHAPES = [(96, 160), (32, 160), (160, 96), (64, 64), (16, 32)]


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _check(y, W_bits, x_bits, rows, cols, y0=None):
    W = _bf16_to_f64(W_bits).reshape(rows, cols)
    x = _bf16_to_f64(x_bits)
    ref = W @ x + (0 if y0 is None else y0)
    bound = 2 * cols * 2.0 ** -24 * (np.abs(W) @ np.abs(x)) + 1e-30
    err = np.abs(y.astype(np.float64) - ref)
    assert np.all(err <= bound), float((err / bound).max())


def _x_bits(cols, key):
    return inputs.gaussian(cols, [99, key], sigma=1.0)


# ------------------------------------------------------------------- host
def test_gemv_argument_checks_run_before_any_launch():
    # invalid matrix lists are refused on the host (no GPU needed: nothing is
    # launched); the arrays here are the host copies, only checked
    lib = df11.load_library()
    w = np.concatenate([inputs.gaussian(r * c, [98, m]) for m, (r, c) in enumerate(SHAPES)])
    fmt = df11.build_format(w)
    a = fmt.c_arrays
    status = (ctypes.c_uint32 * 4)()
    xbuf = (ctypes.c_uint8 * 4096)()
    ybuf = (ctypes.c_float * 1024)()
    xa = (ctypes.addressof(xbuf) + 15) & ~15

    def call(shapes, x=xa, y=ctypes.addressof(ybuf)):
        mats = (df11.df11_gemv_matrix * max(len(shapes), 1))()
        for m, (r, c) in enumerate(shapes):
            mats[m].rows, mats[m].cols, mats[m].x, mats[m].y = r, c, x, y
        return lib.df11_decompress_gemv(ctypes.byref(a), mats, len(shapes), ctypes.addressof(status), None)

    assert call(SHAPES[:-1]) == 1                    # rows*cols do not cover the stream
    assert call(SHAPES + [(1, 16)]) == 1             # more elements than the stream
    assert call([(96 * 160 // 8, 8)] + SHAPES[1:]) == 1  # cols not a multiple of 16
    assert call(SHAPES, x=xa + 2) == 1               # x not 16-byte aligned
    assert call([]) == 1
    assert call([(1, 16)] * 17) == 1                 # more than 16 matrices


# ------------------------------------------------------------------- device
def _torch():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def _run(shapes, mats, T=64, y0=None, seed=0):
    torch = _torch()
    dev = df11.DeviceFormat(df11.build_format(mats, T), "cuda")
    xb = [_x_bits(c, seed * 100 + m) for m, (r, c) in enumerate(shapes)]
    xs = [torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16) for b in xb]
    ys = [torch.zeros(r, dtype=torch.float32, device="cuda") if y0 is None
          else torch.from_numpy(y0[m].astype(np.float32)).cuda() for m, (r, c) in enumerate(shapes)]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_gemv(dev, shapes, xs, ys, status)
    assert df11.read_status(status) == 0
    for m, ((r, c), W) in enumerate(zip(shapes, mats)):
        _check(ys[m].cpu().numpy(), W, xb[m], r, c, None if y0 is None else y0[m].astype(np.float32))


@pytest.mark.gpu
@pytest.mark.parametrize("T", [32, 64])
def test_gemv_small_matrices(T):
    mats = [inputs.gaussian(r * c, [97, m]) for m, (r, c) in enumerate(SHAPES)]
    _run(SHAPES, mats, T)


@pytest.mark.gpu
def test_gemv_accumulates_into_y():
    mats = [inputs.gaussian(r * c, [96, m]) for m, (r, c) in enumerate(SHAPES)]
    y0 = [np.random.default_rng(m).normal(size=r) for m, (r, c) in enumerate(SHAPES)]
    _run(SHAPES, mats, y0=y0)


@pytest.mark.gpu
def test_gemv_stress_values():
    shapes = [(512, 1024), (1024, 512)]
    mats = [inputs.stress(r * c, key=(95, m, 0)) for m, (r, c) in enumerate(shapes)]
    _run(shapes, mats, seed=3)


@pytest.mark.gpu
def test_gemv_llama3_8b_block():
    shapes = [s for _, s in inputs.LLAMA3_8B]
    mats = [m for _, _, m in inputs.block(2, 0)]
    _run(shapes, mats, seed=4)


@pytest.mark.gpu
def test_gemv_reports_a_corrupt_block():
    torch = _torch()
    mats = [inputs.gaussian(r * c, [94, m]) for m, (r, c) in enumerate(SHAPES)]
    dev = df11.DeviceFormat(df11.build_format(mats), "cuda")
    offs = dev.tensors["block_offset"].view(torch.int32)
    offs[2] = offs[2] + 1
    xs = [torch.ones(c, dtype=torch.bfloat16, device="cuda") for r, c in SHAPES]
    ys = [torch.zeros(r, dtype=torch.float32, device="cuda") for r, c in SHAPES]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    df11.decompress_gemv(dev, SHAPES, xs, ys, status)
    assert df11.read_status(status) != 0
