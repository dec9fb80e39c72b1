"""df11_device_encode_static: the device encode with its scratch in a fixed
array inside the library (nothing allocated by the call).  Two calls in a
row must give exactly what the caller-scratch entry point gives; plans
beyond its limit are refused before anything runs.  This file is collected
last, so on a GPU it runs after every other test has used the library."""
import ctypes

import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs


def test_static_scratch_limit_is_refused_on_the_host():
    # 2^29 + 1 elements: one chunk more than the array holds; the size check
    # comes before any CUDA call, so this runs without a GPU
    lib = df11.load_library()
    hist = np.zeros(256, np.uint64)
    hist[120] = (1 << 28) + 1
    hist[121] = 1 << 28
    h = ctypes.c_void_p()
    assert lib.df11_plan_from_histogram(hist.ctypes.data, 64, ctypes.byref(h)) == 0
    plan = df11.Format(h.value, lib)
    dst = df11.df11_arrays()
    st = lib.df11_device_encode_static(plan._h, ctypes.c_void_p(16), ctypes.byref(dst), ctypes.c_void_p(16),
                                       ctypes.c_void_p(16), None)
    assert st == 3  # DF11_ERR_TOO_LARGE
    assert lib.df11_device_encode_static(None, None, ctypes.byref(dst), None, None, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("key,n", [(95, 3_000_017), (96, 70_001)])
def test_static_scratch_matches_caller_scratch_twice(key, n):
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    w = inputs.gaussian(n, [key])
    wt = torch.from_numpy(w.view(np.int16)).cuda()
    ref, _ = df11.encode_device(wt)
    for _ in range(2):  # two calls in a row reuse the same array
        got, _ = df11.encode_device(wt, static_scratch=True)
        for name, t in ref.tensors.items():
            assert torch.equal(got.tensors[name], t), name
        assert got.scalars == ref.scalars
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = df11.decompress(got, None, status)
    assert df11.read_status(status) == 0
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), w)
