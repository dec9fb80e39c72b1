"""B200-native DFloat11 (DF11) decompression: Python binding of the C ABI.

Every entry point forwards to ``libdf11_b200.so`` (declared in
``include/df11.h``); this module only marshals arguments.  PyTorch supplies
device memory and CUDA streams.  There is no CPU fallback: if the library
cannot be loaded, or the CUDA path is used without a GPU, the call raises.

Names follow the DFloat11 page (id.news.hada.io/topic?id=20542): a stream's
``encoded_exponent`` (EncodedExponent), ``packed_sign_mantissa``
(PackedSignMantissa), ``gaps``, ``block_offset``, ``luts`` and
``code_lengths`` (CodeLengths).
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

import numpy as np

from . import build as _build

__all__ = [
    "Df11Error", "Format", "DeviceFormat", "build_format", "decompress",
    "decompress_gemv", "decompress_gemm", "gemm_scratch_bytes", "decompress_host", "encode_device",
    "read_status", "tile_major", "load_library", "RansFormat", "RansDeviceFormat", "rans_build_format",
    "rans_decompress",
]

DF11_OK = 0
DF11_ERR_CORRUPT = 6


class df11_gemv_matrix(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_uint32),
        ("cols", ctypes.c_uint32),
        ("x", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
    ]


class df11_gemm_matrix(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_uint32),
        ("cols", ctypes.c_uint32),
        ("x", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
    ]


class Df11Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        msg = _strerror(status)
        super().__init__(f"{what}: {msg} (status {status})" if what else msg)


class df11_arrays(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_uint64),
        ("total_bits", ctypes.c_uint64),
        ("num_segments", ctypes.c_uint64),
        ("threads_per_block", ctypes.c_uint32),
        ("num_blocks", ctypes.c_uint32),
        ("num_luts", ctypes.c_uint32),
        ("max_code_len", ctypes.c_uint32),
        ("max_block_elems", ctypes.c_uint32),
        ("min_code_len", ctypes.c_uint32),
        ("encoded_exponent", ctypes.c_void_p),
        ("encoded_exponent_bytes", ctypes.c_uint64),
        ("packed_sign_mantissa", ctypes.c_void_p),
        ("packed_sign_mantissa_bytes", ctypes.c_uint64),
        ("gaps", ctypes.c_void_p),
        ("gaps_words", ctypes.c_uint64),
        ("block_offset", ctypes.c_void_p),
        ("luts", ctypes.c_void_p),
        ("code_lengths", ctypes.c_void_p),
        ("symbol_table", ctypes.c_void_p),
    ]


class df11_rans_arrays(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_uint64),
        ("num_words", ctypes.c_uint64),
        ("prob_bits", ctypes.c_uint32),
        ("chunks", ctypes.c_uint32),
        ("num_blocks", ctypes.c_uint32),
        ("max_block_words", ctypes.c_uint32),
        ("words", ctypes.c_void_p),
        ("states", ctypes.c_void_p),
        ("block_word", ctypes.c_void_p),
        ("lane_words", ctypes.c_void_p),
        ("freq", ctypes.c_void_p),
        ("packed_sign_mantissa", ctypes.c_void_p),
        ("packed_sign_mantissa_bytes", ctypes.c_uint64),
    ]


class df11_info(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_uint64),
        ("total_bits", ctypes.c_uint64),
        ("compressed_bytes", ctypes.c_uint64),
        ("entropy_bits", ctypes.c_double),
        ("avg_code_len", ctypes.c_double),
        ("distinct_exponents", ctypes.c_uint32),
        ("max_code_len", ctypes.c_uint32),
        ("num_luts", ctypes.c_uint32),
        ("threads_per_block", ctypes.c_uint32),
        ("histogram", ctypes.c_uint64 * 256),
    ]


EXPORTS = (
    "df11_build_format", "df11_format_arrays", "df11_format_info", "df11_free",
    "df11_strerror", "df11_decompress", "df11_decompress_sms", "df11_decompress_gemv", "df11_decompress_gemm",
    "df11_gemm_scratch_bytes", "df11_tile_major", "df11_decompress_host", "df11_read_status", "df11_device_histogram", "df11_plan_from_histogram",
    "df11_device_encode_scratch_words", "df11_device_encode", "df11_device_encode_static",
    "df11_rans_build", "df11_rans_format_arrays", "df11_rans_free", "df11_rans_decompress",
    "df11_symbol_table",
)

_lib = None


def load_library(path: str | None = None):
    """Loads (building first when the sources are newer) the C-ABI library."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    if path is None:
        path = _build.LIB_PATH
        if not os.path.exists(path) or _build._stale():
            _build.build()
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.df11_build_format.argtypes = [P, P, ctypes.c_int, ctypes.c_uint32, ctypes.POINTER(P)]
    lib.df11_build_format.restype = ctypes.c_int
    lib.df11_format_arrays.argtypes = [P, ctypes.POINTER(df11_arrays)]
    lib.df11_format_arrays.restype = ctypes.c_int
    lib.df11_format_info.argtypes = [P, ctypes.POINTER(df11_info)]
    lib.df11_format_info.restype = ctypes.c_int
    lib.df11_free.argtypes = [P]
    lib.df11_free.restype = None
    lib.df11_strerror.argtypes = [ctypes.c_int]
    lib.df11_strerror.restype = ctypes.c_char_p
    lib.df11_decompress.argtypes = [ctypes.POINTER(df11_arrays), P, P, P]
    lib.df11_decompress.restype = ctypes.c_int
    lib.df11_decompress_sms.argtypes = [ctypes.POINTER(df11_arrays), P, P, P, ctypes.c_uint32]
    lib.df11_decompress_sms.restype = ctypes.c_int
    lib.df11_decompress_gemv.argtypes = [ctypes.POINTER(df11_arrays), ctypes.POINTER(df11_gemv_matrix),
                                         ctypes.c_uint32, P, P]
    lib.df11_decompress_gemv.restype = ctypes.c_int
    lib.df11_decompress_gemm.argtypes = [ctypes.POINTER(df11_arrays), ctypes.POINTER(df11_gemm_matrix),
                                         ctypes.c_uint32, ctypes.c_uint32, P, ctypes.c_uint64, P, P]
    lib.df11_decompress_gemm.restype = ctypes.c_int
    lib.df11_gemm_scratch_bytes.argtypes = [ctypes.POINTER(df11_gemm_matrix), ctypes.c_uint32, ctypes.c_uint32]
    lib.df11_gemm_scratch_bytes.restype = ctypes.c_uint64
    lib.df11_tile_major.argtypes = [P, ctypes.c_uint32, ctypes.c_uint32, P]
    lib.df11_symbol_table.argtypes = [P, P, ctypes.c_uint32, P]
    lib.df11_symbol_table.restype = ctypes.c_int
    lib.df11_tile_major.restype = ctypes.c_int
    lib.df11_decompress_host.argtypes = [
        ctypes.POINTER(df11_arrays), ctypes.POINTER(df11_arrays), P, P, P, P]
    lib.df11_decompress_host.restype = ctypes.c_int
    lib.df11_read_status.argtypes = [P, P]
    lib.df11_read_status.restype = ctypes.c_int
    lib.df11_device_histogram.argtypes = [P, ctypes.c_uint64, P, P]
    lib.df11_device_histogram.restype = ctypes.c_int
    lib.df11_plan_from_histogram.argtypes = [P, ctypes.c_uint32, ctypes.POINTER(P)]
    lib.df11_plan_from_histogram.restype = ctypes.c_int
    lib.df11_device_encode_scratch_words.argtypes = [ctypes.c_uint64]
    lib.df11_device_encode_scratch_words.restype = ctypes.c_uint64
    lib.df11_device_encode.argtypes = [P, P, ctypes.POINTER(df11_arrays), P, ctypes.c_uint64, P, P, P]
    lib.df11_device_encode.restype = ctypes.c_int
    lib.df11_device_encode_static.argtypes = [P, P, ctypes.POINTER(df11_arrays), P, P, P]
    lib.df11_device_encode_static.restype = ctypes.c_int
    lib.df11_rans_build.argtypes = [P, P, ctypes.c_int, ctypes.c_uint32, ctypes.POINTER(P)]
    lib.df11_rans_build.restype = ctypes.c_int
    lib.df11_rans_format_arrays.argtypes = [P, ctypes.POINTER(df11_rans_arrays)]
    lib.df11_rans_format_arrays.restype = ctypes.c_int
    lib.df11_rans_free.argtypes = [P]
    lib.df11_rans_free.restype = None
    lib.df11_rans_decompress.argtypes = [ctypes.POINTER(df11_rans_arrays), P, P, P]
    lib.df11_rans_decompress.restype = ctypes.c_int
    if path == _build.LIB_PATH:
        _lib = lib
    return lib


def _strerror(status: int) -> str:
    try:
        return load_library().df11_strerror(int(status)).decode()
    except OSError:
        return f"status {status}"


def _check(status: int, what: str):
    if status != DF11_OK:
        raise Df11Error(status, what)


# --------------------------------------------------------------------- host
class Format:
    """A host-resident DF11 stream (handle from ``df11_build_format``)."""

    def __init__(self, handle: int, lib):
        self._h = ctypes.c_void_p(handle)
        self._lib = lib
        a = df11_arrays()
        _check(lib.df11_format_arrays(self._h, ctypes.byref(a)), "df11_format_arrays")
        self.c_arrays = a

    def __del__(self):
        self.free()

    def free(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._lib.df11_free(h)
            self._h = None

    @property
    def n(self) -> int:
        return int(self.c_arrays.n)

    def _view(self, ptr, count, dtype):
        if count == 0 or not ptr:
            return np.zeros(0, dtype)
        nbytes = int(count) * np.dtype(dtype).itemsize
        buf = (ctypes.c_uint8 * nbytes).from_address(ptr)
        buf._owner = self  # the array keeps the buffer, the buffer keeps the handle
        return np.frombuffer(buf, dtype=dtype, count=int(count))

    def arrays(self) -> dict:
        """numpy views of the host arrays; each view keeps this handle (and
        so its memory) alive."""
        a = self.c_arrays
        return {
            "encoded_exponent": self._view(a.encoded_exponent, a.encoded_exponent_bytes, np.uint8),
            "packed_sign_mantissa": self._view(a.packed_sign_mantissa, a.packed_sign_mantissa_bytes, np.uint8),
            "gaps": self._view(a.gaps, a.gaps_words, np.uint64),
            "block_offset": self._view(a.block_offset, a.num_blocks + 1, np.uint32),
            "luts": self._view(a.luts, a.num_luts * 256, np.uint8).reshape(a.num_luts, 256),
            "code_lengths": self._view(a.code_lengths, 256, np.uint8),
            # the decoders' derived table (not part of the compressed bytes)
            "symbol_table": self._view(a.symbol_table, 4096 if a.symbol_table else 0, np.uint32),
        }

    def info(self) -> dict:
        i = df11_info()
        _check(self._lib.df11_format_info(self._h, ctypes.byref(i)), "df11_format_info")
        return {
            "n": int(i.n), "total_bits": int(i.total_bits), "compressed_bytes": int(i.compressed_bytes),
            "entropy_bits": float(i.entropy_bits), "avg_code_len": float(i.avg_code_len),
            "distinct_exponents": int(i.distinct_exponents), "max_code_len": int(i.max_code_len),
            "num_luts": int(i.num_luts), "threads_per_block": int(i.threads_per_block),
            "num_segments": int(self.c_arrays.num_segments), "num_blocks": int(self.c_arrays.num_blocks),
            "max_block_elems": int(self.c_arrays.max_block_elems),
            "histogram": np.array(i.histogram[:], np.uint64),
        }

    def scalars(self) -> dict:
        a = self.c_arrays
        return {f: int(getattr(a, f)) for f in (
            "n", "total_bits", "num_segments", "threads_per_block", "num_blocks", "num_luts",
            "max_code_len", "max_block_elems", "min_code_len")}


def build_format(mats: Sequence[np.ndarray] | np.ndarray, threads_per_block: int = 64) -> Format:
    """Compresses BF16 bit patterns (uint16 arrays, or torch bfloat16/int16
    CPU tensors) into one DF11 stream; matrices are concatenated in order."""
    lib = load_library()
    if isinstance(mats, np.ndarray) or hasattr(mats, "data_ptr"):
        mats = [mats]
    keep = []
    for m in mats:
        if hasattr(m, "data_ptr"):  # torch tensor
            m = m.detach().contiguous().cpu().view(-1)
            import torch
            m = m.view(torch.int16).numpy().view(np.uint16)
        keep.append(np.ascontiguousarray(np.asarray(m).view(np.uint16).reshape(-1)))
    k = len(keep)
    ptrs = (ctypes.c_void_p * max(k, 1))(*[m.ctypes.data if m.size else None for m in keep])
    counts = (ctypes.c_uint64 * max(k, 1))(*[m.size for m in keep])
    h = ctypes.c_void_p()
    _check(lib.df11_build_format(ptrs, counts, k, int(threads_per_block), ctypes.byref(h)),
           "df11_build_format")
    return Format(h.value, lib)


# ------------------------------------------------------------------- device
class DeviceFormat:
    """A DF11 stream resident in device memory (arrays held as torch tensors)."""

    def __init__(self, fmt: Format, device="cuda", pin_host: bool = False):
        import torch

        self.device = torch.device(device)
        self.scalars = fmt.scalars()
        arrs = fmt.arrays()
        self.tensors = {}
        self.host_tensors = {}
        for name, arr in arrs.items():
            if arr.size == 0 and name == "symbol_table":
                continue
            t = torch.from_numpy(np.ascontiguousarray(arr).reshape(-1).view(np.uint8))
            if pin_host:
                t = t.pin_memory()
                self.host_tensors[name] = t
            self.tensors[name] = t.to(self.device, non_blocking=False)
        self.c_arrays = self._struct(self.tensors)
        self.c_host_arrays = self._struct(self.host_tensors) if pin_host else None

    @classmethod
    def from_tensors(cls, scalars: dict, tensors: dict, device) -> "DeviceFormat":
        """A stream whose arrays are already device tensors (uint8, named as in
        ``Format.arrays()``), e.g. the output of ``encode_device``."""
        import torch

        self = cls.__new__(cls)
        self.device = torch.device(device)
        self.scalars = dict(scalars)
        self.tensors = dict(tensors)
        self.host_tensors = {}
        self.c_arrays = self._struct(self.tensors)
        self.c_host_arrays = None
        return self

    def _struct(self, ts) -> df11_arrays:
        a = df11_arrays()
        for k, v in self.scalars.items():
            setattr(a, k, v)
        a.encoded_exponent = ts["encoded_exponent"].data_ptr()
        a.encoded_exponent_bytes = ts["encoded_exponent"].numel()
        a.packed_sign_mantissa = ts["packed_sign_mantissa"].data_ptr()
        a.packed_sign_mantissa_bytes = ts["packed_sign_mantissa"].numel()
        a.gaps = ts["gaps"].data_ptr()
        a.gaps_words = ts["gaps"].numel() // 8
        a.block_offset = ts["block_offset"].data_ptr()
        a.luts = ts["luts"].data_ptr()
        a.code_lengths = ts["code_lengths"].data_ptr()
        if "symbol_table" in ts:
            a.symbol_table = ts["symbol_table"].data_ptr()
        return a

    @property
    def n(self) -> int:
        return self.scalars["n"]

    def nbytes(self) -> int:
        return sum(t.numel() for t in self.tensors.values())


def _stream_ptr(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def decompress(dev: DeviceFormat, out=None, status=None, stream=None, max_sms: int = 0):
    """Rebuilds the BF16 stream on the GPU (asynchronous, stream-ordered).
    Returns ``out`` (a torch.bfloat16 tensor of n elements, allocated if None).
    ``max_sms`` > 0 caps the SMs the decoder occupies (df11_decompress_sms)."""
    import torch

    if out is None:
        out = torch.empty(dev.n, dtype=torch.bfloat16, device=dev.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev.device)
    assert out.is_cuda and out.is_contiguous() and out.numel() >= dev.n and out.element_size() == 2
    args = (ctypes.byref(dev.c_arrays), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(status.data_ptr()),
            _stream_ptr(stream))
    if max_sms:
        _check(load_library().df11_decompress_sms(*args, int(max_sms)), "df11_decompress_sms")
    else:
        _check(load_library().df11_decompress(*args), "df11_decompress")
    return out


def decompress_gemv(dev: DeviceFormat, shapes, xs, ys, status=None, stream=None):
    """Decode and use in one pass (df11_decompress_gemv): ``ys[m] += W_m @ xs[m]``
    for the stream's matrices, of ``shapes[m] = (rows, cols)`` in stream order;
    the decoded weights never reach memory.  ``xs``: CUDA bfloat16 vectors of
    length cols (16-byte aligned); ``ys``: CUDA float32 vectors of length rows,
    accumulated (zero them for y = W x).  Asynchronous; returns ``ys``."""
    import torch

    k = len(shapes)
    if not (len(xs) == len(ys) == k):
        raise ValueError("one activation vector and one output vector per matrix")
    mats = (df11_gemv_matrix * max(k, 1))()
    for m, ((rows, cols), x, y) in enumerate(zip(shapes, xs, ys)):
        if x.dtype != torch.bfloat16 or y.dtype != torch.float32 or not (x.is_cuda and y.is_cuda):
            raise ValueError("x must be CUDA bfloat16 and y CUDA float32")
        if x.numel() != cols or y.numel() != rows or not (x.is_contiguous() and y.is_contiguous()):
            raise ValueError(f"matrix {m}: x needs {cols} and y {rows} contiguous elements")
        mats[m].rows, mats[m].cols, mats[m].x, mats[m].y = rows, cols, x.data_ptr(), y.data_ptr()
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev.device)
    _check(load_library().df11_decompress_gemv(ctypes.byref(dev.c_arrays), mats, k,
                                               ctypes.c_void_p(status.data_ptr()), _stream_ptr(stream)),
           "df11_decompress_gemv")
    return ys


def tile_major(w, rows: int, cols: int) -> np.ndarray:
    """The rows x cols row-major BF16 matrix ``w`` (uint16 bit patterns) in
    the tile-major order ``decompress_gemm`` reads (df11_tile_major): 128 x 64
    tiles, row tiles in order, within one the column tiles in order, within a
    tile its rows.  Compress the result with ``build_format``."""
    src = np.ascontiguousarray(np.asarray(w).view(np.uint16).reshape(-1))
    if src.size != rows * cols:
        raise ValueError(f"{src.size} elements for a {rows} x {cols} matrix")
    dst = np.empty_like(src)
    _check(load_library().df11_tile_major(src.ctypes.data, rows, cols, dst.ctypes.data), "df11_tile_major")
    return dst


def _gemm_mats(shapes, xs, ys, batch):
    import torch

    k = len(shapes)
    if not (len(xs) == len(ys) == k):
        raise ValueError("one activation matrix and one output matrix per weight matrix")
    mats = (df11_gemm_matrix * max(k, 1))()
    for m, ((rows, cols), x, y) in enumerate(zip(shapes, xs, ys)):
        if x.dtype != torch.bfloat16 or y.dtype != torch.float32 or not (x.is_cuda and y.is_cuda):
            raise ValueError("x must be CUDA bfloat16 and y CUDA float32")
        if tuple(x.shape) != (batch, cols) or tuple(y.shape) != (batch, rows) or not (
                x.is_contiguous() and y.is_contiguous()):
            raise ValueError(f"matrix {m}: x must be ({batch}, {cols}) and y ({batch}, {rows}), contiguous")
        mats[m].rows, mats[m].cols, mats[m].x, mats[m].y = rows, cols, x.data_ptr(), y.data_ptr()
    return mats


def decompress_gemm(dev: DeviceFormat, shapes, xs, ys, status=None, stream=None, scratch=None):
    """Decode and multiply on the tensor cores (df11_decompress_gemm):
    ``ys[m] += xs[m] @ W_m.T`` for the stream's matrices, of ``shapes[m] =
    (rows, cols)`` in stream order, each stored tile-major (``tile_major``);
    the decoded weights never reach memory.  ``xs[m]``: CUDA bfloat16
    (batch, cols); ``ys[m]``: CUDA float32 (batch, rows), accumulated; batch
    a multiple of 16 up to 256.  ``scratch``: a CUDA uint8 tensor of at least
    ``gemm_scratch_bytes`` bytes (allocated when None).  Asynchronous; returns
    ``ys``."""
    import torch

    batch = int(xs[0].shape[0]) if len(xs) else 0
    mats = _gemm_mats(shapes, xs, ys, batch)
    lib = load_library()
    need = int(lib.df11_gemm_scratch_bytes(mats, len(shapes), batch))
    if need == 0:
        raise Df11Error(1, "df11_gemm_scratch_bytes")
    if scratch is None:
        scratch = torch.empty(need, dtype=torch.uint8, device=dev.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev.device)
    _check(lib.df11_decompress_gemm(ctypes.byref(dev.c_arrays), mats, len(shapes), batch,
                                    ctypes.c_void_p(scratch.data_ptr()), scratch.numel(),
                                    ctypes.c_void_p(status.data_ptr()), _stream_ptr(stream)),
           "df11_decompress_gemm")
    return ys


def gemm_scratch_bytes(shapes, batch: int) -> int:
    """Scratch bytes ``decompress_gemm`` needs (0: invalid shapes or batch)."""
    mats = (df11_gemm_matrix * max(len(shapes), 1))()
    for m, (rows, cols) in enumerate(shapes):
        mats[m].rows, mats[m].cols = rows, cols
    return int(load_library().df11_gemm_scratch_bytes(mats, len(shapes), int(batch)))


def decompress_host(dev: DeviceFormat, out_dev, out_host, status, stream=None):
    """Host-to-host decode: copies the pinned host arrays in, decodes, copies
    the BF16 result to ``out_host`` (pinned, 2n bytes).  Asynchronous."""
    assert dev.c_host_arrays is not None, "DeviceFormat(pin_host=True) required"
    _check(load_library().df11_decompress_host(
        ctypes.byref(dev.c_host_arrays), ctypes.byref(dev.c_arrays), ctypes.c_void_p(out_dev.data_ptr()),
        ctypes.c_void_p(out_host.data_ptr()), ctypes.c_void_p(status.data_ptr()), _stream_ptr(stream)),
        "df11_decompress_host")
    return out_host


def encode_device(w, threads_per_block: int = 64, stream=None, static_scratch: bool = False):
    """Compresses BF16 weights that are already on the GPU: exponent histogram
    on the device (df11_device_histogram), the code from the 256 counts on the
    host (df11_plan_from_histogram), every array on the device
    (df11_device_encode).  ``w``: a contiguous CUDA tensor of bfloat16 (or
    16-bit integer) patterns, any shape, read in memory order.  Returns
    ``(DeviceFormat, Format)``: the stream, whose arrays never left the device,
    and its plan (code, LUTs, statistics).  Synchronises ``stream`` twice: the
    counts and the largest block size come back to the host.  With
    ``static_scratch`` the encode step runs through df11_device_encode_static
    (scratch inside the library; streams of at most 2^29 elements)."""
    import torch

    lib = load_library()
    flat = w.detach().reshape(-1)
    if flat.dtype == torch.bfloat16:
        flat = flat.view(torch.int16)
    if not (flat.is_cuda and flat.element_size() == 2 and flat.is_contiguous()):
        raise ValueError("encode_device needs a contiguous CUDA tensor of 16-bit patterns")
    dev = flat.device
    n = flat.numel()
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(s.cuda_stream)
    wp = ctypes.c_void_p(flat.data_ptr() if n else None)
    hist = torch.empty(256, dtype=torch.int64, device=dev)
    _check(lib.df11_device_histogram(wp, n, ctypes.c_void_p(hist.data_ptr()), sp), "df11_device_histogram")
    s.synchronize()
    hist_host = hist.cpu().numpy()
    h = ctypes.c_void_p()
    _check(lib.df11_plan_from_histogram(hist_host.ctypes.data, int(threads_per_block), ctypes.byref(h)),
           "df11_plan_from_histogram")
    plan = Format(h.value, lib)
    a = plan.c_arrays
    sizes = {
        "encoded_exponent": int(a.encoded_exponent_bytes),
        "packed_sign_mantissa": int(a.packed_sign_mantissa_bytes),
        "gaps": 8 * int(a.gaps_words),
        "block_offset": 4 * (int(a.num_blocks) + 1),
        "luts": 256 * int(a.num_luts),
        "code_lengths": 256,
    }
    with torch.cuda.stream(s):
        tensors = {k: torch.empty(v, dtype=torch.uint8, device=dev) for k, v in sizes.items()}
        words = int(lib.df11_device_encode_scratch_words(n))
        scratch = None if static_scratch else torch.empty(max(words, 1), dtype=torch.int64, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        maxb = torch.zeros(1, dtype=torch.int32, device=dev)
    dst = df11_arrays()
    dst.encoded_exponent = tensors["encoded_exponent"].data_ptr()
    dst.encoded_exponent_bytes = sizes["encoded_exponent"]
    dst.packed_sign_mantissa = tensors["packed_sign_mantissa"].data_ptr()
    dst.packed_sign_mantissa_bytes = sizes["packed_sign_mantissa"]
    dst.gaps = tensors["gaps"].data_ptr()
    dst.gaps_words = int(a.gaps_words)
    dst.block_offset = tensors["block_offset"].data_ptr()
    dst.luts = tensors["luts"].data_ptr()
    dst.code_lengths = tensors["code_lengths"].data_ptr()
    if static_scratch:
        _check(lib.df11_device_encode_static(plan._h, wp, ctypes.byref(dst), ctypes.c_void_p(maxb.data_ptr()),
                                             ctypes.c_void_p(status.data_ptr()), sp),
               "df11_device_encode_static")
    else:
        _check(lib.df11_device_encode(plan._h, wp, ctypes.byref(dst), ctypes.c_void_p(scratch.data_ptr()), words,
                                      ctypes.c_void_p(maxb.data_ptr()), ctypes.c_void_p(status.data_ptr()), sp),
               "df11_device_encode")
    s.synchronize()
    st = int(status.item())
    if st:
        raise Df11Error(6, f"df11_device_encode: the elements do not match their histogram (status word {st})")
    scalars = plan.scalars()
    scalars["max_block_elems"] = int(maxb.item())
    table = plan.arrays()["symbol_table"]
    if table.size:  # the decoders' derived table, from the plan's code
        tensors["symbol_table"] = torch.from_numpy(table.view(np.uint8).copy()).to(dev)
    return DeviceFormat.from_tensors(scalars, tensors, dev), plan


def read_status(status, stream=None) -> int:
    """Synchronises the stream and returns the kernel status (0 = ok)."""
    return int(load_library().df11_read_status(ctypes.c_void_p(status.data_ptr()), _stream_ptr(stream)))


# --------------------------------------------------------------------- rANS
class RansFormat:
    """A host-resident stream of the rANS variant (handle from ``df11_rans_build``):
    the same BF16 values, exponents coded with rANS instead of Huffman codes."""

    def __init__(self, handle: int, lib):
        self._h = ctypes.c_void_p(handle)
        self._lib = lib
        a = df11_rans_arrays()
        _check(lib.df11_rans_format_arrays(self._h, ctypes.byref(a)), "df11_rans_format_arrays")
        self.c_arrays = a

    def __del__(self):
        self.free()

    def free(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._lib.df11_rans_free(h)
            self._h = None

    def _view(self, ptr, count, dtype):
        if count == 0 or not ptr:
            return np.zeros(0, dtype)
        nbytes = int(count) * np.dtype(dtype).itemsize
        buf = (ctypes.c_uint8 * nbytes).from_address(ptr)
        buf._owner = self
        return np.frombuffer(buf, dtype=dtype, count=int(count))

    def arrays(self) -> dict:
        a = self.c_arrays
        return {
            "words": self._view(a.words, a.num_words + 8 if a.n else 0, np.uint16),
            "states": self._view(a.states, 32 * a.num_blocks, np.uint32),
            "block_word": self._view(a.block_word, a.num_blocks + 1 if a.n else 0, np.uint32),
            "lane_words": self._view(a.lane_words, 32 * a.num_blocks, np.uint8),
            "freq": self._view(a.freq, 256 if a.n else 0, np.uint16),
            "packed_sign_mantissa": self._view(a.packed_sign_mantissa, a.packed_sign_mantissa_bytes, np.uint8),
        }

    def scalars(self) -> dict:
        a = self.c_arrays
        return {f: int(getattr(a, f)) for f in ("n", "num_words", "prob_bits", "chunks", "num_blocks",
                                                 "max_block_words")}

    def compressed_bytes(self) -> int:
        """Bytes of the stream: words, start states, lane counts, block
        offsets, the model and the sign/mantissa bytes (without padding)."""
        s = self.scalars()
        return (2 * s["num_words"] + (4 + 1) * 32 * s["num_blocks"] + 4 * (s["num_blocks"] + 1) + 2 * 256
                + s["n"])


def rans_build_format(mats, chunks: int = 10) -> RansFormat:
    """Compresses BF16 bit patterns (uint16 arrays) into one stream of the
    rANS variant (df11_rans_build); matrices are concatenated in order."""
    lib = load_library()
    if isinstance(mats, np.ndarray):
        mats = [mats]
    keep = [np.ascontiguousarray(np.asarray(m).view(np.uint16).reshape(-1)) for m in mats]
    k = len(keep)
    ptrs = (ctypes.c_void_p * max(k, 1))(*[m.ctypes.data if m.size else None for m in keep])
    counts = (ctypes.c_uint64 * max(k, 1))(*[m.size for m in keep])
    h = ctypes.c_void_p()
    _check(lib.df11_rans_build(ptrs, counts, k, int(chunks), ctypes.byref(h)), "df11_rans_build")
    return RansFormat(h.value, lib)


class RansDeviceFormat:
    """A rANS-variant stream resident in device memory (torch tensors)."""

    def __init__(self, fmt: RansFormat, device="cuda"):
        import torch

        self.device = torch.device(device)
        self.scalars = fmt.scalars()
        self.tensors = {}
        for name, arr in fmt.arrays().items():
            t = torch.from_numpy(np.ascontiguousarray(arr).reshape(-1).view(np.uint8).copy())
            self.tensors[name] = t.to(self.device)
        a = df11_rans_arrays()
        for k, v in self.scalars.items():
            setattr(a, k, v)
        ts = self.tensors
        a.words = ts["words"].data_ptr()
        a.states = ts["states"].data_ptr()
        a.block_word = ts["block_word"].data_ptr()
        a.lane_words = ts["lane_words"].data_ptr()
        a.freq = ts["freq"].data_ptr()
        a.packed_sign_mantissa = ts["packed_sign_mantissa"].data_ptr()
        a.packed_sign_mantissa_bytes = ts["packed_sign_mantissa"].numel()
        self.c_arrays = a

    @property
    def n(self) -> int:
        return self.scalars["n"]


def rans_decompress(dev: RansDeviceFormat, out=None, status=None, stream=None):
    """Rebuilds the BF16 stream of the rANS variant on the GPU (asynchronous,
    stream-ordered); returns ``out`` (allocated if None)."""
    import torch

    if out is None:
        out = torch.empty(dev.n, dtype=torch.bfloat16, device=dev.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=dev.device)
    assert out.is_cuda and out.is_contiguous() and out.numel() >= dev.n and out.element_size() == 2
    _check(load_library().df11_rans_decompress(ctypes.byref(dev.c_arrays), ctypes.c_void_p(out.data_ptr()),
                                               ctypes.c_void_p(status.data_ptr()), _stream_ptr(stream)),
           "df11_rans_decompress")
    return out
