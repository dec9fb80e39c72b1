"""The C-ABI library loads without a GPU and exports every entry point that
include/df11.h declares; the header's struct layouts match the binding."""
import ctypes
import os
import re
import subprocess

import numpy as np

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import build as build_mod

HEADER_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(df11_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_binding_exports():
    assert set(declared_functions()) == set(df11.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = df11.load_library()
    out = subprocess.run(["nm", "-D", "--defined-only", build_mod.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_struct_sizes_match_c():
    # compile a tiny probe against the header and compare sizeof/offsetof
    src = r'''
#include <stdio.h>
#include <stddef.h>
#include "df11.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(df11_arrays), offsetof(df11_arrays, encoded_exponent),
         offsetof(df11_arrays, code_lengths), sizeof(df11_info), offsetof(df11_info, histogram),
         sizeof(df11_gemv_matrix), offsetof(df11_gemv_matrix, x), offsetof(df11_gemv_matrix, y),
         sizeof(df11_rans_arrays), offsetof(df11_rans_arrays, words),
         offsetof(df11_rans_arrays, packed_sign_mantissa_bytes));
  return 0;
}
'''
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "probe.c")
        exe = os.path.join(d, "probe")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", HEADER_DIR, c, "-o", exe], check=True)
        got = [int(x) for x in subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()]
    A, I, G, R = df11.df11_arrays, df11.df11_info, df11.df11_gemv_matrix, df11.df11_rans_arrays
    assert got == [ctypes.sizeof(A), A.encoded_exponent.offset, A.code_lengths.offset,
                   ctypes.sizeof(I), I.histogram.offset, ctypes.sizeof(G), G.x.offset, G.y.offset,
                   ctypes.sizeof(R), R.words.offset, R.packed_sign_mantissa_bytes.offset]


def test_strerror_covers_all_codes():
    lib = df11.load_library()
    texts = {lib.df11_strerror(i).decode() for i in range(8)}
    assert len(texts) == 8 and "unknown status" not in texts


def test_array_views_keep_the_format_alive():
    # views of a temporary Format stay valid: each keeps the handle alive
    import gc

    from huffman_decode_03_b200 import inputs

    w = inputs.gaussian(1 << 20, [5])
    ref = df11.build_format(w)
    want = ref.arrays()["block_offset"].copy()
    offs = df11.build_format(w).arrays()["block_offset"]
    gc.collect()
    others = [df11.build_format(inputs.gaussian(1 << 18, [6, i])) for i in range(4)]  # reuse freed memory
    assert np.array_equal(offs, want)
    assert len(others) == 4
