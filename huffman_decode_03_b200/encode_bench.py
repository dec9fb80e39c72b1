"""Throughput of compressing device-resident weights (``encode_device``).

    python -m huffman_decode_03_b200.encode_bench --workload 2 --reps 5

Times, with CUDA events around each stage on one stream, the exponent
histogram (df11_device_histogram), the host step that turns the 256 counts
into the code (df11_plan_from_histogram, including the device-to-host
read of the counts it waits for) and the device encode (df11_device_encode), on the
synthetic workload's elements already in device memory; checks that the
stream equals the host builder's byte for byte, and times the host builder
(df11_build_format, all host cores) on the same elements for comparison.
Prints one JSON line.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import time

import numpy as np

from . import Df11Error, build_format, df11_arrays, encode_device, inputs, load_library


def main(argv=None):
    import torch

    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--threads-per-block", type=int, default=64)
    args = ap.parse_args(argv)

    mats = [m for _, _, m in inputs.workload_arrays(args.workload)]
    w = np.concatenate(mats)
    n = w.size
    dev = torch.device("cuda")
    wt = torch.from_numpy(w.view(np.int16)).to(dev)
    lib = load_library()
    s = torch.cuda.current_stream()
    sp = ctypes.c_void_p(s.cuda_stream)

    # one full pass through the public call, checked against the host builder
    devfmt, plan = encode_device(wt, args.threads_per_block)
    t0 = time.perf_counter()
    fmt = build_format(mats, args.threads_per_block)
    host_s = time.perf_counter() - t0
    ref = fmt.arrays()
    exact = all(np.array_equal(t.cpu().numpy(), np.ascontiguousarray(ref[k]).reshape(-1).view(np.uint8))
                for k, t in devfmt.tensors.items())

    # stage times: reuse the buffers of the pass above
    hist = torch.empty(256, dtype=torch.int64, device=dev)
    a = plan.c_arrays
    words = int(lib.df11_device_encode_scratch_words(n))
    scratch = torch.empty(words, dtype=torch.int64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    maxb = torch.zeros(1, dtype=torch.int32, device=dev)
    dst = df11_arrays()
    for name in ("encoded_exponent", "packed_sign_mantissa", "gaps", "block_offset", "luts", "code_lengths"):
        setattr(dst, name, devfmt.tensors[name].data_ptr())
    dst.encoded_exponent_bytes = a.encoded_exponent_bytes
    dst.packed_sign_mantissa_bytes = a.packed_sign_mantissa_bytes
    dst.gaps_words = a.gaps_words
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    t_plan, t_enc = [], []
    wp = ctypes.c_void_p(wt.data_ptr())
    for _ in range(args.reps + 1):
        ev[0].record(s)
        if lib.df11_device_histogram(wp, n, ctypes.c_void_p(hist.data_ptr()), sp):
            raise Df11Error(5, "df11_device_histogram")
        ev[1].record(s)
        t1 = time.perf_counter()
        counts = hist.cpu().numpy()  # waits for the histogram
        h = ctypes.c_void_p()
        if lib.df11_plan_from_histogram(counts.ctypes.data, args.threads_per_block, ctypes.byref(h)):
            raise Df11Error(5, "df11_plan_from_histogram")
        lib.df11_free(h)
        t_plan.append(time.perf_counter() - t1)
        ev[1].record(s)
        st = lib.df11_device_encode(plan._h, wp, ctypes.byref(dst), ctypes.c_void_p(scratch.data_ptr()), words,
                                    ctypes.c_void_p(maxb.data_ptr()), ctypes.c_void_p(status.data_ptr()), sp)
        if st:
            raise Df11Error(st, "df11_device_encode")
        ev[2].record(s)
        torch.cuda.synchronize()
        t_enc.append(ev[1].elapsed_time(ev[2]))
    # the histogram alone (its events are not interleaved with host work)
    hs = []
    for _ in range(args.reps + 1):
        ev[0].record(s)
        lib.df11_device_histogram(wp, n, ctypes.c_void_p(hist.data_ptr()), sp)
        ev[1].record(s)
        torch.cuda.synchronize()
        hs.append(ev[0].elapsed_time(ev[1]))
    med = lambda xs: float(np.median(xs[1:]))  # first repetition is a warm-up
    hist_ms, enc_ms, plan_ms = med(hs), med(t_enc), 1000 * med(t_plan)
    total_ms = hist_ms + plan_ms + enc_ms
    print(json.dumps({
        "workload": inputs.WORKLOADS[args.workload], "elements": n, "bf16_bytes": 2 * n,
        "histogram_ms": round(hist_ms, 4), "plan_host_ms": round(plan_ms, 4), "encode_ms": round(enc_ms, 4),
        "total_ms": round(total_ms, 4), "bf16_in_GBps": round(2 * n / total_ms / 1e6, 1),
        "bytes_equal_host_builder": bool(exact and int(status.item()) == 0),
        "host_builder_s": round(host_s, 3), "host_cores": os.cpu_count(),
    }))


if __name__ == "__main__":
    main()
