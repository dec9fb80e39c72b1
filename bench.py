#!/usr/bin/env python3
"""DF11 decompression benchmark on B200.

One step = one pass of the whole decode path over one compressed stream
(stage, locate, decode, scan, place, merge, store) -- one kernel launch per
stream; the 32-block streaming workload makes 32 launches per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2]
    python bench.py --impl reference ...   # the CPU oracle as the reference arm

Prints ONE JSON line (rank 0).  ``value`` is BF16-out GB/s (2 bytes per
element written / kernel time, summed over ranks); ``roofline`` relates the
kernel's algorithmic HBM bytes (compressed bytes read + BF16 bytes written)
per launch to the measured B200 copy bandwidth.  Under torchrun each rank
decodes its own transformer block (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DF11 decompress GB/s (BF16 out) and % of HBM roofline, 1×B200, bit-exact"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
KERNEL_NAME = "df11_decode_kernel"
# the decode kernel's source: the kernel and its shared per-block decode
KERNEL_SOURCES = [os.path.join(ROOT, "huffman_decode_03_b200", "csrc", f) for f in ("df11_decode.cu", "df11_block.cuh")]
PROFILES = os.path.join(ROOT, "profiles")


# ----------------------------------------------------------------- helpers
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", type=int, default=2, choices=[1, 2, 3, 4, 5],
                    help="1 single 1024x1024, 2 Llama-3-8B block, 3 stress 64Mi, "
                         "4 Llama-3-70B block, 5 32 Llama-3-8B blocks streamed")
    ap.add_argument("--threads-per-block", type=int, default=64)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-flush", action="store_true", help="do not flush L2 between timed steps")
    return ap.parse_args(argv)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def shard(workload: int, rank: int, world: int):
    """Which streams a rank decodes.  Blocks of a model are independent
    (each has its own code), so ranks take disjoint blocks: weak scaling for
    workloads 1-4 (rank r takes block r of the same shape), an even split of
    the 32 blocks for workload 5."""
    if workload == 5:
        return [(5, b) for b in range(32) if b % world == rank]
    return [(workload, rank)]


def reduce_over_ranks(ms_step, e2e_ms, n_elems, good, device, world):
    """Whole-job numbers: the slowest rank's times, the elements of all
    ranks, and bit-exactness only if every rank was exact."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms_step, e2e_ms], dtype=torch.float64, device=device)
    n = torch.tensor([float(n_elems)], dtype=torch.float64, device=device)
    g = torch.tensor([1.0 if good else 0.0], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(n, op=dist.ReduceOp.SUM)
        dist.all_reduce(g, op=dist.ReduceOp.MIN)
    return float(t[0]), float(t[1]), float(n[0]), bool(g[0] > 0)


def scaling_kind(workload: int) -> str:
    return "strong" if workload == 5 else "weak"


def load_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for path in KERNEL_SOURCES:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: int, n_elems: int):
    """DRAM bytes per launch from a committed ncu capture (profiles/traffic_*.txt),
    if it was taken of the current kernel source; scaled by elements when the
    capture covered a different number of outputs."""
    try:
        names = sorted(os.listdir(PROFILES))
    except OSError:
        return None
    for name in names:
        if not (name.startswith("traffic_") and name.endswith(".txt")):
            continue
        rec = {}
        with open(os.path.join(PROFILES, name)) as f:
            for line in f:
                if line.strip() and not line.startswith("#") and ":" in line:
                    k, v = line.split(":", 1)
                    rec[k.strip()] = v.strip()
        if rec.get("kernel_source_sha256_16") != kernel_source_hash() or rec.get("workload") != str(workload):
            continue
        dram = float(rec["dram_bytes_read"]) + float(rec["dram_bytes_write"])
        return dram * n_elems / float(rec["elements"])
    return None


def stream_algorithmic_bytes(s: dict) -> int:
    """Bytes one launch must move: EncodedExponent + PackedSignMantissa + Gaps
    + BlockOffset + LUTs + CodeLengths read, 2 bytes per BF16 written."""
    n = s["n"]
    read = (s["total_bits"] + 7) // 8 + n + (5 * s["num_segments"] + 7) // 8 + 4 * (s["num_blocks"] + 1) \
        + 256 * s["num_luts"] + 256
    return read + 2 * n


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        inside = [r for ts, r in rows if self.t0 and self.t1 and self.t0 - 0.3 <= ts <= self.t1 + 0.3]
        use = inside or [r for _, r in rows]
        sm = [float(r[1]) for r in use if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in use if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i in range(4) if r[5 + i].lower() == "active"})
        return {
            "sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None,
            "reasons": reasons,
            "samples": len(use),
            "samples_in_timed_region": len(inside),
        }


# ------------------------------------------------------------- GPU arm
def prepare_streams(streams, T, device, verify=True):
    """Builds (host) and uploads each stream; checks one decode bit-exactly."""
    import torch

    import huffman_decode_03_b200 as df11
    from huffman_decode_03_b200 import inputs

    out = []
    for wl, blk in streams:
        mats = [m for _, _, m in inputs.workload_arrays(wl, blk)]
        fmt = df11.build_format(mats, T)
        dev = df11.DeviceFormat(fmt, device, pin_host=True)
        info = fmt.info()
        exact = None
        if verify:
            w = torch.from_numpy(np.concatenate(mats).view(np.int16) if len(mats) > 1 else mats[0].view(np.int16))
            status = torch.zeros(1, dtype=torch.int32, device=device)
            got = df11.decompress(dev, None, status)
            ok_status = df11.read_status(status) == 0
            exact = bool(ok_status and torch.equal(got.view(torch.int16), w.to(device)))
            del got, w
        del mats
        fmt.free()
        out.append({"dev": dev, "info": info, "exact": exact})
    return out


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import huffman_decode_03_b200 as df11

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=device, timeout=timedelta(seconds=300))

    streams = shard(args.workload, rank, world)
    prepared = prepare_streams(streams, args.threads_per_block, device)
    n_total = sum(p["info"]["n"] for p in prepared)
    exact = all(p["exact"] for p in prepared)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    outbuf = torch.empty(max(p["info"]["n"] for p in prepared), dtype=torch.bfloat16, device=device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        for p in prepared:
            df11.decompress(p["dev"], outbuf, status, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.5)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    if sampler:
        sampler.mark("t0")
    for i in range(args.steps):
        if not args.no_flush:
            flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(device)
    if sampler:
        sampler.mark("t1")
    if world > 1:
        dist.barrier()
    ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms_mean = float(np.mean(ms))
    ok = df11.read_status(status) == 0

    # end to end through the host-buffer entry point (pinned host memory)
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    host_out = torch.empty(outbuf.numel(), dtype=torch.int16).pin_memory()
    h2d = sum(sum(t.numel() for t in p["dev"].host_tensors.values()) for p in prepared)
    d2h = 2 * n_total
    for p in prepared:  # warm
        df11.decompress_host(p["dev"], outbuf, host_out, status, stream)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for p in prepared:
            df11.decompress_host(p["dev"], outbuf, host_out, status, stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    ok = ok and df11.read_status(status) == 0
    clocks = sampler.stop() if sampler else None

    ms_step, e2e_ms, n_all, good = reduce_over_ranks(ms_mean, e2e_ms, n_total, exact and ok, device, world)

    if rank == 0:
        info0 = prepared[0]["info"]
        alg = sum(stream_algorithmic_bytes(p["dev"].scalars) for p in prepared) / len(prepared)
        per_launch_ms = ms_mean / len(prepared)
        peak, peak_src = load_peak()
        achieved = alg / (per_launch_ms * 1e-3) / 1e9
        traffic = recorded_traffic(args.workload, prepared[0]["info"]["n"])
        value = 2.0 * n_all / (ms_step * 1e-3) / 1e9
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 5),
            "higher_is_better": True,
            "scaling": scaling_kind(args.workload),
            "vs_baseline": None,
            "dtype": "u16",
            "data": "synthetic (seeded numpy PCG64, BF16 by round-to-nearest-even; no trained weights)",
            "config": {
                "workload": _workload_name(args.workload),
                "elements_per_rank_step": int(n_total),
                "streams_per_step": len(prepared),
                "threads_per_block": args.threads_per_block,
                "compressed_bytes": int(sum(p["info"]["compressed_bytes"] for p in prepared)),
                "bits_per_weight": round(8 + info0["avg_code_len"], 4),
                "exponent_entropy_bits": round(info0["entropy_bits"], 4),
                "max_code_len": info0["max_code_len"],
                "num_luts": info0["num_luts"],
                "l2": "flushed between timed steps (256 MiB write, outside the events)"
                      if not args.no_flush else "not flushed",
                "parallelism": f"dp{world}" if world > 1 else "single",
            },
            "bit_exact": bool(good),
            "roofline": {
                "bound": "hbm",
                "kernel": KERNEL_NAME,
                "achieved": round(achieved, 1),
                "peak": peak,
                "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": None if traffic is None else int(traffic),
                "algorithmic_bytes_per_launch": int(alg),
                "peak_source": peak_src,
            },
            "e2e": {
                "value": round(2.0 * n_all / (e2e_ms * 1e-3) / 1e9, 2),
                "unit": UNIT,
                "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h),
                "steps": e2e_steps,
                "entry_point": "df11_decompress_host (pinned host arrays in, BF16 to pinned host out)",
            },
            "gpu_launches": args.steps * len(prepared),
            "clocks": clocks,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _workload_name(w):
    from huffman_decode_03_b200 import inputs

    return inputs.WORKLOADS[w]


# ------------------------------------------------------------ CPU oracle
def _oracle_sample(workload: int, elems: int):
    from huffman_decode_03_b200 import inputs
    from oracle import oracle

    mats = [m for _, _, m in inputs.workload_arrays(1 if workload == 1 else (2 if workload == 5 else workload), 0)]
    w = np.concatenate(mats) if len(mats) > 1 else mats[0]
    w = np.ascontiguousarray(w[:elems])
    return oracle, oracle.build_format(w, 64)


def cpu_baseline(workload: int, seconds: float) -> dict:
    """The oracle's bit-by-bit tree-walk decode, single thread, on a bounded
    sample of the same workload (its leading elements), repeated for about
    `seconds` of CPU time."""
    elems = 1 << 22
    oracle, fmt = _oracle_sample(workload, elems)
    n = fmt["n"]
    reps, t = 0, 0.0
    while t < seconds:
        t0 = time.perf_counter()
        oracle.decode_format(fmt)
        t += time.perf_counter() - t0
        reps += 1
    gbs = 2.0 * n * reps / t / 1e9
    return {"value": round(gbs, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"first {n} elements of {_workload_name(workload)}, decoded {reps}x "
                      f"({t:.1f} s) by the bit-by-bit tree walk"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    # calibrate: elements per step so that the whole run ends in ~60 s
    oracle, fmt = _oracle_sample(args.workload, 1 << 20)
    t0 = time.perf_counter()
    oracle.decode_format(fmt)
    rate = fmt["n"] / max(time.perf_counter() - t0, 1e-6)
    per_step = int(min(1 << 24, max(1 << 14, rate * 60.0 / max(1, args.steps + args.warmup))))
    oracle, fmt = _oracle_sample(args.workload, per_step)
    n = fmt["n"]
    for _ in range(args.warmup):
        oracle.decode_format(fmt)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.decode_format(fmt)
        times.append(time.perf_counter() - t0)
    mean = float(np.mean(times))
    value = 2.0 * n / mean / 1e9
    sample = f"first {n} elements of {_workload_name(args.workload)} per step, bit-by-bit tree walk"
    print(json.dumps({
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(mean * 1e3, 4),
        "higher_is_better": True,
        "scaling": scaling_kind(args.workload),
        "vs_baseline": None,
        "dtype": "u16",
        "data": "synthetic (seeded numpy PCG64)",
        "config": {"workload": _workload_name(args.workload), "elements_per_step": n},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
