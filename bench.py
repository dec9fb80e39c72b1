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
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, vendor figure (7.7 TB/s HGX, 8 TB/s DGX)
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
    ap.add_argument("--rans", default="2,3,4",
                    help="workloads on which the rANS variant of the exponent coder is measured at N=1 and "
                         "reported in the line's rans object (comma-separated ids, or 'none')")
    ap.add_argument("--per-workload", default="4,3,1",
                    help="further workloads measured after the headline one at N=1, reported in the "
                         "line's per_workload object (comma-separated ids, or 'none')")
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
def prepare_streams(streams, T, device, verify=True, pin_host=True):
    """Builds (host) and uploads each stream; checks one decode bit-exactly."""
    import torch

    import huffman_decode_03_b200 as df11
    from huffman_decode_03_b200 import inputs

    out = []
    for i, (wl, blk) in enumerate(streams):
        mats = [m for _, _, m in inputs.workload_arrays(wl, blk)]
        fmt = df11.build_format(mats, T)
        dev = df11.DeviceFormat(fmt, device, pin_host=pin_host)
        info = fmt.info()
        exact = None
        w = torch.from_numpy(np.concatenate(mats).view(np.int16) if len(mats) > 1 else mats[0].view(np.int16))
        if verify:
            status = torch.zeros(1, dtype=torch.int32, device=device)
            got = df11.decompress(dev, None, status)
            ok_status = df11.read_status(status) == 0
            exact = bool(ok_status and torch.equal(got.view(torch.int16), w.to(device)))
            del got
        del mats
        fmt.free()
        # the last stream's original bits stay (host) for the check after the timed loop
        out.append({"dev": dev, "info": info, "exact": exact, "bits": w if i == len(streams) - 1 else None})
        del w
    return out


def time_steps(prepared, outbuf, status, stream, flush, steps, warmup, between=None):
    """Per-step CUDA-event times (ms) of `steps` steps after `warmup` untimed
    ones; a step decodes every prepared stream into outbuf, one launch each;
    the L2 flush (if any) runs before each step, outside its events."""
    import torch

    import huffman_decode_03_b200 as df11

    def step():
        for p in prepared:
            df11.decompress(p["dev"], outbuf, status, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if between:
        between("t0")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if between:
        between("t1")
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def last_output_exact(prepared, outbuf) -> bool:
    """After timed steps: outbuf holds the last stream's decode; it must equal
    that stream's original bits."""
    import torch

    p = prepared[-1]
    n = p["info"]["n"]
    return bool(torch.equal(outbuf[:n].view(torch.int16), p["bits"].to(outbuf.device)))


def roofline_fraction(prepared, ms_per_launch, peak):
    alg = sum(stream_algorithmic_bytes(p["dev"].scalars) for p in prepared) / len(prepared)
    achieved = alg / (ms_per_launch * 1e-3) / 1e9
    return alg, achieved, achieved / peak


def measure_workload(wl, args, device, peak):
    """One further workload at N=1: build, upload, check, time; its record for
    the line's per_workload object."""
    import torch

    streams = shard(wl, 0, 1)
    prepared = prepare_streams(streams, args.threads_per_block, device, pin_host=False)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    n_max = max(p["info"]["n"] for p in prepared)
    outbuf = torch.empty(n_max, dtype=torch.bfloat16, device=device)
    flush = None if args.no_flush else torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    ms = time_steps(prepared, outbuf, status, stream, flush, args.steps, args.warmup)
    import huffman_decode_03_b200 as df11

    exact = all(p["exact"] for p in prepared) and df11.read_status(status) == 0 and last_output_exact(prepared,
                                                                                                      outbuf)
    med = float(statistics.median(ms))
    n_total = sum(p["info"]["n"] for p in prepared)
    per_launch = med / len(prepared)
    alg, achieved, frac = roofline_fraction(prepared, per_launch, peak)
    info0 = prepared[0]["info"]
    traffic = recorded_traffic(wl, info0["n"])
    rec = {
        "workload": _workload_name(wl),
        "elements": int(n_total),
        "launches_per_step": len(prepared),
        "ms_per_step": round(med, 5),
        "ms_per_launch": round(per_launch, 5),
        "value": round(2.0 * n_total / (med * 1e-3) / 1e9, 2),
        "unit": UNIT,
        "roofline_achieved_gbs": round(achieved, 1),
        "frac": round(frac, 4),
        "frac_vs_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
        "algorithmic_bytes_per_launch": int(alg),
        "traffic": None if traffic is None else int(traffic),
        "bits_per_weight": round(8 + info0["avg_code_len"], 4),
        "max_code_len": info0["max_code_len"],
        "num_luts": info0["num_luts"],
        "bit_exact": bool(exact),
        "steps": args.steps,
        "timing": "median of per-step CUDA-event times",
    }
    del prepared, outbuf, flush
    torch.cuda.empty_cache()
    return rec


def rans_algorithmic_bytes(fmt) -> int:
    """Bytes one rANS-variant launch must move: its compressed arrays read,
    2 bytes per BF16 written."""
    return fmt.compressed_bytes() + 2 * fmt.scalars()["n"]


def measure_rans(wl, args, device, peak):
    """The rANS variant of the exponent coder on one workload at N=1: build,
    upload, check, time (median of per-step CUDA-event times, L2 flushed)."""
    import torch

    import huffman_decode_03_b200 as df11
    from huffman_decode_03_b200 import inputs

    mats = [m for _, _, m in inputs.workload_arrays(wl, 0)]
    w = np.concatenate(mats) if len(mats) > 1 else mats[0]
    del mats
    fmt = df11.rans_build_format(w)
    dev = df11.RansDeviceFormat(fmt, device)
    n = dev.n
    alg = rans_algorithmic_bytes(fmt)
    comp = fmt.compressed_bytes()
    fmt.free()
    bits = torch.from_numpy(w.view(np.int16)).to(device)
    del w
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    flush = None if args.no_flush else torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    df11.rans_decompress(dev, out, status, stream)
    exact = df11.read_status(status) == 0 and bool(torch.equal(out.view(torch.int16), bits))
    out.zero_()
    for _ in range(args.warmup):
        df11.rans_decompress(dev, out, status, stream)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in ev:
        if flush is not None:
            flush.zero_()
        e0.record(stream)
        df11.rans_decompress(dev, out, status, stream)
        e1.record(stream)
    torch.cuda.synchronize()
    med = float(statistics.median([e0.elapsed_time(e1) for e0, e1 in ev]))
    exact = exact and df11.read_status(status) == 0 and bool(torch.equal(out.view(torch.int16), bits))
    achieved = alg / (med * 1e-3) / 1e9
    rec = {
        "workload": _workload_name(wl),
        "kernel": "rans_decode_kernel",
        "elements": int(n),
        "compressed_bytes": int(comp),
        "bits_per_weight": round(8.0 * (comp - n) / n + 8, 4),
        "ms_per_launch": round(med, 5),
        "value": round(2.0 * n / (med * 1e-3) / 1e9, 2),
        "unit": UNIT,
        "roofline_achieved_gbs": round(achieved, 1),
        "frac": round(achieved / peak, 4),
        "algorithmic_bytes_per_launch": int(alg),
        "bit_exact": bool(exact),
        "steps": args.steps,
        "timing": "median of per-step CUDA-event times",
    }
    del dev, out, bits, flush
    torch.cuda.empty_cache()
    return rec


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
    flush = None if args.no_flush else torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.5)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    ms = time_steps(prepared, outbuf, status, stream, flush, args.steps, args.warmup,
                    between=sampler.mark if sampler else None)
    if world > 1:
        dist.barrier()
    ms_med = float(statistics.median(ms))
    ms_mean = float(np.mean(ms))
    # the timed launches' own result: status word, and the last stream's output
    ok = df11.read_status(status) == 0 and last_output_exact(prepared, outbuf)

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
    last_n = prepared[-1]["info"]["n"]
    ok = ok and bool(torch.equal(host_out[:last_n], prepared[-1]["bits"]))
    clocks = sampler.stop() if sampler else None

    ms_step, e2e_ms, n_all, good = reduce_over_ranks(ms_med, e2e_ms, n_total, exact and ok, device, world)

    if rank == 0:
        info0 = prepared[0]["info"]
        per_launch_ms = ms_med / len(prepared)
        peak, peak_src = load_peak()
        alg, achieved, frac = roofline_fraction(prepared, per_launch_ms, peak)
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
            "ms_per_step_mean": round(ms_mean, 5),
            "timing": "ms_per_step and value: median of the per-step CUDA-event times (max over ranks)",
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
                "frac": round(frac, 4),
                "traffic": None if traffic is None else int(traffic),
                "algorithmic_bytes_per_launch": int(alg),
                "peak_source": peak_src,
                "frac_vs_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                "nominal_peak": NOMINAL_HBM_GBS,
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
    # further workloads, measured the same way, at N=1 only
    extra = [] if args.per_workload.strip().lower() in ("", "none") else \
        [int(x) for x in args.per_workload.split(",") if int(x) != args.workload]
    if world == 1 and extra:
        del prepared, outbuf, flush, host_out
        torch.cuda.empty_cache()
        peak, _ = load_peak()
        per = [measure_workload(wl, args, device, peak) for wl in extra]
        line["per_workload"] = per
        line["gpu_launches"] += sum(r["steps"] * r["launches_per_step"] for r in per)
    rans = [] if args.rans.strip().lower() in ("", "none") else [int(x) for x in args.rans.split(",")]
    if world == 1 and rans:
        peak, _ = load_peak()
        line["rans"] = [measure_rans(wl, args, device, peak) for wl in rans]
        line["gpu_launches"] += sum(r["steps"] for r in line["rans"])
    if rank == 0:
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
def _oracle_sample(workload: int, elems: int, keep: bool = False):
    from huffman_decode_03_b200 import inputs
    from oracle import oracle

    mats = [m for _, _, m in inputs.workload_arrays(1 if workload == 1 else (2 if workload == 5 else workload), 0)]
    w = np.concatenate(mats) if len(mats) > 1 else mats[0]
    w = np.ascontiguousarray(w[:elems])
    fmt = oracle.build_format(w, 64)
    return (oracle, fmt, w) if keep else (oracle, fmt)


def host_cpu() -> dict:
    """The host's CPU model and the cores this process may run on."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    return {"cpu_model": model, "nproc": cores}


CPU_BASELINE_MAX_ELEMS = 1 << 28


def _oracle_decode_all_cores(oracle, fmt, threads: int) -> np.ndarray:
    """The oracle's tree walk run on `threads` threads at once: each decodes
    the exponents of a run of whole format blocks (df11o_decode_range from the
    run's first code start to the next run's), and the BF16 values are then
    reassembled from them and the sign/mantissa bytes.  ctypes releases the
    GIL during the C calls."""
    from concurrent.futures import ThreadPoolExecutor

    T = fmt["threads_per_block"]
    offs = fmt["block_offset"]
    gaps = fmt["gaps"]
    nb = len(offs) - 1
    bits = int(fmt["total_bits"])
    out = np.empty(fmt["n"], np.uint16)
    sm = fmt["packed_sign_mantissa"]
    cuts = [nb * k // (4 * threads) for k in range(4 * threads + 1)]

    def start(b):
        return bits if b >= nb else 64 * T * b + int(gaps[T * b])

    def work(k):
        b0, b1 = cuts[k], cuts[k + 1]
        if b0 == b1:
            return
        e = oracle.decode_range(fmt["encoded_exponent"], bits, start(b0), start(b1), fmt["code_lengths"],
                                fmt["codes"]).astype(np.uint16)
        o0, o1 = int(offs[b0]), int(offs[b1])
        m = sm[o0:o1].astype(np.uint16)
        out[o0:o1] = ((m & 0x80) << 8) | (e << 7) | (m & 0x7F)

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, range(len(cuts) - 1)))
    return out


def cpu_baseline(workload: int, seconds: float) -> dict:
    """The oracle's bit-by-bit tree-walk decode of the workload's stream
    (the whole stream, or its first 2^28 elements; one block of the 32-block
    workload) on the host: on one core (df11o_decode), and on every core
    (df11o_decode_range over runs of whole blocks, one thread each); each
    repeated for about seconds / 2."""
    hc = host_cpu()
    oracle, fmt, w = _oracle_sample(workload, CPU_BASELINE_MAX_ELEMS, keep=True)
    n = fmt["n"]

    def timed(fn):
        reps, t, exact = 0, 0.0, True
        while reps == 0 or t < seconds / 2:
            t0 = time.perf_counter()
            got = fn()
            t += time.perf_counter() - t0
            reps += 1
            exact = exact and np.array_equal(got, w)
        return 2.0 * n * reps / t / 1e9, reps, t, exact

    one, r1, t1, x1 = timed(lambda: oracle.decode_format(fmt))
    allc, ra, ta, xa = timed(lambda: _oracle_decode_all_cores(oracle, fmt, hc["nproc"]))
    what = "whole stream" if n < CPU_BASELINE_MAX_ELEMS else "first elements"
    return {"value": round(one, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{what} of {_workload_name(workload)} ({n} elements), decoded {r1}x ({t1:.1f} s) "
                      f"by the bit-by-bit tree walk on one core",
            "bit_exact": bool(x1),
            "all_cores": {"value": round(allc, 4), "unit": UNIT, "cores": hc["nproc"], "reps": ra,
                          "seconds": round(ta, 2), "bit_exact": bool(xa),
                          "how": "the same tree walk over runs of whole format blocks, one thread per run "
                                 "(df11o_decode_range), BF16 reassembled per run"},
            **hc}


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
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample,
                         **host_cpu()},
        "timing": "ms_per_step and value: mean of the per-step wall-clock times of the oracle decode",
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
