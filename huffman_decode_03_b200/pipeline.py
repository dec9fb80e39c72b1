"""Per-block decompress-and-use pipeline.

"Dekompresi per transformer block" (DFloat11 page): a transformer block's
weights are decompressed right before the block runs, used, and discarded,
so only one block's BF16 weights exist at a time.  Decompressing block i+1
on a second CUDA stream while block i's matrices are being multiplied hides
the decompression behind the work that consumes it.

``BlockPipeline`` holds two BF16 scratch buffers (each sized for the largest
block) and orders the two streams with events:

  * block i decodes into buffer i % 2 on the decode stream;
  * the consumer of block i waits for that decode, runs on the caller's
    stream and marks buffer i % 2 free when it is done;
  * the decode of block i + 2 waits until buffer i % 2 is free.

Every decode goes through ``df11_decompress`` (the CUDA kernel); this module
only orders launches.  Run as a module it times one such pass with a
stand-in consumer (the block's seven GEMMs against a batch of activations):
``python -m huffman_decode_03_b200.pipeline --blocks 8 --batch 64``; with
``--gemv`` it compares, at batch 1, decompress + cuBLAS matrix-vector
products against the fused ``df11_decompress_gemv``; with ``--gemm``, at
``--batch`` activation vectors, decompress + cuBLAS GEMMs against the fused
tensor-core ``df11_decompress_gemm`` (weights stored tile-major).
"""
from __future__ import annotations

import argparse
import json

from . import DeviceFormat, build_format, decompress, inputs


class BlockPipeline:
    """Decompress blocks one ahead of their use, on a side stream."""

    def __init__(self, blocks, device="cuda", decode_sms: int = 0):
        """``decode_sms`` > 0 caps the SMs each decode occupies, leaving the
        others to the consumer's kernels (0 = every SM: the decoder then
        holds the whole GPU while it runs and overlap is limited to its
        tail)."""
        import torch

        if not blocks:
            raise ValueError("BlockPipeline needs at least one block")
        self.decode_sms = int(decode_sms)
        self.blocks = list(blocks)
        self.device = torch.device(device)
        nmax = max(b.n for b in self.blocks)
        self.bufs = [torch.empty(nmax, dtype=torch.bfloat16, device=self.device) for _ in range(2)]
        self.status = torch.zeros(len(self.blocks), dtype=torch.int32, device=self.device)
        self.decode_stream = torch.cuda.Stream(self.device)
        self._decoded = [torch.cuda.Event() for _ in range(2)]
        self._released = [torch.cuda.Event() for _ in range(2)]

    def run(self, consume, stream=None, overlap: bool = True):
        """Enqueues the whole pass.  ``consume(i, w)`` enqueues the use of block
        i's weights ``w`` (a bfloat16 view of its n elements, valid until the
        call returns) on the current stream, which is ``stream`` (default: the
        current stream).  With ``overlap=False`` every decode runs on that same
        stream, in order, before its block's use.  Asynchronous; returns the
        per-block status words (int32, non-zero = corrupt block)."""
        import torch

        main = stream if stream is not None else torch.cuda.current_stream(self.device)
        dec = self.decode_stream if overlap else main
        self.status.zero_()
        dec.wait_stream(main)  # uploads, status reset and earlier work come first
        nb = len(self.blocks)

        def launch(i):
            j = i % 2
            if i >= 2:
                dec.wait_event(self._released[j])  # block i-2 is done with buffer j
            n = self.blocks[i].n
            decompress(self.blocks[i], self.bufs[j][:n], self.status[i:i + 1], stream=dec,
                       max_sms=self.decode_sms)
            self._decoded[j].record(dec)

        launch(0)
        for i in range(nb):
            if i + 1 < nb:
                launch(i + 1)  # queued before block i's use: runs alongside it
            j = i % 2
            main.wait_event(self._decoded[j])
            with torch.cuda.stream(main):
                consume(i, self.bufs[j][:self.blocks[i].n])
            self._released[j].record(main)
        return self.status


# ------------------------------------------------------------ stand-in use
def block_gemms(shapes, x):
    """A consumer that multiplies each matrix of a block (row-major, shapes
    (rows, cols) in stream order) by the activations ``x`` [batch, >= cols]
    and returns the list of outputs [batch, rows]."""
    def consume(w):
        outs, off = [], 0
        for rows, cols in shapes:
            m = w[off:off + rows * cols].view(rows, cols)
            outs.append(x[:, :cols] @ m.t())
            off += rows * cols
        return outs
    return consume


def _timed(fn, reps, inner):
    """Median over `reps` samples of the device time of one call of `fn`;
    each sample times `inner` calls back to back between two CUDA events, so
    that host-side launch gaps between calls (small kernels the host cannot
    feed fast enough) do not count as device time."""
    import numpy as np
    import torch

    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for _ in range(reps):
        e0.record()
        for _ in range(inner):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / inner)
    return float(np.median(ts))


def _bench(args):
    import numpy as np
    import torch

    dev = torch.device("cuda")
    shapes = [s for _, s in inputs.LLAMA3_8B]
    fmts, dense = [], []
    for b in range(args.blocks):
        mats = [m for _, _, m in inputs.block(5, b)]
        fmts.append(DeviceFormat(build_format(mats), dev))
        if args.dense:
            dense.append(torch.from_numpy(np.concatenate(mats).view(np.int16)).to(dev).view(torch.bfloat16))
    g = torch.Generator(device="cpu").manual_seed(7)
    x = (torch.randn(args.batch, max(c for _, c in shapes), generator=g) * 0.5).to(torch.bfloat16).to(dev)
    gemm = block_gemms(shapes, x)
    pipe = BlockPipeline(fmts, dev)
    sink = []

    def consume(i, w):
        gemm(w)

    def consume_keep(i, w):
        sink.append(gemm(w))

    def timed(fn, reps):
        return _timed(fn, reps, args.inner)

    out = torch.empty_like(pipe.bufs[0])
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def decode_only():
        for f in fmts:
            decompress(f, out[:f.n], st)

    res = {
        "blocks": args.blocks, "batch": args.batch, "block": "llama3_8b (q,k,v,o,gate,up,down)",
        "decode_only_ms": timed(decode_only, args.reps),
        "serial_ms": timed(lambda: pipe.run(consume, overlap=False), args.reps),
        "overlapped_ms": timed(lambda: pipe.run(consume, overlap=True), args.reps),
    }
    for sms in args.decode_sms:
        pipe.decode_sms = sms
        res[f"overlapped_decode_{sms}sms_ms"] = timed(lambda: pipe.run(consume, overlap=True), args.reps)
    pipe.decode_sms = 0
    if args.dense:
        res["dense_gemm_only_ms"] = timed(lambda: [gemm(w) for w in dense], args.reps)
    if args.check:
        pipe.run(consume_keep, overlap=True)
        torch.cuda.synchronize()
        assert int(pipe.status.abs().sum()) == 0
        exact = all(torch.equal(a.view(torch.int16), b.view(torch.int16))
                    for i, w in enumerate(dense) for a, b in zip(sink[i], gemm(w)))
        res["gemm_outputs_equal_dense"] = bool(exact)
    nb = args.blocks
    res["per_block_us"] = {k[:-3]: round(1000 * v / nb, 1) for k, v in res.items() if k.endswith("_ms")}
    print(json.dumps(res))


def _bench_gemv(args):
    """Batch-1 use of each block: decompress, then the seven matrix-vector
    products with cuBLAS, against df11_decompress_gemv (decode and product
    in one pass, no BF16 weights written)."""
    import numpy as np
    import torch

    from . import decompress_gemv

    dev = torch.device("cuda")
    shapes = [s for _, s in inputs.LLAMA3_8B]
    fmts, dense = [], []
    for b in range(args.blocks):
        mats = [m for _, _, m in inputs.block(5, b)]
        fmts.append(DeviceFormat(build_format(mats), dev))
        dense.append(torch.from_numpy(np.concatenate(mats).view(np.int16)).to(dev).view(torch.bfloat16))
    g = torch.Generator(device="cpu").manual_seed(11)
    xs = [(torch.randn(c, generator=g)).to(torch.bfloat16).to(dev) for _, c in shapes]
    ys = [torch.zeros(r, dtype=torch.float32, device=dev) for r, _ in shapes]
    buf = torch.empty(max(f.n for f in fmts), dtype=torch.bfloat16, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def gemvs(w):
        off, outs = 0, []
        for (r, c), x in zip(shapes, xs):
            outs.append(w[off:off + r * c].view(r, c) @ x)
            off += r * c
        return outs

    def separate():
        for f in fmts:
            decompress(f, buf[:f.n], st)
            gemvs(buf[:f.n])

    def fused():
        for y in ys:
            y.zero_()
        for f in fmts:
            decompress_gemv(f, shapes, xs, ys, st)

    def timed(fn, reps):
        return _timed(fn, reps, args.inner)

    nb = args.blocks
    res = {"blocks": nb, "batch": 1, "block": "llama3_8b (q,k,v,o,gate,up,down)",
           "decode_then_cublas_gemv_ms": timed(separate, args.reps),
           "fused_decode_gemv_ms": timed(fused, args.reps),
           "cublas_gemv_dense_ms": timed(lambda: [gemvs(w) for w in dense], args.reps)}
    # the fused result of the last block against cuBLAS on the original weights
    for y in ys:
        y.zero_()
    decompress_gemv(fmts[-1], shapes, xs, ys, st)
    ref = gemvs(dense[-1])
    torch.cuda.synchronize()
    rel = max(float(((y - r.float()).abs().max() / r.float().abs().max()).item()) for y, r in zip(ys, ref))
    res["max_rel_diff_vs_cublas_bf16_out"] = rel
    res["per_block_us"] = {k[:-3]: round(1000 * v / nb, 1) for k, v in res.items() if k.endswith("_ms")}
    print(json.dumps(res))


def _bench_gemm(args):
    """Batch-B use of each block: decompress, then the seven GEMMs with
    cuBLAS, against df11_decompress_gemm (decode into tensor-core operand
    tiles and multiply in one kernel, no BF16 weights written)."""
    import numpy as np
    import torch

    from . import decompress_gemm, gemm_scratch_bytes, tile_major

    dev = torch.device("cuda")
    shapes = [s for _, s in inputs.LLAMA3_8B]
    B = args.batch
    rowmajor, tiled, dense = [], [], []
    for b in range(args.blocks):
        mats = [m for _, _, m in inputs.block(5, b)]
        rowmajor.append(DeviceFormat(build_format(mats), dev))
        tiled.append(DeviceFormat(build_format([tile_major(m, r, c) for m, (r, c) in zip(mats, shapes)]), dev))
        if args.dense:
            dense.append(torch.from_numpy(np.concatenate(mats).view(np.int16)).to(dev).view(torch.bfloat16))
    g = torch.Generator(device="cpu").manual_seed(12)
    xs = [torch.randn(B, c, generator=g).to(torch.bfloat16).to(dev) for _, c in shapes]
    ys = [torch.zeros(B, r, dtype=torch.float32, device=dev) for r, _ in shapes]
    buf = torch.empty(max(f.n for f in rowmajor), dtype=torch.bfloat16, device=dev)
    scratch = torch.empty(gemm_scratch_bytes(shapes, B), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def gemms(w):
        off, outs = 0, []
        for (r, c), x in zip(shapes, xs):
            outs.append(x @ w[off:off + r * c].view(r, c).T)
            off += r * c
        return outs

    def separate():
        for f in rowmajor:
            decompress(f, buf[:f.n], st)
            gemms(buf[:f.n])

    def fused():
        for y in ys:
            y.zero_()
        for f in tiled:
            decompress_gemm(f, shapes, xs, ys, st, scratch=scratch)

    def timed(fn, reps):
        return _timed(fn, reps, args.inner)

    nb = args.blocks
    res = {"blocks": nb, "batch": B, "block": "llama3_8b (q,k,v,o,gate,up,down)",
           "decode_then_cublas_gemm_ms": timed(separate, args.reps),
           "fused_decode_gemm_ms": timed(fused, args.reps)}
    if args.dense:
        res["cublas_gemm_dense_ms"] = timed(lambda: [gemms(w) for w in dense], args.reps)
        # the fused result of the last block against cuBLAS on the original weights
        for y in ys:
            y.zero_()
        decompress_gemm(tiled[-1], shapes, xs, ys, st, scratch=scratch)
        ref = gemms(dense[-1])
        torch.cuda.synchronize()
        res["max_rel_diff_vs_cublas_bf16_out"] = max(
            float(((y - r.float()).abs().max() / r.float().abs().max()).item()) for y, r in zip(ys, ref))
    torch.cuda.synchronize()
    res["status"] = int(st.item())
    res["per_block_us"] = {k[:-3]: round(1000 * v / nb, 1) for k, v in res.items() if k.endswith("_ms")}
    print(json.dumps(res))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--blocks", type=int, default=8)
    ap.add_argument("--batch", type=int, default=64)
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--decode-sms", type=int, nargs="*", default=[132, 116, 100],
                    help="also time the overlapped pass with the decoder capped at these SM counts")
    ap.add_argument("--no-dense", dest="dense", action="store_false",
                    help="skip the uncompressed-weights GEMM baseline (saves device memory)")
    ap.add_argument("--no-check", dest="check", action="store_false")
    ap.add_argument("--gemv", action="store_true",
                    help="batch-1 comparison: decompress + cuBLAS matrix-vector products vs df11_decompress_gemv")
    ap.add_argument("--inner", type=int, default=4,
                    help="calls timed back to back per sample (their mean is the sample)")
    ap.add_argument("--gemm", action="store_true",
                    help="batch-B comparison: decompress + cuBLAS GEMMs vs df11_decompress_gemm")
    args = ap.parse_args(argv)
    if args.gemm:
        _bench_gemm(args)
        return
    if args.gemv:
        _bench_gemv(args)
        return
    if args.check and not args.dense:
        ap.error("--check needs the dense baseline")
    _bench(args)


if __name__ == "__main__":
    main()
