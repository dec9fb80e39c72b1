"""Per-block decompress-and-use pipeline ("Dekompresi per transformer block"):
block i+1 decompresses on a side stream while block i's GEMMs run.  The
pipeline's results must equal the same GEMMs on the original weights bit for
bit, with and without overlap, whatever the consumer's speed."""
import numpy as np
import pytest

import huffman_decode_03_b200 as df11
from huffman_decode_03_b200 import inputs
from huffman_decode_03_b200.pipeline import BlockPipeline, block_gemms

SHAPES = [(96, 160), (32, 160), (160, 96), (64, 64)]


def _block_bits(b):
    return [inputs.gaussian(r * c, [70, b, m]) for m, (r, c) in enumerate(SHAPES)]


def test_block_gemms_cpu():
    # the stand-in consumer on CPU tensors: each matrix of the flat block
    # times the activations, in stream order
    import torch

    mats = _block_bits(0)
    w = torch.from_numpy(np.concatenate(mats).view(np.int16)).view(torch.bfloat16).float()
    x = torch.randn(3, 160, generator=torch.Generator().manual_seed(1))
    ys = block_gemms(SHAPES, x)(w)
    off = 0
    for (r, c), y in zip(SHAPES, ys):
        ref = x[:, :c] @ w[off:off + r * c].view(r, c).t()
        assert torch.equal(y, ref)
        off += r * c


def _setup(nblocks):
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    blocks, dense = [], []
    for b in range(nblocks):
        mats = _block_bits(b)
        blocks.append(df11.DeviceFormat(df11.build_format(mats), "cuda"))
        dense.append(torch.from_numpy(np.concatenate(mats).view(np.int16)).cuda().view(torch.bfloat16))
    x = (torch.randn(8, 160, generator=torch.Generator().manual_seed(2)) * 0.5).to(torch.bfloat16).cuda()
    return torch, blocks, dense, x


@pytest.mark.gpu
@pytest.mark.parametrize("overlap,decode_sms", [(True, 0), (False, 0), (True, 40)])
@pytest.mark.parametrize("slow_consumer", [False, True])
def test_pipeline_matches_dense_gemms(overlap, decode_sms, slow_consumer):
    torch, blocks, dense, x = _setup(5)
    gemm = block_gemms(SHAPES, x)
    got = {}

    def consume(i, w):
        if slow_consumer:
            # keeps the consumer stream busy so that the decode stream runs
            # ahead and the buffer-reuse waits are exercised
            big = torch.randn(1024, 1024, device="cuda")
            for _ in range(20):
                big = big @ big * 1e-3
        got[i] = gemm(w)

    status = BlockPipeline(blocks, decode_sms=decode_sms).run(consume, overlap=overlap)
    torch.cuda.synchronize()
    assert status.cpu().tolist() == [0] * len(blocks)
    for i, w in enumerate(dense):
        for a, b in zip(got[i], gemm(w)):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.gpu
def test_pipeline_reports_the_corrupt_block():
    torch, blocks, dense, x = _setup(3)
    offs = blocks[1].tensors["block_offset"].view(torch.int32)
    offs[1] = offs[1] + 1  # block 1's first format block claims one output too many
    status = BlockPipeline(blocks).run(lambda i, w: None)
    torch.cuda.synchronize()
    st = status.cpu().tolist()
    assert st[0] == 0 and st[2] == 0 and st[1] != 0
