"""Compress and decompress captured in a CUDA graph and replayed.

The calls used with device-side bit counts enqueue kernels, memsets and
programmatic dependent launches only (no host wait, no allocation), so a
whole compress + decompress round trip can be captured once and replayed on
new input data written into the same buffers.  Every replay must give the
oracle's streams and the input bits back.
"""
import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def eh():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exponent_entropy_coding_b200 import build, exphuff
    build.build()
    exphuff.lib()
    return exphuff


def _block(seed):
    return [x for _, x in synth.llama8b_block(seed=seed, scale=64, count=4)]


def test_round_trip_replays(eh, oracle):
    p = eh.plan(0)
    first = _block(60)
    xs = [torch.from_numpy(x.view(np.int16)).cuda() for x in first]
    outs = [eh.alloc_compressed(p, x.numel(), "cuda") for x in xs]
    ys = [torch.empty_like(x) for x in xs]
    wsc = torch.empty(eh.compress_batch_workspace(p, [x.numel() for x in xs]), dtype=torch.uint8, device="cuda")
    wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device="cuda")
    bits = torch.zeros(len(xs), dtype=torch.int64, device="cuda")
    # first calls outside the capture (one-time device setup)
    eh.compress_batch(p, xs, outs, wsc, bits_dev=bits)
    eh.decompress_batch(p, outs, ys, wsd)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            eh.compress_batch(p, xs, outs, wsc, bits_dev=bits)
            eh.decompress_batch(p, outs, ys, wsd)
    torch.cuda.current_stream().wait_stream(s)

    for seed in (61, 62):
        data = _block(seed)
        for x, d in zip(xs, data):
            x.copy_(torch.from_numpy(d.view(np.int16)))
        for y in ys:
            y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert eh.get_status(wsd) == eh.EH_OK
        nb = bits.cpu().numpy()
        for d, c, y, b in zip(data, outs, ys, nb):
            ref = oracle.compress(0, d)
            assert int(b) == ref.bits
            assert np.array_equal(c.chunk_bit_off.cpu().numpy().view(np.uint64), ref.chunk_bit_off)
            assert np.array_equal(c.exp_stream[:(ref.bits + 7) // 8].cpu().numpy(), ref.stream)
            assert np.array_equal(y.cpu().numpy().view(np.uint16), d)
