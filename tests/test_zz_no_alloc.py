"""The no-allocation block decompression entry point.

Callers that cannot allocate device memory (graph capture, statically planned
runtimes, allocator callbacks) use eh_decompress_batch_noalloc, whose scratch
is a fixed array inside the library.  Its output must equal the output of the
workspace-based eh_decompress_batch exactly (the codec is lossless, so the
tolerance is zero), on two calls in a row that reuse the shared array.
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


def _dev(x):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return (t.view(torch.int16) if t.dtype == torch.uint16 else t).cuda()


def _compress_all(eh, p, xs):
    outs = [eh.alloc_compressed(p, x.numel(), "cuda") for x in xs]
    ws = torch.empty(eh.compress_batch_workspace(p, [x.numel() for x in xs]), dtype=torch.uint8,
                     device="cuda")
    eh.compress_batch(p, xs, outs, ws)
    return outs


@pytest.mark.parametrize("dtype", [0, 1])
def test_noalloc_matches_workspace_decode(eh, dtype):
    if dtype == 0:
        _, items = synth.workload("llama8b_block", scale=64)   # 7 matrices
        xs = [_dev(x) for _, x in items[:eh.EH_NOALLOC_MAX_BATCH]]
    else:
        xs = [_dev(synth.normal_fp8(n, seed=n)) for n in (3 * 65536 + 5, 65536, 17)]
    p = eh.plan(dtype)
    cs = _compress_all(eh, p, xs)
    ref = [torch.empty_like(x) for x in xs]
    ws = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device="cuda")
    eh.decompress_batch(p, cs, ref, ws)
    assert eh.get_status(ws) == eh.EH_OK
    for call in range(2):
        ys = [torch.full_like(x, 0x5A5A if dtype == 0 else 0x5A) for x in xs]
        assert eh.decompress_batch_noalloc(p, cs, ys) == eh.EH_OK, f"call {call}"
        for r, y, x in zip(ref, ys, xs):
            assert torch.equal(y, r)
            assert torch.equal(y, x)


def test_noalloc_rejects_too_many_tensors(eh):
    p = eh.plan(0)
    xs = [_dev(synth.normal_bf16(1000 + i, seed=i)) for i in range(eh.EH_NOALLOC_MAX_BATCH + 1)]
    cs = _compress_all(eh, p, xs)
    ys = [torch.empty_like(x) for x in xs]
    assert eh.decompress_batch_noalloc(p, cs, ys) == eh.EH_ERR_INVALID_ARG


def test_noalloc_reports_corruption_then_recovers(eh):
    p = eh.plan(0)
    x = _dev(synth.normal_bf16(2 * 65536 + 3, seed=21))
    (c,) = _compress_all(eh, p, [x])
    good = c.chunk_bit_off.clone()
    c.chunk_bit_off[1] += 1
    y = torch.empty_like(x)
    assert eh.decompress_batch_noalloc(p, [c], [y]) == eh.EH_ERR_CORRUPT
    c.chunk_bit_off.copy_(good)
    assert eh.decompress_batch_noalloc(p, [c], [y]) == eh.EH_OK
    assert torch.equal(y, x)
