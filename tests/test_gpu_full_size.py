"""Byte parity at the workloads' full sizes, in the benchmark's launch layout.

Each workload is generated at full size, compressed on the GPU (one batched
call per workload, as bench.py does for the block) and compared with the CPU
oracle byte for byte: code lengths, codes, chunk offsets, the whole exponent
stream and the packed sign/mantissa array.  The GPU decompression (batched
for the block, per tensor elsewhere, per 64-token page range for the K/V
cache) must reproduce the input bits exactly.  The oracle is fast enough to
run on every value, so nothing is sampled.
"""
import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


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


def _same(c, ref):
    assert c.exp_stream_bits == ref.bits
    assert np.array_equal(c.code_len.cpu().numpy(), ref.code_len)
    assert np.array_equal(c.code.cpu().numpy().view(np.uint32), ref.code)
    assert np.array_equal(c.chunk_bit_off.cpu().numpy().view(np.uint64), ref.chunk_bit_off)
    nb = (ref.bits + 7) // 8
    assert np.array_equal(c.exp_stream[:nb].cpu().numpy(), ref.stream)
    assert np.array_equal(c.sign_mant.cpu().numpy(), ref.sign_mant)


def _run(eh, oracle, name, page_ranges=False):
    dt, items = synth.workload(name)
    dtype = {"bf16": 0, "fp8_e4m3": 1, "bytes": 2}[dt]
    p = eh.plan(dtype)
    xs = [_dev(x) for _, x in items]
    outs = [eh.alloc_compressed(p, x.numel(), "cuda") for x in xs]
    ws = torch.empty(eh.compress_batch_workspace(p, [x.numel() for x in xs]), dtype=torch.uint8,
                     device="cuda")
    eh.compress_batch(p, xs, outs, ws)
    del ws
    for (_, x), c in zip(items, outs):
        _same(c, oracle.compress(dtype, x))
    ys = [torch.empty_like(x) for x in xs]
    wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device="cuda")
    eh.decompress_batch(p, outs, ys, wsd)
    assert eh.get_status(wsd) == eh.EH_OK
    for x, y in zip(xs, ys):
        assert torch.equal(x, y)
    if page_ranges:
        # 64-token pages: one chunk each; decode scattered page ranges
        for c, x in zip(outs, xs):
            C = c.n_chunks
            for first, count in [(0, 1), (C // 2, 3), (C - 2, 2)]:
                y = eh.decompress_chunks(c, first, count, p)
                assert torch.equal(y, x[first * 65536:(first + count) * 65536])
    return outs


def test_bf16_1m(eh, oracle):
    (c,) = _run(eh, oracle, "bf16_1m")
    assert c.n_chunks == 16


def test_fp8_16m(eh, oracle):
    (c,) = _run(eh, oracle, "fp8_16m")
    assert c.n_chunks == 256


def test_llama8b_block(eh, oracle):
    outs = _run(eh, oracle, "llama8b_block")
    assert sum(c.n_chunks for c in outs) == 3328


def test_kv_layer(eh, oracle):
    outs = _run(eh, oracle, "kv_layer", page_ranges=True)
    assert [c.n_chunks for c in outs] == [1024, 1024]


def test_lm_head(eh, oracle):
    (c,) = _run(eh, oracle, "lm_head")
    assert c.n_chunks == 8016


@pytest.mark.parametrize("name", list(synth.SCALE_WORKLOADS))
def test_fp4_block_scales(eh, oracle, name):
    outs = _run(eh, oracle, name)
    assert len(outs) == 7


def test_zipfloat_comparison_codec_on_the_block(eh, oracle):
    """The ZipFloat comparison codec over the whole block, byte parity per
    block against the oracle (record ranges compared through their offsets)."""
    from test_gpu_zipfloat import check_parity
    for _, x in synth.llama8b_block():
        check_parity(eh, oracle, x)
