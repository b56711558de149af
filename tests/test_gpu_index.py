"""The optional value index on the GPU: parity with the oracle and use.

Compressing with an index writes, beside the unchanged stream, the bit offset
of every 128th value of each chunk; it must equal the oracle's value_index
entry for entry.  Decompressing with it (whole tensors, batches, chunk
ranges) must give the input back; an entry that does not match the stream
must be reported as corrupt.
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


def _host(y, dtype):
    a = y.cpu().numpy()
    return a.view(np.uint16) if dtype == 0 else a


def _compress_indexed(eh, p, x):
    c = eh.alloc_compressed(p, x.size, "cuda", index=True)
    ws = torch.empty(eh.compress_batch_workspace(p, [x.size]), dtype=torch.uint8, device="cuda")
    eh.compress_batch(p, [_dev(x)], [c], ws)
    return c


CASES = [(0, 65536, 3 * 65536 + 3392, 1), (0, 65536, 1 << 20, 2), (0, 4096, 70000, 3), (1, 65536, 200001, 4),
         (2, 65536, 150000, 5), (0, 65536, 100, 6),
         # enough chunks for the encoder's 256-thread CTAs (a full wave of them)
         (0, 1024, 650 * 1024 + 77, 7), (1, 1024, 700 * 1024 + 5, 8)]


@pytest.mark.parametrize("dtype,chunk,n,seed", CASES)
def test_index_parity_and_decode(eh, oracle, dtype, chunk, n, seed):
    if dtype == 0:
        x = synth.normal_bf16(n, seed)
    elif dtype == 1:
        x = synth.normal_fp8(n, seed)
    else:
        x = np.random.default_rng(seed).integers(100, 140, n).astype(np.uint8)
    p = eh.plan(dtype, chunk)
    c = _compress_indexed(eh, p, x)
    ref = oracle.compress(dtype, x, chunk=chunk)
    ridx = oracle.value_index(dtype, x, ref.code_len, chunk=chunk)
    assert c.exp_stream_bits == ref.bits
    assert np.array_equal(c.exp_stream[:(ref.bits + 7) // 8].cpu().numpy(), ref.stream)
    assert np.array_equal(c.value_index[:ridx.size].cpu().numpy().view(np.uint32), ridx)
    y = eh.decompress(c, p)
    assert np.array_equal(_host(y, dtype), x)
    C = c.n_chunks
    if C >= 3:
        yy = eh.decompress_chunks(c, 1, C - 2, p)
        assert np.array_equal(_host(yy, dtype), x[chunk:(C - 1) * chunk])


def test_block_batch_with_index(eh, oracle):
    items = [x for _, x in synth.llama8b_block(seed=7, scale=16)]
    p = eh.plan(0)
    xs = [_dev(x) for x in items]
    outs = [eh.alloc_compressed(p, x.size, "cuda", index=True) for x in items]
    ws = torch.empty(eh.compress_batch_workspace(p, [x.size for x in items]), dtype=torch.uint8, device="cuda")
    eh.compress_batch(p, xs, outs, ws)
    ys = [torch.empty_like(x) for x in xs]
    wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device="cuda")
    eh.decompress_batch(p, outs, ys, wsd)
    assert eh.get_status(wsd) == eh.EH_OK
    for x, c, y in zip(items, outs, ys):
        ref = oracle.compress(0, x)
        ridx = oracle.value_index(0, x, ref.code_len)
        assert np.array_equal(c.value_index.cpu().numpy().view(np.uint32), ridx)
        assert np.array_equal(_host(y, 0), x)


def test_mismatched_index_is_corrupt(eh):
    x = synth.normal_bf16(4 * 65536, seed=8)
    p = eh.plan(0)
    c = _compress_indexed(eh, p, x)
    ws = torch.empty(eh.decompress_workspace(p), dtype=torch.uint8, device="cuda")
    good = c.value_index.clone()
    for k, delta in [(700, 3), (512 + 5, -1), (1023, 50)]:
        c.value_index.copy_(good)
        c.value_index[k] += delta
        eh.decompress(c, p, workspace=ws, check=False)
        assert eh.get_status(ws) == eh.EH_ERR_CORRUPT
    c.value_index.copy_(good)
    y = eh.decompress(c, p, workspace=ws)
    assert np.array_equal(_host(y, 0), x)
    # without the index the same arrays decode through the boundary search
    c.value_index = None
    y = eh.decompress(c, p, workspace=ws)
    assert np.array_equal(_host(y, 0), x)
