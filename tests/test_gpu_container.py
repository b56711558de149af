"""The stored form of a tensor compressed on the GPU.

A container written from the GPU's compressed arrays must equal, byte for
byte, the oracle's container of the same input (the two are independent
writers of one layout); read back onto the device it must decompress to the
input, and a container with one changed byte must be refused before any
decode runs.
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


def _input(dtype, n, seed):
    if dtype == 0:
        return synth.normal_bf16(n, seed)
    if dtype == 1:
        return synth.normal_fp8(n, seed)
    return np.random.default_rng(seed).integers(90, 150, n).astype(np.uint8)


CASES = [(0, 65536, 3 * 65536 + 4321, False), (0, 65536, 2 * 65536 + 9, True), (1, 65536, 200001, True),
         (2, 4096, 50001, False), (0, 1024, 70 * 1024 + 3, True), (1, 65536, 7, False)]


@pytest.mark.parametrize("dtype,chunk,n,with_index", CASES)
def test_gpu_container_matches_oracle_and_decodes(eh, oracle, dtype, chunk, n, with_index):
    x = _input(dtype, n, seed=n % 97)
    p = eh.plan(dtype, chunk)
    if with_index:
        c = eh.alloc_compressed(p, n, "cuda", index=True)
        ws = torch.empty(eh.compress_batch_workspace(p, [n]), dtype=torch.uint8, device="cuda")
        eh.compress_batch(p, [_dev(x)], [c], ws)
    else:
        c = eh.compress(_dev(x), p)
    torch.cuda.synchronize()
    ref = oracle.compress(dtype, x, chunk=chunk)
    idx = oracle.value_index(dtype, x, ref.code_len, chunk=chunk) if with_index else None
    buf = eh.to_container(c, p)
    assert buf == oracle.container(ref, idx)

    c2, p2 = eh.from_container(buf, "cuda")
    assert (p2.dtype, p2.chunk_elems, p2.max_code_len) == (p.dtype, p.chunk_elems, p.max_code_len)
    y = eh.decompress(c2, p2)
    assert np.array_equal(_host(y, dtype), x)
    if with_index:  # the decode above went through the index read back
        assert np.array_equal(c2.value_index.cpu().numpy().view(np.uint32), idx)


def test_changed_byte_is_refused_before_decoding(eh):
    x = synth.normal_bf16(65536 + 100, 3)
    p = eh.plan(0, 65536)
    buf = bytearray(eh.to_container(eh.compress(_dev(x), p), p))
    for pos in (5, 60, 200, len(buf) // 2, len(buf) - 1):
        bad = bytearray(buf)
        bad[pos] ^= 1
        with pytest.raises(eh.EhError):
            eh.from_container(bytes(bad), "cuda")
