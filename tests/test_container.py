"""The library's stored form of a compressed tensor, on the host (no GPU).

eh_container_write on the oracle's compressed arrays must produce the
oracle's container byte for byte; eh_container_read must return the same
arrays; any flipped byte of the header or of a section, a truncation or a
wrong version must be reported as EH_ERR_CORRUPT.
"""
import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import exphuff as eh
from exponent_entropy_coding_b200 import synth

CASES = [(0, 3 * 65536 + 123, 65536, False), (1, 70001, 1024, True), (2, 4097, 1024, False),
         (0, 0, 65536, False), (1, 65536, 65536, False), (0, 5000, 4096, True)]


def _input(dtype, n):
    if dtype == 0:
        return synth.normal_bf16(n, seed=4)
    if dtype == 1:
        return synth.normal_fp8(n, seed=4)
    return np.random.default_rng(4).integers(0, 256, n).astype(np.uint8)


def _host_compressed(oracle, dtype, n, chunk, with_index):
    """The oracle's arrays as a binding Compressed of CPU tensors."""
    x = _input(dtype, n)
    r = oracle.compress(dtype, x, chunk=chunk)
    p = eh.plan(dtype, chunk)
    cap = eh.compress_bound(p, n)[0]
    stream = np.zeros(cap if n else 0, np.uint8)
    stream[:r.stream.size] = r.stream
    idx = oracle.value_index(dtype, x, r.code_len, chunk=chunk) if with_index else None
    c = eh.Compressed(dtype=dtype, n=n, code_len=torch.from_numpy(r.code_len.copy()),
                      code=torch.from_numpy(r.code.view(np.int32).copy()),
                      chunk_bit_off=torch.from_numpy(r.chunk_bit_off.view(np.int64).copy()),
                      exp_stream=torch.from_numpy(stream), sign_mant=torch.from_numpy(r.sign_mant.copy()),
                      exp_stream_bits=r.bits,
                      value_index=torch.from_numpy(idx.view(np.int32).copy()) if with_index else None)
    return x, r, idx, c, p


@pytest.mark.parametrize("dtype,n,chunk,with_index", CASES)
def test_container_equals_the_oracles(oracle, dtype, n, chunk, with_index):
    x, r, idx, c, p = _host_compressed(oracle, dtype, n, chunk, with_index)
    buf = eh.to_container(c, p)
    assert buf == oracle.container(r, idx)
    assert len(buf) == eh.container_size(p, n, r.bits, with_index)


@pytest.mark.parametrize("dtype,n,chunk,with_index", CASES)
def test_container_round_trip(oracle, dtype, n, chunk, with_index):
    x, r, idx, c, p = _host_compressed(oracle, dtype, n, chunk, with_index)
    c2, p2 = eh.from_container(eh.to_container(c, p), "cpu")
    assert (p2.dtype, p2.chunk_elems, p2.max_code_len) == (p.dtype, p.chunk_elems, p.max_code_len)
    assert c2.n == n and c2.exp_stream_bits == r.bits and c2.n_chunks == c.n_chunks
    for name in ("code_len", "code", "chunk_bit_off", "sign_mant"):
        assert torch.equal(getattr(c2, name), getattr(c, name)), name
    nb = (r.bits + 7) // 8
    assert torch.equal(c2.exp_stream[:nb], c.exp_stream[:nb])
    if with_index:
        assert torch.equal(c2.value_index, c.value_index)
    # the oracle decodes what was read back
    back = oracle.Compressed(dtype, n, chunk, 32, c2.code_len.numpy(), c2.code.numpy().view(np.uint32),
                             c2.chunk_bit_off.numpy().view(np.uint64), c2.exp_stream[:nb].numpy(),
                             c2.sign_mant.numpy(), c2.exp_stream_bits)
    assert np.array_equal(oracle.decompress(back), x)


def test_container_detects_corruption(oracle):
    x, r, idx, c, p = _host_compressed(oracle, 0, 2 * 65536 + 77, 65536, True)
    buf = bytearray(eh.to_container(c, p))
    rng = np.random.default_rng(6)
    # every header byte, and bytes of every section
    positions = list(range(0, 192)) + [int(i) for i in rng.integers(192, len(buf), 200)]
    for pos in positions:
        bad = bytearray(buf)
        bad[pos] ^= 0x10
        if bad == buf:
            continue
        with pytest.raises(eh.EhError) as ei:
            eh.from_container(bytes(bad), "cpu")
        assert ei.value.code == eh.EH_ERR_CORRUPT, pos
    for cut in (0, 100, 191, len(buf) - 16, len(buf) - 1):
        with pytest.raises(eh.EhError) as ei:
            eh.from_container(bytes(buf[:cut]), "cpu")
        assert ei.value.code == eh.EH_ERR_CORRUPT, cut
    eh.from_container(bytes(buf), "cpu")  # the intact one reads


def test_container_write_needs_room(oracle):
    x, r, idx, c, p = _host_compressed(oracle, 1, 3000, 1024, False)
    size = eh.container_size(p, 3000, r.bits)
    assert size % 16 == 0
    import ctypes as C
    out = np.zeros(size - 16, np.uint8)
    host = {k: getattr(c, k).numpy() for k in ("code_len", "code", "chunk_bit_off", "exp_stream", "sign_mant")}
    s = eh.eh_compressed_t()
    s.dtype, s.n, s.n_chunks, s.exp_stream_bits = c.dtype, c.n, c.n_chunks, c.exp_stream_bits
    s.code_len, s.code = host["code_len"].ctypes.data, host["code"].ctypes.data
    s.chunk_bit_off, s.exp_stream = host["chunk_bit_off"].ctypes.data, host["exp_stream"].ctypes.data
    s.exp_stream_cap, s.sign_mant = host["exp_stream"].size, host["sign_mant"].ctypes.data
    rc = eh.lib().eh_container_write(C.byref(p), C.byref(s), out.ctypes.data_as(C.c_void_p), out.size)
    assert rc == eh.EH_ERR_NOMEM


def test_container_inside_a_larger_buffer(oracle):
    # bytes after the container are ignored; a container cut short is refused
    x, r, idx, c, p = _host_compressed(oracle, 0, 70000, 65536, False)
    buf = eh.to_container(c, p)
    c2, _ = eh.from_container(buf + bytes(range(200)), "cpu")
    assert torch.equal(c2.sign_mant, c.sign_mant) and c2.exp_stream_bits == c.exp_stream_bits
    for cut in (0, 100, 191, 192, len(buf) - 16, len(buf) - 1):
        with pytest.raises(eh.EhError):
            eh.from_container(buf[:cut], "cpu")
