"""Pins of the oracle's optional value index (CPU only).

Entry k of chunk c is the bit offset, from the chunk's first bit, of value
128k's code; entries past a short chunk's end hold the chunk's bit count.
Pinned two independent ways: the running sum of the code lengths (the
definition), and the stream itself: the bits found at each recorded offset
must be exactly the canonical code of that value's exponent.
"""
import numpy as np
import pytest

from exponent_entropy_coding_b200 import synth

STRIDE = 128


def _exponents(dtype, x):
    return ((x >> 7) & 0xFF) if dtype == 0 else ((x >> 3) & 0xF)


def _bits_at(stream, pos, n):
    v = 0
    for p in range(pos, pos + n):
        v = (v << 1) | ((int(stream[p >> 3]) >> (7 - (p & 7))) & 1)
    return v


@pytest.mark.parametrize("dtype,n,chunk,seed", [(0, 3 * 65536 + 3392, 65536, 1), (0, 5000, 1024, 2),
                                                (1, 70000, 4096, 3), (0, 65536, 65536, 4)])
def test_index_by_definition_and_by_the_stream(oracle, dtype, n, chunk, seed):
    x = synth.normal_bf16(n, seed) if dtype == 0 else synth.normal_fp8(n, seed)
    c = oracle.compress(dtype, x, chunk=chunk)
    idx = oracle.value_index(dtype, x, c.code_len, chunk=chunk)
    per = chunk // STRIDE
    e = _exponents(dtype, x.astype(np.int64))
    lens = c.code_len[e].astype(np.int64)
    C = (n + chunk - 1) // chunk
    assert idx.size == C * per
    for ci in range(C):
        lc = lens[ci * chunk: (ci + 1) * chunk]
        cum = np.concatenate([[0], np.cumsum(lc)])
        total = int(cum[-1])
        assert total == int(c.chunk_bit_off[ci + 1] - c.chunk_bit_off[ci])
        for k in range(per):
            j = k * STRIDE
            want = int(cum[j]) if j < lc.size else total
            assert int(idx[ci * per + k]) == want
            if j < lc.size:
                # the code found at that bit is the one of value j's exponent
                i = ci * chunk + j
                L = int(c.code_len[e[i]])
                pos = int(c.chunk_bit_off[ci]) + want
                assert _bits_at(c.stream, pos, L) == int(c.code[e[i]])


def test_index_of_an_empty_tensor(oracle):
    x = np.zeros(0, np.uint16)
    c = oracle.compress(0, x)
    assert oracle.value_index(0, x, c.code_len).size == 0
