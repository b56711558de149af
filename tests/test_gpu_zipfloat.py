"""GPU parity of the ZipFloat comparison codec against its CPU oracle.

Equal byte for byte: the sign/mantissa bytes, every block's metadata (l_b and
record count) and bit planes.  The records of each block are compared through
that block's offset, since the GPU reserves the blocks' ranges with an atomic
(ZipFloat §3.3) and only their order depends on scheduling: the ranges must be
disjoint and cover exactly the records written.  Decompression must give the
input back, and the oracle must decompress the GPU's arrays too.
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
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda()


def _host(c):
    from oracle import ehref
    B = c.blocks
    return ehref.ZfCompressed(
        c.n, c.sign_mant[:c.n].cpu().numpy(), c.meta[:B].cpu().numpy().view(np.uint32),
        c.dense[:B * 192].cpu().numpy().view(np.uint32), c.sparse_off[:B].cpu().numpy().view(np.uint32),
        c.sparse[:c.n_records].cpu().numpy().view(np.uint16))


def check_parity(eh, oracle, x):
    c = eh.zf_compress(_dev(x))
    ref = oracle.zf_compress(x)
    got = _host(c)
    assert c.n_records == ref.sparse.size
    assert np.array_equal(got.sign_mant, ref.sign_mant)
    assert np.array_equal(got.meta, ref.meta)
    assert np.array_equal(got.dense, ref.dense)
    nnz = got.meta >> 8
    has = np.nonzero(nnz)[0]
    order = has[np.argsort(got.sparse_off[has])]
    starts, lens = got.sparse_off[order].astype(np.int64), nnz[order].astype(np.int64)
    if starts.size:
        assert starts[0] == 0
        assert np.array_equal(starts[1:], (starts + lens)[:-1])      # disjoint, no gaps
        assert (starts + lens)[-1] == c.n_records
    else:
        assert c.n_records == 0
    for b in np.nonzero(nnz)[0]:
        g = got.sparse[got.sparse_off[b]: got.sparse_off[b] + nnz[b]]
        r = ref.sparse[ref.sparse_off[b]: ref.sparse_off[b] + nnz[b]]
        assert np.array_equal(g, r), b
    y = eh.zf_decompress(c)
    assert np.array_equal(y.cpu().numpy().view(np.uint16), x)
    assert np.array_equal(oracle.zf_decompress(got), x)
    return c


@pytest.mark.parametrize("n,seed", [(2048, 0), (5000, 1), (3 * 2048 + 1, 2), (7, 3), (1 << 20, 4)])
def test_student_t_parity(eh, oracle, n, seed):
    x = synth.student_t_bf16((n,), np.random.default_rng(seed))
    check_parity(eh, oracle, x)


def test_normal_and_every_pattern(eh, oracle):
    check_parity(eh, oracle, synth.normal_bf16(1 << 20, seed=9))
    x = np.random.default_rng(7).permutation(np.arange(65536, dtype=np.uint32)).astype(np.uint16)
    c = check_parity(eh, oracle, x)
    assert c.n_records > 0


def test_uniform_blocks_have_no_records(eh, oracle):
    x = np.full(4 * 2048 + 100, 0x3F80, np.uint16)   # 1.0 everywhere
    c = check_parity(eh, oracle, x)
    assert c.n_records == 0


def test_overflow_and_corruption(eh, oracle):
    x = synth.student_t_bf16((6 * 2048,), np.random.default_rng(5))
    c = eh.ZfCompressed(x.size, "cuda")
    c.sparse = c.sparse[:10]                          # room for 10 records only
    with pytest.raises(eh.EhError) as e:
        eh.zf_compress(_dev(x), out=c)
    assert e.value.code == eh.EH_ERR_NOMEM
    c = eh.zf_compress(_dev(x))
    good = c.meta.clone()
    c.meta[2] = good[2] + (5000 << 8)                 # more records than values
    y = eh.zf_decompress(c, check=False)
    assert eh.get_status(c.workspace) == eh.EH_ERR_CORRUPT
    c.meta.copy_(good)
    y = eh.zf_decompress(c)
    assert np.array_equal(y.cpu().numpy().view(np.uint16), x)
