"""Guard bytes around every caller buffer stay untouched.

compute-sanitizer is not available here, so out-of-bounds writes are caught
this way: every buffer a call receives (inputs, compressed arrays, value
index, outputs, workspaces, page-store slots, sign/mantissa and raw pool) is
a view into a larger allocation whose 256 bytes before and after it are
filled with a canary byte.  After the calls the canaries must be intact, and
the results must still be exact.  Small cases with odd lengths, FP8 nibble
packing, chunk ranges, batches and pages.
"""
import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 256
CANARY = 0xA5


@pytest.fixture(scope="module")
def eh():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exponent_entropy_coding_b200 import build, exphuff
    build.build()
    exphuff.lib()
    return exphuff


class Arena:
    """Allocations with canary-filled guard regions on both sides."""

    def __init__(self):
        self.bufs = []

    def tensor(self, numel, dtype, fill=None):
        size = torch.empty(0, dtype=dtype).element_size()
        nbytes = numel * size
        raw = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.bufs.append((raw, nbytes))
        t = raw[GUARD:GUARD + nbytes].view(dtype)
        if fill is not None:
            t.fill_(fill)
        return t

    def copy_of(self, x):
        t = self.tensor(x.numel(), x.dtype)
        t.copy_(x)
        return t

    def check(self):
        torch.cuda.synchronize()
        for i, (raw, nbytes) in enumerate(self.bufs):
            h = raw.cpu().numpy()
            assert (h[:GUARD] == CANARY).all(), f"buffer {i}: bytes before it were written"
            assert (h[GUARD + nbytes:] == CANARY).all(), f"buffer {i}: bytes after it were written"


def compressed(eh, arena, p, n, index=False):
    cap, smb, _ = eh.compress_bound(p, n)
    A = eh.alphabet(p.dtype)
    nc = -(-n // p.chunk_elems)
    return eh.Compressed(
        dtype=p.dtype, n=n,
        code_len=arena.tensor(A, torch.uint8, 0), code=arena.tensor(A, torch.int32, 0),
        chunk_bit_off=arena.tensor(nc + 1, torch.int64, 0),
        exp_stream=arena.tensor(cap, torch.uint8), sign_mant=arena.tensor(smb, torch.uint8),
        value_index=arena.tensor(nc * (p.chunk_elems // eh.EH_INDEX_STRIDE), torch.int32, 0) if index else None)


def _dev(x):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return (t.view(torch.int16) if t.dtype == torch.uint16 else t).cuda()


@pytest.mark.parametrize("dtype,n,chunk,index", [(0, 3 * 65536 + 123, 65536, False), (1, 2 * 65536 + 7, 65536, False),
                                                 (0, 5 * 1024 + 3, 1024, True), (1, 9 * 1024 + 1, 1024, False),
                                                 (2, 70001, 65536, False)])
def test_canaries_around_codec_buffers(eh, oracle, dtype, n, chunk, index):
    if dtype == 0:
        xs = [synth.normal_bf16(n, seed=1), synth.normal_bf16(n // 3 + 5, seed=2)]
    elif dtype == 1:
        xs = [synth.normal_fp8(n, seed=1), synth.normal_fp8(n // 3 + 5, seed=2)]
    else:
        rng = np.random.default_rng(3)
        xs = [rng.integers(90, 140, n).astype(np.uint8), rng.integers(0, 256, n // 3 + 5).astype(np.uint8)]
    arena = Arena()
    p = eh.plan(dtype, chunk)
    ins = [arena.copy_of(_dev(x)) for x in xs]
    cs = [compressed(eh, arena, p, x.size, index) for x in xs]
    wsc = arena.tensor(eh.compress_batch_workspace(p, [x.size for x in xs]), torch.uint8)
    eh.compress_batch(p, ins, cs, wsc)
    for x, c in zip(xs, cs):
        ref = oracle.compress(dtype, x, chunk=chunk)
        assert c.exp_stream_bits == ref.bits
        nb = (ref.bits + 7) // 8
        assert np.array_equal(c.exp_stream[:nb].cpu().numpy(), ref.stream)
    wsd = arena.tensor(eh.decompress_workspace(p, 2), torch.uint8)
    outs = [arena.tensor(x.size, t.dtype) for x, t in zip(xs, ins)]
    eh.decompress_batch(p, cs, outs, wsd)
    assert eh.get_status(wsd) == eh.EH_OK
    for o, t in zip(outs, ins):
        assert torch.equal(o, t)
    for o, c, t in zip(outs, cs, ins):
        y = arena.tensor(c.n, t.dtype)
        eh.decompress(c, p, out=y, workspace=wsd)
        assert torch.equal(y, t)
    C = cs[0].n_chunks
    first, count = 1, C - 2
    lo, hi = first * chunk, min(n, (first + count) * chunk)
    y = arena.tensor(hi - lo, ins[0].dtype)
    eh.decompress_chunks(cs[0], first, count, p, out=y, workspace=wsd)
    assert torch.equal(y, ins[0][lo:hi])
    arena.check()


def test_canaries_around_page_store(eh, oracle):
    _, items = synth.workload("kv_layer", scale=64)      # 128 tokens: 16 pages per tensor
    k = items[0][1]
    page = 65536
    prefill, new = k[:4 * page], k[4 * page:12 * page]
    p = eh.plan(0)
    cnt = oracle.histogram(0, prefill) + np.uint64(1)
    arena = Arena()
    counts = arena.copy_of(torch.from_numpy(cnt.view(np.int64)).cuda())
    code_len, code = arena.tensor(256, torch.uint8, 0), arena.tensor(256, torch.int32, 0)
    wsb = arena.tensor(eh.compress_bound(p, 0)[2], torch.uint8)
    eh.codebook_from_counts(p, counts, code_len=code_len, code=code, workspace=wsb)
    n_slots, slot_bytes, raw_cap = 10, 24 * 1024, 3
    store = eh.PageStore(p, code_len, code, n_slots, slot_bytes, raw_cap, "cuda")
    store.slots = arena.tensor(n_slots * slot_bytes, torch.uint8, 0)
    store.sign_mant = arena.tensor(n_slots * page, torch.uint8)
    store.page_meta = arena.tensor(n_slots, torch.int32, 0)
    store.raw_pool = arena.tensor(raw_cap * page, torch.uint8)
    store.raw_used = arena.tensor(1, torch.int32, 0)
    store.workspace = arena.tensor(max(256, eh.decompress_workspace(p, 1)), torch.uint8)
    ids = arena.copy_of(torch.tensor([7, 2, 9, 0, 4, 1, 8, 3], dtype=torch.int32, device="cuda"))
    x = arena.copy_of(_dev(new))
    store.append(x, ids)
    assert store.status() == eh.EH_OK
    y = arena.tensor(x.numel(), x.dtype)
    store.read(ids, out=y)
    assert torch.equal(y, x)
    arena.check()
