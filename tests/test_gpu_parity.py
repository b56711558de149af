"""GPU parity: every output of the CUDA path equals the CPU oracle, byte for byte.

Compared per tensor: code lengths, canonical codes, chunk bit offsets, the
meaningful bytes of the exponent stream, the packed sign/mantissa array and
the decompressed values (the DFloat11 article, "实验结果": decompressed weight
matrices are compared bit for bit with the originals).  All work is integer,
so the bar is exact equality.  Calls go through the C ABI (ctypes binding).
"""
import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import synth

pytestmark = pytest.mark.gpu

CHUNK = 65536


@pytest.fixture(scope="module")
def eh():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exponent_entropy_coding_b200 import build, exphuff
    build.build()
    exphuff.lib()
    return exphuff


def dev(x):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if t.dtype == torch.uint16:
        t = t.view(torch.int16)
    return t.cuda()


def host_bits(t, dtype):
    a = t.cpu().numpy()
    return a.view(np.uint16) if dtype == 0 else a


def assert_same(c, ref):
    assert c.exp_stream_bits == ref.bits
    assert np.array_equal(c.code_len.cpu().numpy(), ref.code_len)
    assert np.array_equal(c.code.cpu().numpy().view(np.uint32), ref.code)
    assert np.array_equal(c.chunk_bit_off.cpu().numpy().view(np.uint64), ref.chunk_bit_off)
    nb = (ref.bits + 7) // 8
    assert np.array_equal(c.exp_stream[:nb].cpu().numpy(), ref.stream)
    assert np.array_equal(c.sign_mant.cpu().numpy(), ref.sign_mant)


def roundtrip(eh, oracle, dtype, x, chunk=CHUNK, lmax=32):
    p = eh.plan(dtype, chunk, lmax)
    c = eh.compress(dev(x), p)
    ref = oracle.compress(dtype, x, chunk=chunk, lmax=lmax)
    assert_same(c, ref)
    y = eh.decompress(c, p)
    assert np.array_equal(host_bits(y, dtype), x)
    return c


@pytest.mark.parametrize("n", [1, 2, 1023, 65536, 3 * 65536 + 777, 5 * 65536])
def test_bf16_normal(eh, oracle, n):
    roundtrip(eh, oracle, 0, synth.normal_bf16(n, seed=n))


@pytest.mark.parametrize("n", [1, 7, 2 * 65536 + 1, 4 * 65536])
def test_fp8_normal(eh, oracle, n):
    roundtrip(eh, oracle, 1, synth.normal_fp8(n, seed=n))


@pytest.mark.parametrize("dtype,chunk,n", [(0, 1024, 10 * 1024 + 3), (1, 1024, 9 * 1024 + 1),
                                           (0, 4096, 50_000), (1, 8192, 65_537),
                                           # a full wave of the encoder's 256-thread CTAs
                                           (0, 1024, 600 * 1024 + 3), (1, 1024, 1200 * 1024 + 1)])
def test_small_chunks(eh, oracle, dtype, chunk, n):
    x = synth.normal_bf16(n, seed=3) if dtype == 0 else synth.normal_fp8(n, seed=3)
    roundtrip(eh, oracle, dtype, x, chunk=chunk)


@pytest.mark.parametrize("dtype", [0, 1])
def test_repeated_small_chunk_decodes_are_exact(eh, oracle, dtype):
    # 1024-value chunks are decoded in a few microseconds each, so the warps
    # of a group run far out of step; every warp must store only into its
    # own region of the exponent buffer, or a merge may read a word that
    # another warp is still rewriting.  Thirty decodes of the same tensor
    # must all be exact.
    n = 1200 * 1024 + 1
    x = synth.normal_bf16(n, seed=3) if dtype == 0 else synth.normal_fp8(n, seed=3)
    p = eh.plan(dtype, 1024)
    c = eh.compress(dev(x), p)
    assert_same(c, oracle.compress(dtype, x, chunk=1024))
    t = dev(x)
    ws = torch.empty(eh.decompress_workspace(p, 1), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t)
    for _ in range(30):
        eh.decompress(c, p, out=y, workspace=ws)
        assert torch.equal(y, t)


def test_every_bf16_pattern(eh, oracle):
    rng = np.random.default_rng(1)
    x = np.arange(1 << 16, dtype=np.uint16)[rng.permutation(1 << 16)]
    roundtrip(eh, oracle, 0, np.concatenate([x, x[::-1], x[:1000]]))


def test_every_fp8_pattern(eh, oracle):
    rng = np.random.default_rng(2)
    x = np.tile(np.arange(256, dtype=np.uint8), 700)[rng.permutation(256 * 700)]
    roundtrip(eh, oracle, 1, x)


def test_empty(eh, oracle):
    for dtype in (0, 1):
        x = np.zeros(0, np.uint16 if dtype == 0 else np.uint8)
        c = roundtrip(eh, oracle, dtype, x)
        assert c.exp_stream_bits == 0


def test_single_symbol(eh, oracle):
    roundtrip(eh, oracle, 0, np.full(70_001, 0x3F80, np.uint16))
    roundtrip(eh, oracle, 1, np.full(3 * 65536 + 5, 0x38, np.uint8))


def test_fixed_length_code(eh, oracle):
    # four equally frequent exponents: every code is 2 bits long, a code that
    # never resynchronises from a misaligned start
    rng = np.random.default_rng(4)
    e = rng.integers(0, 4, 5 * 65536 + 11).astype(np.uint16) + 120
    x = (e << 7) | rng.integers(0, 1 << 16, e.size).astype(np.uint16) & 0x807F
    c = roundtrip(eh, oracle, 0, x)
    assert set(c.code_len.cpu().numpy()[120:124]) == {2}


def test_slow_resync_code(eh, oracle):
    # lengths 1,3,3,3,3 - every length odd, resynchronisation is slow
    rng = np.random.default_rng(5)
    e = rng.choice(5, 4 * 65536, p=[0.5, 0.125, 0.125, 0.125, 0.125]).astype(np.uint16) + 100
    x = (e << 7) | (rng.integers(0, 256, e.size).astype(np.uint16) & 0x7F)
    roundtrip(eh, oracle, 0, x)


def test_long_codes(eh, oracle):
    # counts 2^s for 22 symbols: Huffman depths up to 21 bits (second-level
    # tables and the limit search of the decoder)
    rng = np.random.default_rng(6)
    e = np.repeat(np.arange(22, dtype=np.uint16) + 100, [1 << s for s in range(22)][::-1])
    e = e[rng.permutation(e.size)]
    x = (e << 7) | (rng.integers(0, 1 << 16, e.size).astype(np.uint16) & 0x807F)
    c = roundtrip(eh, oracle, 0, x)
    assert c.code_len.cpu().numpy().max() == 21


@pytest.mark.parametrize("lmax", [8, 12, 20])
def test_length_limited(eh, oracle, lmax):
    # Fibonacci counts over 26 symbols force the limit (package-merge path)
    fib = [1, 1]
    while len(fib) < 26:
        fib.append(fib[-1] + fib[-2])
    rng = np.random.default_rng(lmax)
    e = np.repeat(np.arange(26, dtype=np.uint16) + 90, fib)
    e = e[rng.permutation(e.size)]
    x = (e << 7) | (rng.integers(0, 1 << 16, e.size).astype(np.uint16) & 0x807F)
    c = roundtrip(eh, oracle, 0, x, lmax=lmax)
    assert c.code_len.cpu().numpy().max() == lmax


@pytest.mark.parametrize("m", [33, 34])
def test_codes_of_32_bits(eh, oracle, m):
    # Fibonacci counts over 33 symbols give Huffman codes of up to 32 bits
    # (the format's limit); over 34 symbols the Huffman depth is 33 and
    # package-merge limits it to 32.  A 32-bit code sits in a chunk the
    # decoder stages in shared memory (chunk 0) and in one it reads from
    # global memory (chunk 1, above 27 KB of stream).
    x = synth.fibonacci_bf16(m, seed=m)
    c = roundtrip(eh, oracle, 0, x)
    lens = c.code_len.cpu().numpy()
    e = (x >> 7) & 0xFF
    assert lens.max() == 32
    assert lens[e[:CHUNK]].max() == 32 and lens[e[CHUNK:2 * CHUNK]].max() == 32
    off = c.chunk_bit_off.cpu().numpy().view(np.uint64).astype(np.int64)
    # chunk 0 fits the 26.5 KB shared-memory stage, chunk 1 (about 100 KB) does not
    assert (off[1] - off[0]) // 8 < 26 * 1024 < 32 * 1024 < (off[2] - off[1]) // 8
    # chunk ranges that start on each of the two chunks decode too
    for first, count in ((0, 1), (1, 1), (1, 3)):
        y = eh.decompress_chunks(c, first, count, eh.plan(0))
        assert np.array_equal(host_bits(y, 0), x[first * CHUNK:(first + count) * CHUNK])


@pytest.mark.parametrize("m", [33, 34])
def test_byte_codes_of_32_bits(eh, oracle, m):
    # The byte alphabet (FP4 block scales) with the same Fibonacci counts:
    # 32-bit codes through the decoder's byte path, staged and unstaged.
    x = (synth.fibonacci_symbols(m, seed=m) + 40).astype(np.uint8)
    c = roundtrip(eh, oracle, 2, x)
    lens = c.code_len.cpu().numpy()
    assert lens.max() == 32
    assert lens[x[:CHUNK]].max() == 32 and lens[x[CHUNK:2 * CHUNK]].max() == 32


def test_length_limited_real_data(eh, oracle):
    roundtrip(eh, oracle, 0, synth.normal_bf16(3 * 65536, seed=8), lmax=7)
    roundtrip(eh, oracle, 1, synth.normal_fp8(3 * 65536, seed=8), lmax=4)


def test_infeasible_limit(eh, oracle):
    x = (np.arange(64 * 1024, dtype=np.uint16) % 40 + 80) << 7
    p = eh.plan(0, CHUNK, 5)     # 40 distinct exponents > 2^5
    with pytest.raises(eh.EhError) as ei:
        eh.compress(dev(x), p)
    assert ei.value.code == eh.EH_ERR_INFEASIBLE


def test_chunk_larger_than_stage(eh, oracle):
    # chunk 1 holds 200 rare exponents (about 10-bit codes): its stream is
    # about 80 KB, more than the shared-memory stage, so it is decoded from
    # global memory
    rng = np.random.default_rng(9)
    n = 10 * 65536
    e = np.full(n, 127, np.uint16)
    e[65536:2 * 65536] = rng.integers(20, 220, 65536)
    e[e == 127] = np.where(rng.random((e == 127).sum()) < 0.3, 126, 127)
    x = (e << 7) | (rng.integers(0, 1 << 16, n).astype(np.uint16) & 0x807F)
    c = roundtrip(eh, oracle, 0, x)
    off = c.chunk_bit_off.cpu().numpy()
    assert (off[2] - off[1]) // 8 > 32 * 1024


@pytest.mark.parametrize("dtype", [0, 1])
def test_runs_of_every_length_are_exact(eh, oracle, dtype):
    # A batch whose tensors split the decoding CTAs' chunk ranges into runs
    # of one to eight chunks (1024-value chunks): runs of one chunk leave a
    # group idle, runs of two start both groups at once, longer runs stagger
    # them, and a range may change tensors (and tables) in its middle.
    # Decoded many times, every decode must be exact.
    p = eh.plan(dtype, 1024)
    sizes = [148 * 3 * 1024 + 5, 7 * 1024, 149 * 1024 - 1, 1024, 3 * 148 * 1024 + 2 * 1024 + 17]
    xs = [synth.normal_bf16(n, seed=11 + i) if dtype == 0 else synth.normal_fp8(n, seed=11 + i)
          for i, n in enumerate(sizes)]
    ts = [dev(x) for x in xs]
    outs = [eh.alloc_compressed(p, t.numel(), "cuda") for t in ts]
    ws = torch.empty(eh.compress_batch_workspace(p, sizes), dtype=torch.uint8, device="cuda")
    eh.compress_batch(p, ts, outs, ws)
    for x, c in zip(xs, outs):
        assert_same(c, oracle.compress(dtype, x, chunk=1024))
    ys = [torch.empty_like(t) for t in ts]
    wsd = torch.empty(eh.decompress_workspace(p, len(ts)), dtype=torch.uint8, device="cuda")
    for _ in range(10):
        for y in ys:
            y.fill_(0x55)
        eh.decompress_batch(p, outs, ys, wsd)
        assert eh.get_status(wsd) == eh.EH_OK
        for t, y in zip(ts, ys):
            assert torch.equal(t, y)


def test_batch_block(eh, oracle):
    _, items = synth.workload("llama8b_block", scale=64)
    p = eh.plan(0)
    xs = [dev(x) for _, x in items]
    outs = [eh.alloc_compressed(p, x.numel(), "cuda") for x in xs]
    ws = torch.empty(eh.compress_batch_workspace(p, [x.numel() for x in xs]), dtype=torch.uint8,
                     device="cuda")
    eh.compress_batch(p, xs, outs, ws)
    for (_, x), c in zip(items, outs):
        assert_same(c, oracle.compress(0, x))
    ys = [torch.empty_like(x) for x in xs]
    wsd = torch.empty(eh.decompress_workspace(p, len(xs)), dtype=torch.uint8, device="cuda")
    eh.decompress_batch(p, outs, ys, wsd)
    assert eh.get_status(wsd) == eh.EH_OK
    for x, y in zip(xs, ys):
        assert torch.equal(x, y)
    # device-side bit counts (no host wait inside the call)
    bits = torch.zeros(len(xs), dtype=torch.int64, device="cuda")
    outs2 = [eh.alloc_compressed(p, x.numel(), "cuda") for x in xs]
    eh.compress_batch(p, xs, outs2, ws, bits_dev=bits)
    assert bits.cpu().tolist() == [c.exp_stream_bits for c in outs]


def test_kv_pages(eh, oracle):
    _, items = synth.workload("kv_layer", scale=64)   # 128 tokens: 2 pages per batch row
    p = eh.plan(0)
    for _, x in items:
        c = roundtrip(eh, oracle, 0, x)
        C = c.n_chunks
        for first, count in [(0, 1), (3, 2), (C - 1, 1), (1, C - 1)]:
            y = eh.decompress_chunks(c, first, count, p)
            ref = oracle.decompress(oracle.compress(0, x), first, count)
            assert np.array_equal(host_bits(y, 0), ref)
            assert np.array_equal(ref, x[first * CHUNK:(first + count) * CHUNK])


def test_corruption_is_reported(eh, oracle):
    x = synth.normal_bf16(4 * 65536, seed=10)
    p = eh.plan(0)
    c = eh.compress(dev(x), p)
    ws = torch.empty(eh.decompress_workspace(p), dtype=torch.uint8, device="cuda")
    good = c.chunk_bit_off.clone()
    c.chunk_bit_off[2] += 3                          # a chunk boundary moves
    eh.decompress(c, p, workspace=ws, check=False)
    assert eh.get_status(ws) == eh.EH_ERR_CORRUPT
    c.chunk_bit_off.copy_(good)
    eh.decompress(c, p, workspace=ws, check=False)
    assert eh.get_status(ws) == eh.EH_OK              # the status word is per call
    lens = c.code_len.clone()
    c.code_len[int(torch.argmax(c.code_len))] = 1     # over-subscribed code
    eh.decompress(c, p, workspace=ws, check=False)
    assert eh.get_status(ws) == eh.EH_ERR_CORRUPT
    c.code_len.copy_(lens)
    c.chunk_bit_off[-1] = c.exp_stream.numel() * 8   # claims more bits than the buffer holds
    eh.decompress(c, p, workspace=ws, check=False)
    assert eh.get_status(ws) == eh.EH_ERR_CORRUPT
    c.chunk_bit_off.copy_(good)
    y = eh.decompress(c, p, workspace=ws)
    assert np.array_equal(host_bits(y, 0), x)


def test_side_stream(eh, oracle):
    # calls take the caller's stream (a torch stream handle, not the default)
    x = synth.normal_bf16(3 * 65536 + 9, seed=12)
    p = eh.plan(0)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        t = dev(x)
        c = eh.compress(t, p, stream=s)
        y = eh.decompress(c, p, stream=s)
    s.synchronize()
    assert_same(c, oracle.compress(0, x))
    assert torch.equal(y, t)


def test_sharded_compress_on_one_gpu(eh, oracle):
    # the two shard entry points for three shards of one tensor, with the
    # counts summed on the device in place of the all-reduce; the stitched
    # shards equal the single-rank stream and every shard decodes alone
    from exponent_entropy_coding_b200 import parallel
    n, world = 5 * 65536 + 123, 3
    x = synth.normal_bf16(n, seed=31)
    p = eh.plan(0)
    counts = torch.zeros(256, dtype=torch.int64, device="cuda")
    backends, xs = [], []
    for r in range(world):
        a, b = parallel.shard_value_range(n, CHUNK, world, r)
        xr = dev(x[a:b])
        be = parallel.GpuShardBackend(0)
        counts += be.begin(xr)
        backends.append(be)
        xs.append(xr)
    outs = []
    for be, xr in zip(backends, xs):
        out, bits = be.finish(xr, counts)
        out.exp_stream_bits = int(bits.item())
        outs.append(out)
    ref = oracle.compress(0, x)
    stream, nbits = parallel.stitch_streams(
        [(o.exp_stream[:o.stream_bytes()].cpu().numpy(), o.exp_stream_bits) for o in outs])
    assert nbits == ref.bits and np.array_equal(stream, ref.stream)
    offs = parallel.stitch_offsets([o.chunk_bit_off.cpu().numpy().view(np.uint64) for o in outs],
                                   [o.exp_stream_bits for o in outs])
    assert np.array_equal(offs, ref.chunk_bit_off)
    assert np.array_equal(np.concatenate([o.sign_mant.cpu().numpy() for o in outs]), ref.sign_mant)
    for o in outs:
        assert np.array_equal(o.code_len.cpu().numpy(), ref.code_len)
    for o, xr in zip(outs, xs):
        assert torch.equal(eh.decompress(o, p), xr)


@pytest.mark.parametrize("n,chunk", [(1, 65536), (3 * 65536 + 17, 65536), (10 * 1024 + 5, 1024)])
def test_bytes_alphabet(eh, oracle, n, chunk):
    # FP4 block scale bytes: every byte is a symbol, no sign/mantissa array
    _, items = synth.workload("nvfp4_scales", scale=16)
    x = np.concatenate([v for _, v in items])[:n]
    c = roundtrip(eh, oracle, 2, x, chunk=chunk)
    assert c.sign_mant.numel() == 0


def test_bytes_every_value(eh, oracle):
    rng = np.random.default_rng(8)
    x = np.tile(np.arange(256, dtype=np.uint8), 1000)[rng.permutation(256 * 1000)]
    roundtrip(eh, oracle, 2, x)


@pytest.mark.parametrize("name,dtype,npdt", [("handworked_bf16.txt", 0, np.uint16),
                                             ("handworked_fp8.txt", 1, np.uint8)])
def test_handworked_goldens(eh, name, dtype, npdt):
    """The hand-worked examples' codes, stream and sign/mantissa bytes, straight
    from the fixtures (no oracle in between)."""
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
    rows = [ln.strip() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    g = dict(r.split(":", 1) for r in rows)
    x = np.array([int(h, 16) for h in g["input_hex"].split()], npdt)
    p = eh.plan(dtype)
    c = eh.compress(dev(x), p)
    lens = c.code_len.cpu().numpy()
    codes = c.code.cpu().numpy().view(np.uint32)
    want_lens = dict(item.split(":") for item in g["lengths"].split())
    for s in range(lens.size):
        assert int(lens[s]) == int(want_lens.get(str(s), 0))
    for item in g["codes"].split():
        s, bits = item.split(":")
        assert format(int(codes[int(s)]), f"0{len(bits)}b") == bits
    assert c.exp_stream_bits == int(g["bits"])
    assert list(c.chunk_bit_off.cpu().numpy().view(np.uint64)) == [int(v) for v in g["offsets"].split()]
    want = bytes(int(h, 16) for h in g["stream_hex"].split())
    assert bytes(c.exp_stream[:len(want)].cpu().numpy()) == want
    assert bytes(c.sign_mant.cpu().numpy()) == bytes(int(h, 16) for h in g["sign_mant_hex"].split())
    assert np.array_equal(host_bits(eh.decompress(c, p), dtype), x)
