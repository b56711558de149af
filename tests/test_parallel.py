"""Sharded compression protocol across ranks, on CPU with gloo.

The protocol code of exponent_entropy_coding_b200.parallel (all-reduce of the
exponent counts, all-gather of the shard bit counts) runs in 2 and 3 spawned
processes; the per-rank compute steps come from the CPU oracle.  The shards
stitched together must equal the single-rank stream byte for byte, and every
shard must decode on its own with the shared codebook.
"""
import os
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exponent_entropy_coding_b200 import parallel, synth


class OracleShardBackend:
    def __init__(self, dtype, chunk, lmax=32):
        from oracle import ehref
        self.o, self.dtype, self.chunk, self.lmax = ehref, dtype, chunk, lmax

    def begin(self, x):
        return torch.from_numpy(self.o.histogram(self.dtype, x.numpy()).astype(np.int64))

    def finish(self, x, counts):
        o, d = self.o, self.dtype
        lens = o.code_lengths(counts.numpy().astype(np.uint64), self.lmax)
        codes = o.canonical_codes(lens)
        off, stream, bits = o.encode(d, x.numpy(), self.chunk, lens, codes)
        res = {"len": lens, "code": codes, "off": off, "stream": stream, "bits": bits,
               "sm": o.pack_sm(d, x.numpy())}
        return res, torch.tensor([bits], dtype=torch.int64)


def _worker(rank, world, initfile, dtype, n, chunk, q):
    dist.init_process_group("gloo", init_method=f"file://{initfile}", rank=rank, world_size=world)
    try:
        full = synth.normal_bf16(n, seed=n) if dtype == 0 else synth.normal_fp8(n, seed=n)
        a, b = parallel.shard_value_range(n, chunk, world, rank)
        x = torch.from_numpy(full[a:b].copy())
        res = parallel.compress_sharded(x, OracleShardBackend(dtype, chunk))
        r = res.compressed
        # every shard decodes alone with the shared codebook
        from oracle import ehref
        part = ehref.Compressed(dtype, b - a, chunk, 32, r["len"], r["code"], r["off"], r["stream"],
                                r["sm"], r["bits"])
        assert np.array_equal(ehref.decompress(part), full[a:b])
        got = [None] * world
        dist.all_gather_object(got, (r["stream"], r["bits"], r["off"], r["sm"], r["len"], res.base_bit))
        if rank == 0:
            ref = ehref.compress(dtype, full, chunk=chunk)
            stream, nbits = parallel.stitch_streams([(g[0], g[1]) for g in got])
            offs = parallel.stitch_offsets([g[2] for g in got], [g[1] for g in got])
            ok = (nbits == ref.bits and np.array_equal(stream, ref.stream)
                  and np.array_equal(offs, ref.chunk_bit_off)
                  and np.array_equal(np.concatenate([g[3] for g in got]), ref.sign_mant)
                  and all(np.array_equal(g[4], ref.code_len) for g in got)
                  and [g[5] for g in got] == [int(ref.chunk_bit_off[parallel.shard_chunk_range(
                      n, chunk, world, r_)[0]]) for r_ in range(world)])
            q.put(bool(ok))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,dtype,n,chunk", [(2, 0, 10 * 1024 + 37, 1024), (3, 1, 7 * 1024 + 1, 1024),
                                                 (2, 0, 3 * 65536 + 5, 65536)])
def test_sharded_protocol_gloo(world, dtype, n, chunk):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with tempfile.TemporaryDirectory() as d:
        initfile = os.path.join(d, "init")
        mp.start_processes(_worker, args=(world, initfile, dtype, n, chunk, q), nprocs=world,
                           join=True, start_method="spawn")
    assert q.get(timeout=30) is True


def test_shard_ranges_cover_whole_chunks():
    for n, chunk, world in [(10 * 1024 + 37, 1024, 3), (65536 * 5, 65536, 8), (5, 1024, 4)]:
        spans = [parallel.shard_value_range(n, chunk, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == n
        for (a, b), (c, d) in zip(spans, spans[1:]):
            assert b == c and a % chunk == 0
        sizes = [parallel.shard_chunk_range(n, chunk, world, r) for r in range(world)]
        counts = [c1 - c0 for c0, c1 in sizes]
        assert max(counts) - min(counts) <= 1


def test_stitch_matches_bit_concatenation():
    rng = np.random.default_rng(0)
    parts, bits = [], []
    for nb in (13, 0, 64, 7, 100):
        bb = rng.integers(0, 2, nb).astype(np.uint8)
        bits.append(bb)
        parts.append((np.packbits(bb, bitorder="big"), nb))
    s, n = parallel.stitch_streams(parts)
    assert n == sum(p[1] for p in parts)
    assert np.array_equal(np.unpackbits(s, bitorder="big")[:n], np.concatenate(bits))
