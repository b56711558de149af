"""Compression of one tensor split across ranks (one process per GPU).

Every rank holds a contiguous shard of whole 64K-value chunks.  The codebook
must be the one of the whole tensor (the DFloat11 article, "方法介绍": the
Huffman tree comes from the distribution of all exponents), so the protocol
has exactly two small exchanges:

1. each rank histograms its shard; one all-reduce (sum) of the A exponent
   counts (2 KB for BF16) gives every rank the global histogram, from which
   every rank builds the identical codebook;
2. each rank encodes its shard into its own stream (offsets from bit 0); one
   all-gather of the per-rank bit counts gives every shard its global bit
   offset.

Decompression needs no communication: a shard decodes on its own with the
shared codebook.  `stitch_streams` concatenates shard streams into the
stream a single rank would have produced.

The compute steps come from a backend object with ``begin(x) -> counts`` and
``finish(x, counts) -> (compressed, bits)``; `GpuShardBackend` runs them with
libexphuff on the local GPU.  Collectives go through torch.distributed.
"""
from dataclasses import dataclass
from typing import List, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist


def shard_chunk_range(n: int, chunk: int, world: int, rank: int) -> Tuple[int, int]:
    """Chunk range [c0, c1) of `rank` for a tensor of n values: contiguous,
    balanced to within one chunk."""
    C = -(-n // chunk)
    return C * rank // world, C * (rank + 1) // world


def shard_value_range(n: int, chunk: int, world: int, rank: int) -> Tuple[int, int]:
    c0, c1 = shard_chunk_range(n, chunk, world, rank)
    return min(n, c0 * chunk), min(n, c1 * chunk)


@dataclass
class ShardResult:
    compressed: object   # backend's compressed shard
    base_bit: int        # global bit offset of the shard's first code
    total_bits: int      # bits of the whole tensor
    shard_bits: List[int]  # bits of every rank's shard


def compress_sharded(x_local: torch.Tensor, backend, group=None) -> ShardResult:
    """Runs the two-exchange protocol for this rank's shard."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    counts = backend.begin(x_local)
    dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    obj, bits = backend.finish(x_local, counts)
    gathered = [torch.zeros_like(bits) for _ in range(world)]
    dist.all_gather(gathered, bits, group=group)
    shard_bits = [int(g.reshape(-1)[0].item()) for g in gathered]
    if hasattr(obj, "exp_stream_bits"):
        obj.exp_stream_bits = shard_bits[rank]
    return ShardResult(obj, sum(shard_bits[:rank]), sum(shard_bits), shard_bits)


def stitch_streams(parts: Sequence[Tuple[np.ndarray, int]]) -> Tuple[np.ndarray, int]:
    """Concatenates MSB-first bit streams (bytes, bit count) into one."""
    bits = [np.unpackbits(np.asarray(b, dtype=np.uint8), bitorder="big")[:n] for b, n in parts]
    allbits = np.concatenate(bits) if bits else np.zeros(0, np.uint8)
    return np.packbits(allbits, bitorder="big"), int(allbits.size)


def stitch_offsets(offs: Sequence[np.ndarray], shard_bits: Sequence[int]) -> np.ndarray:
    """Global chunk offsets from the shards' local offsets (each [C_r + 1])."""
    out, base = [], 0
    for o, nb in zip(offs, shard_bits):
        o = np.asarray(o, dtype=np.uint64)
        out.append(o[:-1] + np.uint64(base))
        base += nb
    out.append(np.array([base], dtype=np.uint64))
    return np.concatenate(out)


class GpuShardBackend:
    """libexphuff on the local GPU: begin = eh_compress_shard_begin, finish =
    eh_compress_shard_finish (bit count written on the device, no host wait)."""

    def __init__(self, dtype: int, chunk_elems: int = 0, max_code_len: int = 0):
        from . import exphuff as eh
        self.eh = eh
        self.plan = eh.plan(dtype, chunk_elems, max_code_len)
        self._out = None
        self._ws = None

    def begin(self, x: torch.Tensor) -> torch.Tensor:
        eh = self.eh
        n = x.numel()
        self._out = eh.alloc_compressed(self.plan, n, x.device)
        self._ws = torch.empty(eh.compress_bound(self.plan, n)[2], dtype=torch.uint8, device=x.device)
        counts = torch.zeros(eh.alphabet(self.plan.dtype), dtype=torch.int64, device=x.device)
        eh.compress_shard_begin(x, self._out, counts, self.plan, self._ws)
        return counts

    def finish(self, x: torch.Tensor, counts: torch.Tensor):
        bits = torch.zeros(1, dtype=torch.int64, device=x.device)
        self.eh.compress_shard_finish(x, self._out, counts, self.plan, self._ws, bits_dev=bits)
        return self._out, bits
