"""Prefetcher: decompression into a ring of operand slots on a decode stream.

The consumer reads each slot on its own stream between acquire() and
release().  Parity: every slot view holds exactly the original bits (the
oracle's decompression of the same tensor is checked against it too), and a
GEMM that reads a slot view gives exactly the result of the same GEMM on the
uncompressed weights.  The ordering tests make the consumer slow
(torch.cuda._sleep) so that a decode that did not wait for the release would
overwrite a slot before it is read.
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


def _blocks(n_blocks, seed):
    # blocks of three matrices: Llama-3.1-8B q, k, v rows divided by 64 (several
    # chunks, ragged tails), plus a tensor shorter than a chunk
    out = []
    for b in range(n_blocks):
        mats = [x for _, x in synth.llama8b_block(seed=seed + b, scale=64, count=3)]
        mats.append(synth.normal_bf16(1000 + 37 * b, seed=seed + 100 + b))
        out.append(mats)
    return out


def _slot_bytes(blocks):
    return max(sum((2 * x.size + 255) // 256 * 256 for x in blk) for blk in blocks)


@pytest.mark.parametrize("depth,max_ctas", [(1, 0), (2, 0), (3, 8)])
def test_ring_roundtrip(eh, oracle, depth, max_ctas):
    blocks = _blocks(5, seed=40)
    p = eh.plan(0)
    comp = [[eh.compress(_dev(x), p) for x in blk] for blk in blocks]
    pf = eh.Prefetcher(p, depth, _slot_bytes(blocks), "cuda", max_ctas=max_ctas)
    cons = torch.cuda.Stream()
    outs = [[torch.empty(x.size, dtype=torch.int16, device="cuda") for x in blk] for blk in blocks]
    pending = []
    for i in range(min(depth, len(blocks))):
        pending.append(pf.submit(comp[i]))
    with torch.cuda.stream(cons):
        for i in range(len(blocks)):
            slot, views = pending.pop(0)
            pf.acquire(slot, cons)
            torch.cuda._sleep(200000)  # a slow consumer
            for v, o in zip(views, outs[i]):
                o.copy_(v)
            pf.release(slot, cons)
            if i + depth < len(blocks):
                pending.append(pf.submit(comp[i + depth]))
    torch.cuda.synchronize()
    for s in range(depth):
        assert pf.status(s) == eh.EH_OK
    for blk, ob in zip(blocks, outs):
        for x, o in zip(blk, ob):
            assert np.array_equal(o.cpu().numpy().view(np.uint16), x)
    ref = oracle.decompress(oracle.compress(0, blocks[-1][0]))
    assert np.array_equal(outs[-1][0].cpu().numpy().view(np.uint16), ref)
    pf.close()


def test_gemm_reads_slot(eh):
    blocks = _blocks(3, seed=50)
    p = eh.plan(0)
    comp = [[eh.compress(_dev(x), p) for x in blk[:3]] for blk in blocks]
    pf = eh.Prefetcher(p, 2, _slot_bytes([b[:3] for b in blocks]), "cuda")
    cons = torch.cuda.current_stream()
    torch.manual_seed(0)
    xs = torch.randn(16, 4096, device="cuda").to(torch.bfloat16)
    pending = [pf.submit(comp[0]), pf.submit(comp[1])]
    for i, blk in enumerate(blocks):
        slot, views = pending.pop(0)
        pf.acquire(slot)
        got = [xs @ v.view(torch.bfloat16).view(-1, 4096).t() for v in views]
        pf.release(slot)
        if i + 2 < len(blocks):
            pending.append(pf.submit(comp[i + 2]))
        for w, g in zip(blk[:3], got):
            wt = _dev(w).view(torch.bfloat16).view(-1, 4096)
            assert torch.equal(g, xs @ wt.t())
    cons.synchronize()
    pf.close()


def test_slot_state_errors(eh):
    p = eh.plan(0)
    x = synth.normal_bf16(70000, seed=3)
    c = eh.compress(_dev(x), p)
    pf = eh.Prefetcher(p, 1, 2 * x.size, "cuda")
    with pytest.raises(eh.EhError):
        pf.acquire(0)                       # nothing submitted
    slot, (v,) = pf.submit([c])
    with pytest.raises(eh.EhError):
        pf.submit([c])                      # the only slot is not released
    with pytest.raises(eh.EhError):
        pf.release(slot)                    # not acquired
    pf.acquire(slot)
    with pytest.raises(eh.EhError):
        pf.acquire(slot)                    # already acquired
    y = v.clone()
    pf.release(slot)
    slot2, _ = pf.submit([c])               # released: the slot is reusable
    assert slot2 == slot
    assert pf.status(slot) == eh.EH_OK
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy().view(np.uint16), x)
    big = eh.compress(_dev(synth.normal_bf16(x.size + 200, seed=4)), p)
    pf.acquire(slot)
    pf.release(slot)
    with pytest.raises(eh.EhError) as e:
        pf.submit([big])                    # larger than the slot
    assert e.value.code == eh.EH_ERR_NOMEM
    pf.close()


def test_corrupt_block_sets_slot_status(eh):
    p = eh.plan(0)
    x = synth.normal_bf16(3 * 65536, seed=11)
    c = eh.compress(_dev(x), p)
    good = eh.compress(_dev(x), p)
    c.chunk_bit_off[1] += 5                 # a chunk boundary moves
    pf = eh.Prefetcher(p, 2, 2 * x.size, "cuda")
    s0, _ = pf.submit([c])
    s1, (v1,) = pf.submit([good])
    assert pf.status(s0) == eh.EH_ERR_CORRUPT
    assert pf.status(s1) == eh.EH_OK        # each slot keeps its own status word
    torch.cuda.synchronize()
    assert np.array_equal(v1.cpu().numpy().view(np.uint16), x)
    pf.close()
