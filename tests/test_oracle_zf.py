"""Pins of the ZipFloat comparison codec's oracle (CPU only).

Source: "ZipFloat: An Ultra-fast and Lossless Floating-Point Compressor for
LLM Inference Systems", §3.2 (dominant range [MD - 6, MD + 2), Eq. 4) and
§3.3 (3-bit dense bit planes, 16-bit sparse records, raw sign/mantissa).
What pins it:
  - the page's own remap example (+1 -> 00000101, -1 -> 00000011) and
    hand-worked blocks (tests/golden/zipfloat_block.txt);
  - the sparse records equal the elements outside the dominant range, listed
    here with numpy from the definition;
  - the dense planes re-read bit by bit give the low three bits of e - l_b;
  - every BF16 bit pattern round-trips; sizes follow the closed form.
"""
import os

import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "zipfloat_block.txt")


def _cases():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, val = line.partition(":")
        key, val = key.strip(), val.strip()
        if key == "case":
            cur = {"case": val}
            cases.append(cur)
        else:
            cur[key] = val
    return cases


def bf16_bits(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _plane_bits(dense, block, p, count):
    words = dense[block * 192 + p * 64: block * 192 + p * 64 + 64]
    return np.array([(int(words[i // 32]) >> (i % 32)) & 1 for i in range(count)], np.uint32)


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["case"])
def test_golden_blocks(oracle, case):
    x = bf16_bits([float(v) for v in case["values"].split()])
    md, lb = oracle.zf_block_base(x)
    assert (md, lb) == (int(case["md"]), int(case["lb"]))
    c = oracle.zf_compress(x)
    r = [int(v) for v in case["r"].split()]
    planes = [int(v, 16) for v in case["planes_hex"].split()]
    assert [int(c.dense[p * 64]) for p in range(3)] == planes
    assert all(int(c.dense[p * 64 + w]) == 0 for p in range(3) for w in range(1, 64))
    assert c.sparse.tolist() == [int(v) for v in case["records"].split()]
    assert int(c.meta[0]) == lb | (len(c.sparse) << 8)
    low = sum(_plane_bits(c.dense, 0, p, x.size) << p for p in range(3))
    assert low.tolist() == [v & 7 for v in r]
    assert np.array_equal(oracle.zf_decompress(c), x)


def test_page_remap_example(oracle):
    # +1 and -1 in a block whose mode is field 129 (the page's l_b = 123)
    x = bf16_bits([4.0] * 6 + [2.0, 0.5])
    c = oracle.zf_compress(x)
    low = sum(_plane_bits(c.dense, 0, p, x.size) << p for p in range(3))
    assert format(int(low[6]), "08b") == "00000101"   # +1
    assert format(int(low[7]), "08b") == "00000011"   # -1
    assert c.sparse.size == 0


def _records_by_definition(x):
    """Sparse records straight from the definition, block by block."""
    out, offs, lbs = [], [], []
    e = ((x >> 7) & 0xFF).astype(np.int64)
    for b0 in range(0, x.size, 2048):
        eb = e[b0:b0 + 2048]
        hist = np.bincount(eb, minlength=256)
        md = int(np.argmax(hist))          # first maximum = smaller field on ties
        lb = (md - 6) % 256
        r = (eb - lb) % 256
        idx = np.nonzero(r >= 8)[0]
        offs.append(len(out))
        lbs.append(lb)
        out.extend(((idx << 5) | (r[idx] >> 3)).tolist())
    return np.array(out, np.uint16), np.array(offs, np.uint32), np.array(lbs, np.uint32)


@pytest.mark.parametrize("n,seed", [(2048, 0), (5000, 1), (3 * 2048 + 1, 2), (20000, 3)])
def test_records_and_planes_by_definition(oracle, n, seed):
    rng = np.random.default_rng(seed)
    x = synth.student_t_bf16((n,), rng)
    c = oracle.zf_compress(x)
    rec, offs, lbs = _records_by_definition(x)
    assert np.array_equal(c.sparse, rec)
    assert np.array_equal(c.sparse_off, offs)
    assert np.array_equal(c.meta & 0xFF, lbs)
    B = (n + 2047) // 2048
    for b in range(B):
        cnt = min(2048, n - 2048 * b)
        eb = ((x[2048 * b: 2048 * b + cnt] >> 7) & 0xFF).astype(np.int64)
        low = sum(_plane_bits(c.dense, b, p, cnt) << p for p in range(3))
        assert np.array_equal(low, ((eb - lbs[b]) % 256) & 7)
        assert int(c.meta[b]) >> 8 == (offs[b + 1] if b + 1 < B else rec.size) - offs[b]
    # closed-form size
    assert c.nbytes() == n + 8 * B + 768 * B + 2 * rec.size
    assert np.array_equal(oracle.zf_decompress(c), x)


def test_every_bf16_pattern_roundtrips(oracle):
    x = np.random.default_rng(7).permutation(np.arange(65536, dtype=np.uint32)).astype(np.uint16)
    c = oracle.zf_compress(x)
    assert np.array_equal(oracle.zf_decompress(c), x)
    # sign/mantissa are the raw low bits of every value
    assert np.array_equal(c.sign_mant, (((x >> 8) & 0x80) | (x & 0x7F)).astype(np.uint8))


def test_empty_and_corrupt(oracle):
    c = oracle.zf_compress(np.zeros(0, np.uint16))
    assert c.sparse.size == 0 and oracle.zf_decompress(c).size == 0
    x = synth.normal_bf16(4096, seed=5)
    c = oracle.zf_compress(x)
    c.meta[1] = (c.meta[1] & 0xFF) | ((int(c.meta[1] >> 8) + 5) << 8)   # claims records it lacks
    with pytest.raises(oracle.OracleError):
        oracle.zf_decompress(c)


def test_ratio_against_the_huffman_format(oracle):
    # same synthetic weights as the block: the Huffman code of the exponents is
    # smaller than 3 dense bits plus 16-bit records (the page reports DFloat11
    # slightly ahead of ZipFloat in ratio); both stay well below 1
    x = synth.student_t_bf16((64, 4096), np.random.default_rng(2)).reshape(-1)
    c = oracle.zf_compress(x)
    z = c.nbytes() / (2 * x.size)
    h = oracle.compress(oracle.BF16, x)
    hb = (h.stream.size + h.sign_mant.size + 8 * h.chunk_bit_off.size) / (2 * x.size)
    assert hb < z < 0.85
    # the records are the elements outside [MD - 6, MD + 2): a few percent
    assert 0.0 < c.sparse.size / x.size < 0.15
