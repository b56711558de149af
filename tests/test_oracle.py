"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against one of: values printed on the pages
(golden files with citations), hand-worked examples, closed forms (entropy
bounds, optimal-cost identities), brute force over tiny alphabets, or the
floating-point arithmetic of the formats (frexp).  A mistake in the oracle
(a wrong tie rule, a dropped level in package-merge, a flipped bit order,
a wrong bias) fails at least one of them.
"""
import heapq
import itertools
import math
import os

import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def golden_cases(name):
    cases, cur = [], None
    for row in read_golden(name):
        key, _, val = row.partition(":")
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


def fp8_bits(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


# ---------------------------------------------------------------- S1 split

def test_zipfloat_biased_exponent_example(oracle):
    for row in read_golden("zipfloat_biased_exponent.txt"):
        value, exp, binary = row.split()
        e, sm = oracle.split(oracle.BF16, bf16_bits([float(value)]))
        assert format(int(e[0]), "08b") == binary
        assert int(e[0]) == int(exp) + 127
        assert sm[0] == 0


def test_fp8_field_examples(oracle):
    for row in read_golden("fp8_e4m3_fields.txt"):
        value, bits_hex, e_s, sm_hex = row.split()
        bits = fp8_bits([float(value)])
        assert int(bits[0]) == int(bits_hex, 16)
        e, sm = oracle.split(oracle.FP8_E4M3, bits)
        assert int(e[0]) == int(e_s) and int(sm[0]) == int(sm_hex, 16)


def _fields_from_value(x, bias, mbits, emax_field):
    """Exponent field and sign+mantissa of a finite float from frexp."""
    s = 1 if math.copysign(1.0, x) < 0 else 0
    a = abs(x)
    if a == 0.0:
        return 0, s << mbits
    m, k = math.frexp(a)            # a = m * 2^k, m in [0.5, 1)
    unb = k - 1                      # a = (2m) * 2^(k-1), 2m in [1, 2)
    field = unb + bias
    if field <= 0:                   # subnormal: a = frac * 2^(1-bias)
        frac = a / 2.0 ** (1 - bias)
        return 0, (s << mbits) | int(round(frac * 2 ** mbits))
    assert field <= emax_field
    mant = int(round((2 * m - 1) * 2 ** mbits))
    return field, (s << mbits) | mant


def test_split_matches_frexp_bf16(oracle):
    rng = np.random.default_rng(11)
    vals = np.concatenate([rng.standard_normal(2000) * 0.02, rng.standard_normal(500) * 1e3,
                           rng.standard_normal(200) * 1e-39, [0.0, -0.0, 1.0, -2.5]])
    bits = bf16_bits(vals.tolist())
    back = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    e, sm = oracle.split(oracle.BF16, bits)
    for i, x in enumerate(back.astype(np.float64)):
        f, s = _fields_from_value(float(x), 127, 7, 254)
        assert (int(e[i]), int(sm[i])) == (f, s), (x, hex(bits[i]))


def test_split_matches_frexp_fp8(oracle):
    bits = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(bits.copy()).view(torch.float8_e4m3fn).float().numpy()
    e, sm = oracle.split(oracle.FP8_E4M3, bits)
    for i, x in enumerate(vals.astype(np.float64)):
        if math.isnan(x):               # 0x7F / 0xFF: all-ones exponent and mantissa
            assert int(e[i]) == 15 and (int(sm[i]) & 7) == 7
            continue
        f, s = _fields_from_value(float(x), 7, 3, 15)
        assert (int(e[i]), int(sm[i])) == (f, s), (x, hex(i))


@pytest.mark.parametrize("dtype,count", [(0, 1 << 16), (1, 1 << 8)])
def test_exhaustive_roundtrip(oracle, dtype, count):
    """Every bit pattern (NaN, Inf, zeros, subnormals included) round-trips."""
    x = np.arange(count, dtype=np.uint16 if dtype == 0 else np.uint8)
    rng = np.random.default_rng(5)
    x = x[rng.permutation(count)]
    e, sm = oracle.split(dtype, x)
    assert np.array_equal(oracle.merge(dtype, e, sm), x)
    for chunk in (65536, 1024, 4096):
        c = oracle.compress(dtype, x, chunk=chunk)
        assert np.array_equal(oracle.decompress(c), x)


# ------------------------------------------------------------ S3 code lengths

def brute_min_cost(cnt, lmax):
    m = len(cnt)
    best = None
    cnt = np.asarray(cnt, dtype=np.int64)
    for lens in itertools.product(range(1, lmax + 1), repeat=m):
        if sum(2.0 ** -l for l in lens) <= 1.0:
            c = int(np.dot(cnt, lens))
            best = c if best is None else min(best, c)
    return best


def kraft(lens):
    return sum(2.0 ** -int(l) for l in lens if l)


@pytest.mark.parametrize("seed", range(12))
def test_huffman_bruteforce_optimal(oracle, seed):
    rng = np.random.default_rng(seed)
    m = int(rng.integers(2, 7))
    cnt = rng.integers(1, 60, size=m).astype(np.uint64)
    if seed % 3 == 0:
        cnt[:] = rng.integers(1, 4, size=m)   # many ties
    lens = oracle.code_lengths(cnt, 32)
    assert int(np.dot(cnt.astype(np.int64), lens.astype(np.int64))) == brute_min_cost(cnt, m - 1)
    assert kraft(lens) == 1.0


@pytest.mark.parametrize("lmax", [3, 4, 5, 6])
@pytest.mark.parametrize("seed", range(4))
def test_length_limited_bruteforce(oracle, lmax, seed):
    rng = np.random.default_rng(100 + seed)
    m = int(rng.integers(4, 7 if lmax == 3 else 8))
    # Fibonacci-like skew forces the limit to bind
    fib = [1, 1]
    while len(fib) < m:
        fib.append(fib[-1] + fib[-2])
    cnt = np.array(fib, dtype=np.uint64)[rng.permutation(m)]
    lens = oracle.code_lengths(cnt, lmax)
    assert lens.max() <= lmax
    assert kraft(lens) == 1.0
    assert int(np.dot(cnt.astype(np.int64), lens.astype(np.int64))) == brute_min_cost(cnt, lmax)


def huffman_cost_heapq(cnt):
    """Optimal prefix-code cost = sum of the merged weights (any Huffman tree)."""
    h = [int(c) for c in cnt if c]
    if len(h) < 2:
        return sum(h)
    heapq.heapify(h)
    cost = 0
    while len(h) > 1:
        a, b = heapq.heappop(h), heapq.heappop(h)
        cost += a + b
        heapq.heappush(h, a + b)
    return cost


@pytest.mark.parametrize("seed", range(6))
def test_huffman_cost_full_alphabet(oracle, seed):
    rng = np.random.default_rng(200 + seed)
    cnt = np.zeros(256, np.uint64)
    k = int(rng.integers(2, 257))
    idx = rng.choice(256, k, replace=False)
    cnt[idx] = (rng.pareto(1.2, k) * 50 + 1).astype(np.uint64)
    lens = oracle.code_lengths(cnt, 32)
    if oracle.huffman_depths(cnt).max() <= 32:
        assert int(np.dot(cnt.astype(np.int64), lens.astype(np.int64))) == huffman_cost_heapq(cnt)
    assert kraft(lens) == 1.0
    assert np.all((lens > 0) == (cnt > 0))


def entropy_bits(cnt):
    p = cnt[cnt > 0].astype(np.float64) / cnt.sum()
    return float(-(p * np.log2(p)).sum())


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_entropy_bound_workloads(oracle, name):
    dt, items = synth.workload(name, scale=64)
    dtype = 0 if dt == "bf16" else 1
    for _, x in items:
        cnt = oracle.histogram(dtype, x)
        lens = oracle.code_lengths(cnt, 32)
        H = entropy_bits(cnt)
        Lbar = float(np.dot(cnt.astype(np.float64), lens)) / cnt.sum()
        assert H <= Lbar < H + 1
        # the pages put BF16 exponent entropy at about 2-3 bits (ZipFloat §2)
        if dtype == 0:
            assert 2.0 < H < 3.2


def test_tie_rules_golden(oracle):
    for case in golden_cases("tie_rules.txt"):
        cnt = np.array([int(v) for v in case["counts"].split()], np.uint64)
        lmax = int(case["lmax"])
        depths = [int(v) for v in case["depths"].split()]
        want = [int(v) for v in case["lengths"].split()]
        assert list(oracle.huffman_depths(cnt)) == depths, case["case"]
        assert list(oracle.code_lengths(cnt, lmax)) == want, case["case"]
        if case["case"] == "package_merge":
            assert list(oracle.package_merge(cnt, lmax)) == want
        if "codes" in case:
            ln = oracle.code_lengths(cnt, lmax)
            codes = oracle.canonical_codes(ln)
            got = [format(int(c), f"0{int(l)}b") for c, l in zip(codes, ln)]
            assert got == case["codes"].split()


def test_rfc1951_canonical_example(oracle):
    rows = dict(r.split(":", 1) for r in read_golden("rfc1951_canonical.txt"))
    lens = np.array([int(v) for v in rows["lengths"].split()], np.uint8)
    codes = oracle.canonical_codes(lens)
    got = [format(int(c), f"0{int(l)}b") for c, l in zip(codes, lens)]
    assert got == rows["codes"].split()


def test_infeasible_and_degenerate_lengths(oracle):
    cnt = np.ones(9, np.uint64)
    with pytest.raises(oracle.OracleError) as ei:
        oracle.code_lengths(cnt, 3)             # 9 symbols > 2^3
    assert ei.value.code == oracle.EINFEASIBLE
    assert list(oracle.code_lengths(np.ones(8, np.uint64), 3)) == [3] * 8
    one = np.zeros(256, np.uint64)
    one[77] = 5
    ln = oracle.code_lengths(one, 32)
    assert ln[77] == 1 and ln.sum() == 1
    assert oracle.code_lengths(np.zeros(16, np.uint64), 32).sum() == 0
    assert list(oracle.code_lengths(np.array([3, 9], np.uint64), 1)) == [1, 1]


# ------------------------------------------------------------ S4/S5 stream

def test_handworked_example(oracle):
    g = dict(r.split(":", 1) for r in read_golden("handworked_bf16.txt"))
    x = np.array([int(h, 16) for h in g["input_hex"].split()], np.uint16)
    e, _ = oracle.split(oracle.BF16, x)
    assert list(e) == [int(v) for v in g["exponents"].split()]
    c = oracle.compress(oracle.BF16, x)
    for item in g["lengths"].split():
        s, l = item.split(":")
        assert c.code_len[int(s)] == int(l)
    for item in g["codes"].split():
        s, bits = item.split(":")
        assert format(int(c.code[int(s)]), f"0{len(bits)}b") == bits
    assert c.bits == int(g["bits"])
    assert list(c.chunk_bit_off) == [int(v) for v in g["offsets"].split()]
    assert bytes(c.stream) == bytes(int(h, 16) for h in g["stream_hex"].split())
    assert bytes(c.sign_mant) == bytes(int(h, 16) for h in g["sign_mant_hex"].split())
    cnt = oracle.histogram(oracle.BF16, x)
    assert abs(entropy_bits(cnt) - float(g["entropy_bits"])) < 1e-12
    assert np.array_equal(oracle.decompress(c), x)


def test_handworked_fp8_example(oracle):
    g = dict(r.split(":", 1) for r in read_golden("handworked_fp8.txt"))
    x = np.array([int(h, 16) for h in g["input_hex"].split()], np.uint8)
    e, _ = oracle.split(oracle.FP8_E4M3, x)
    assert list(e) == [int(v) for v in g["exponents"].split()]
    c = oracle.compress(oracle.FP8_E4M3, x)
    for item in g["lengths"].split():
        s, l = item.split(":")
        assert c.code_len[int(s)] == int(l)
    assert int(np.count_nonzero(c.code_len)) == len(g["lengths"].split())
    for item in g["codes"].split():
        s, bits = item.split(":")
        assert format(int(c.code[int(s)]), f"0{len(bits)}b") == bits
    assert c.bits == int(g["bits"])
    assert list(c.chunk_bit_off) == [int(v) for v in g["offsets"].split()]
    assert bytes(c.stream) == bytes(int(h, 16) for h in g["stream_hex"].split())
    assert bytes(c.sign_mant) == bytes(int(h, 16) for h in g["sign_mant_hex"].split())
    cnt = oracle.histogram(oracle.FP8_E4M3, x)
    assert abs(entropy_bits(cnt) - float(g["entropy_bits"])) < 1e-12
    assert np.array_equal(oracle.decompress(c), x)


def _bits_of(stream, nbits):
    return np.unpackbits(stream, bitorder="big")[:nbits]


@pytest.mark.parametrize("dtype,n,chunk", [(0, 200_003, 65536), (1, 150_001, 65536),
                                           (0, 70_000, 1024), (1, 4097, 1024)])
def test_stream_invariants(oracle, dtype, n, chunk):
    rng = np.random.default_rng(n)
    x = synth.normal_bf16(n, seed=n) if dtype == 0 else synth.normal_fp8(n, seed=n)
    c = oracle.compress(dtype, x, chunk=chunk)
    e, sm = oracle.split(dtype, x)
    cnt = np.bincount(e, minlength=oracle.alphabet(dtype)).astype(np.uint64)
    assert np.array_equal(cnt, oracle.histogram(dtype, x))
    lens = c.code_len.astype(np.int64)
    # closed-form sizes
    assert c.bits == int(np.dot(cnt.astype(np.int64), lens))
    assert c.stream.size == (c.bits + 7) // 8
    assert c.sign_mant.size == (n if dtype == 0 else (n + 1) // 2)
    # offsets = running sums of per-element lengths at chunk starts
    per = lens[e]
    cum = np.concatenate([[0], np.cumsum(per)])
    C = -(-n // chunk)
    assert list(c.chunk_bit_off) == [int(cum[min(k * chunk, n)]) for k in range(C + 1)]
    # the stream is the concatenation of codes, MSB first; zero padding
    bits = _bits_of(c.stream, c.stream.size * 8)
    probe = rng.choice(n, 300, replace=False)
    for i in probe:
        L = int(per[i])
        word = int("".join(map(str, bits[cum[i]:cum[i] + L])), 2)
        assert word == int(c.code[e[i]])
    assert not bits[c.bits:].any()
    # prefix-free, complete code
    present = np.nonzero(lens)[0]
    words = [format(int(c.code[s]), f"0{int(lens[s])}b") for s in present]
    for a in words:
        for b in words:
            assert a == b or not b.startswith(a)
    if present.size >= 2:
        assert kraft(lens) == 1.0
    # sign/mantissa layout
    if dtype == 0:
        assert np.array_equal(c.sign_mant, sm)
    else:
        assert np.array_equal(c.sign_mant & 0xF, sm[0::2])
        assert np.array_equal(c.sign_mant[: n // 2] >> 4, sm[1::2])
        if n % 2:
            assert c.sign_mant[-1] >> 4 == 0
    assert np.array_equal(oracle.decompress(c), x)
    # partial chunk-range decode
    if C >= 3:
        part = oracle.decompress(c, 1, C - 2)
        assert np.array_equal(part, x[chunk:(C - 1) * chunk])


def test_degenerate_inputs(oracle):
    for dtype in (0, 1):
        dt = np.uint16 if dtype == 0 else np.uint8
        c = oracle.compress(dtype, np.zeros(0, dt))
        assert c.bits == 0 and list(c.chunk_bit_off) == [0] and c.code_len.sum() == 0
        assert oracle.decompress(c).size == 0
        one = np.array([0x3F80 if dtype == 0 else 0x38], dt)
        c = oracle.compress(dtype, one)
        assert c.bits == 1 and bytes(c.stream) == b"\x00"
        assert np.array_equal(oracle.decompress(c), one)
        same = np.full(70_001, one[0], dt)     # single symbol, ragged chunk
        c = oracle.compress(dtype, same)
        assert c.bits == 70_001 and not c.stream.any()
        assert np.array_equal(oracle.decompress(c), same)
    odd = synth.normal_fp8(7, seed=3)
    c = oracle.compress(1, odd)
    assert c.sign_mant.size == 4 and c.sign_mant[-1] >> 4 == 0
    assert np.array_equal(oracle.decompress(c), odd)


def optimal_limited_cost(cnt, lmax):
    """Minimum of sum(count * length) over prefix codes with lengths <= lmax,
    computed exactly level by level, independently of package-merge: with the
    counts sorted in decreasing order the lengths are nondecreasing, so a code
    is a choice, at each depth d, of how many of the open nodes become leaves
    (taking the next most frequent symbols); the others become internal and
    open twice as many nodes at depth d + 1."""
    w = sorted((int(c) for c in cnt if c), reverse=True)
    n = len(w)
    if n <= 1:
        return sum(w)
    pre = [0]
    for v in w:
        pre.append(pre[-1] + v)
    best = None
    cur = {(0, 2): 0}  # (symbols placed, nodes open at depth d) -> cost
    for d in range(1, lmax + 1):
        nxt = {}
        for (j, a), c in cur.items():
            for k in range(0, min(a, n - j) + 1):
                cost = c + d * (pre[j + k] - pre[j])
                if j + k == n:
                    best = cost if best is None else min(best, cost)
                    continue
                na = min(2 * (a - k), n - j - k)
                if na and cost < nxt.get((j + k, na), cost + 1):
                    nxt[(j + k, na)] = cost
        cur = nxt
    return best


@pytest.mark.parametrize("lmax", [3, 4, 5, 7, 9])
@pytest.mark.parametrize("seed", range(3))
def test_length_limited_matches_exact_dp(oracle, lmax, seed):
    rng = np.random.default_rng(300 + seed)
    m = int(rng.integers(lmax + 1, min(2 ** lmax, 40) + 1))
    cnt = (rng.pareto(1.0, m) * 20 + 1).astype(np.uint64)
    lens = oracle.code_lengths(cnt, lmax)
    assert lens.max() <= lmax and kraft(lens) == 1.0
    assert int(np.dot(cnt.astype(np.int64), lens.astype(np.int64))) == optimal_limited_cost(cnt, lmax)


def _fib(m):
    f = [1, 1]
    while len(f) < m:
        f.append(f[-1] + f[-2])
    return f[:m]


def test_fibonacci_depth_32_at_the_format_limit(oracle):
    # 33 Fibonacci counts: Huffman depth exactly 32 = the format's longest
    # code; the limit does not bind, so the cost is the plain Huffman cost
    cnt = np.zeros(256, np.uint64)
    cnt[60:93] = _fib(33)
    assert oracle.huffman_depths(cnt).max() == 32
    lens = oracle.code_lengths(cnt, 32)
    assert lens.max() == 32 and int((lens == 32).sum()) == 2
    assert kraft(lens) == 1.0
    cost = int(np.dot(cnt.astype(np.int64), lens.astype(np.int64)))
    assert cost == huffman_cost_heapq(cnt) == optimal_limited_cost(cnt, 32)


def test_package_merge_at_limit_32(oracle):
    # 34 Fibonacci counts: Huffman depth 33 exceeds the format's 32, so the
    # lengths come from package-merge; they are optimal among codes of at
    # most 32 bits (exact level DP) and strictly costlier than Huffman
    cnt = np.zeros(256, np.uint64)
    cnt[60:94] = _fib(34)
    assert oracle.huffman_depths(cnt).max() == 33
    lens = oracle.code_lengths(cnt, 32)
    assert lens.max() == 32
    assert kraft(lens) == 1.0
    cost = int(np.dot(cnt.astype(np.int64), lens.astype(np.int64)))
    assert cost == optimal_limited_cost(cnt, 32)
    assert cost > huffman_cost_heapq(cnt)


@pytest.mark.parametrize("m", [33, 34])
def test_32_bit_codes_on_the_stream(oracle, m):
    # codes of 32 bits inside a chunk staged by the decoder (chunk 0) and in
    # one larger than its stage (chunk 1): canonical codes prefix-free, every
    # code readable at its offset, the stream round-trips
    x = synth.fibonacci_bf16(m, seed=m)
    c = oracle.compress(0, x)
    e = (x >> 7) & 0xFF
    assert c.code_len.max() == 32
    assert c.code_len[e[:65536]].max() == 32 and c.code_len[e[65536:131072]].max() == 32
    used = [(int(c.code_len[s]), int(c.code[s])) for s in range(256) if c.code_len[s]]
    for la, ca in used:
        for lb, cb in used:
            if (la, ca) != (lb, cb) and la <= lb:
                assert (cb >> (lb - la)) != ca  # no code is a prefix of another
    off = c.chunk_bit_off.astype(np.int64)
    bits = _bits_of(c.stream, int(c.bits))
    for i in (0, 1, 65536, 65537):
        j = i // 65536
        p0 = off[j] + int(np.sum(c.code_len[e[j * 65536:i]].astype(np.int64)))
        L = int(c.code_len[e[i]])
        assert int("".join(map(str, bits[p0:p0 + L])), 2) == int(c.code[e[i]])
    assert np.array_equal(oracle.decompress(c), x)


def test_length_limit_on_stream(oracle):
    # a Fibonacci histogram forces codes longer than 8 under Lmax 32 and the
    # limit under Lmax 9; both round-trip
    fib = [1, 1]
    while len(fib) < 16:
        fib.append(fib[-1] + fib[-2])
    e = np.repeat(np.arange(16, dtype=np.uint8), fib)
    rng = np.random.default_rng(9)
    e = e[rng.permutation(e.size)]
    sm = rng.integers(0, 16, e.size, dtype=np.uint8)
    x = oracle.merge(1, e, sm)
    for lmax in (32, 9, 4):
        c = oracle.compress(1, x, chunk=1024, lmax=lmax)
        assert c.code_len.max() == min(15, lmax)
        assert np.array_equal(oracle.decompress(c), x)


def test_decoder_rejects_corruption(oracle):
    x = synth.normal_bf16(3 * 65536 + 17, seed=7)
    c = oracle.compress(0, x)

    def bad(**kw):
        d = dict(c.__dict__)
        d.update(kw)
        with pytest.raises(oracle.OracleError) as ei:
            oracle.decompress(oracle.Compressed(**d))
        assert ei.value.code == oracle.ECORRUPT

    off = c.chunk_bit_off.copy()
    off[2] += 1
    bad(chunk_bit_off=off)                       # chunk boundary moved
    bad(stream=c.stream[:-4])                    # truncated stream
    ln = c.code_len.copy()
    ln[np.argmax(ln)] = 1                        # over-subscribed code
    bad(code_len=ln)
    cd = c.code.copy()
    cd[np.nonzero(c.code_len)[0][0]] ^= 1        # not the canonical code
    bad(code=cd)


# ------------------------------------------------------- byte alphabet (FP4 scales)

def test_bytes_handworked(oracle):
    g = dict(r.split(":", 1) for r in read_golden("bytes_handworked.txt"))
    x = np.array([int(h, 16) for h in g["input_hex"].split()], np.uint8)
    c = oracle.compress(oracle.BYTES, x)
    for item in g["lengths"].split():
        s, l = item.split(":")
        assert c.code_len[int(s)] == int(l)
    for item in g["codes"].split():
        s, bits = item.split(":")
        assert format(int(c.code[int(s)]), f"0{len(bits)}b") == bits
    assert c.bits == int(g["bits"])
    assert bytes(c.stream) == bytes(int(h, 16) for h in g["stream_hex"].split())
    assert c.sign_mant.size == 0
    assert np.array_equal(oracle.decompress(c), x)


def test_bytes_every_value_roundtrip(oracle):
    rng = np.random.default_rng(3)
    x = np.tile(np.arange(256, dtype=np.uint8), 300)[rng.permutation(256 * 300)]
    e, sm = oracle.split(oracle.BYTES, x)
    assert np.array_equal(e, x) and not sm.any()
    for chunk in (1024, 65536):
        c = oracle.compress(oracle.BYTES, x, chunk=chunk)
        assert np.array_equal(oracle.decompress(c), x)


@pytest.mark.parametrize("name", list(synth.SCALE_WORKLOADS))
def test_entropy_bound_fp4_scales(oracle, name):
    _, items = synth.workload(name, scale=64)
    x = np.concatenate([v for _, v in items])
    cnt = oracle.histogram(oracle.BYTES, x)
    assert np.array_equal(cnt, np.bincount(x, minlength=256).astype(np.uint64))
    lens = oracle.code_lengths(cnt, 32)
    H = entropy_bits(cnt)
    Lbar = float(np.dot(cnt.astype(np.float64), lens)) / cnt.sum()
    assert H <= Lbar < H + 1
    # the scales are compressible (well below 8 bits per byte)
    assert Lbar < 6.0


def test_fp4_scale_generators():
    # E8M0: 2^(floor(log2 amax) - 2) stored as exponent + 127
    w = np.zeros(64, np.float32)
    w[5] = 3.0        # block 0: amax 3 -> floor(log2 3) = 1 -> 1 - 2 + 127
    w[40] = -0.25     # block 1: amax 0.25 -> -2 -> -4 + 127
    assert list(synth.mxfp4_block_scales(w)) == [126, 123]
    # E4M3 (NVFP4): amax/6 rescaled so the largest block scale is 448
    w = np.zeros(32, np.float32)
    w[0] = 6.0
    w[20] = 1.5
    s = synth.nvfp4_block_scales(w)
    vals = torch.from_numpy(s.copy()).view(torch.float8_e4m3fn).float().tolist()
    assert vals == [448.0, 112.0]


# ------------------------------------------------ fixed-slot K/V page store

def _kv_pages(n_pages=6):
    _, items = synth.workload("kv_layer", scale=64)
    return items[0][1][: n_pages * 65536]


def _smoothed_book(oracle, prefill):
    """Codebook of the prefill's counts plus one for every symbol."""
    cnt = oracle.histogram(0, prefill) + np.uint64(1)
    lens = oracle.code_lengths(cnt, 32)
    return lens, oracle.canonical_codes(lens)


def test_page_slot_equals_chunk_stream(oracle):
    k = _kv_pages()
    lens, codes = _smoothed_book(oracle, k[: 3 * 65536])
    assert lens.min() > 0 and lens.max() <= 32          # every exponent has a code
    page = k[4 * 65536: 5 * 65536]
    pg = oracle.page_encode(0, page, lens, codes, 32 * 1024)
    assert not pg.raw
    off, stream, bits = oracle.encode(0, page, 65536, lens, codes)
    assert pg.bits == bits and list(off) == [0, bits]
    assert np.array_equal(pg.slot[: stream.size], stream) and not pg.slot[stream.size:].any()
    assert np.array_equal(pg.sign_mant, oracle.pack_sm(0, page))
    assert np.array_equal(oracle.page_decode(0, 65536, lens, codes, pg), page)


def test_page_capacity_boundary(oracle):
    k = _kv_pages()
    lens, codes = _smoothed_book(oracle, k[: 3 * 65536])
    page = k[3 * 65536: 4 * 65536]
    bits = oracle.page_encode(0, page, lens, codes, 1 << 20).bits
    need = (bits + 7) // 8 + 16
    assert not oracle.page_encode(0, page, lens, codes, need).raw
    pg = oracle.page_encode(0, page, lens, codes, need - 1)
    assert pg.raw and pg.bits == 0
    assert np.array_equal(pg.raw_exps, oracle.split(0, page)[0])
    assert np.array_equal(oracle.page_decode(0, 65536, lens, codes, pg), page)


def test_page_missing_symbol_is_raw(oracle):
    k = _kv_pages()
    book = oracle.compress(0, k[: 2 * 65536])
    page = k[2 * 65536: 3 * 65536].copy()
    page[100] = 0x7F00                      # exponent 254: not in the codebook
    assert book.code_len[254] == 0
    pg = oracle.page_encode(0, page, book.code_len, book.code, 64 * 1024)
    assert pg.raw
    assert np.array_equal(oracle.page_decode(0, 65536, book.code_len, book.code, pg), page)


# ------------------------------------------------------------ stored form

def test_crc32_is_the_zlib_crc(oracle):
    import zlib
    assert oracle.crc32(b"123456789") == 0xCBF43926  # the standard check value
    rng = np.random.default_rng(5)
    for n in (0, 1, 7, 1000, 65537):
        data = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        assert oracle.crc32(data) == zlib.crc32(data)


@pytest.mark.parametrize("dtype,n,chunk,with_index", [(0, 3 * 65536 + 123, 65536, False), (1, 70001, 1024, True),
                                                       (2, 4097, 1024, False), (0, 0, 65536, False)])
def test_container_layout(oracle, dtype, n, chunk, with_index):
    """The oracle's container, parsed field by field with the layout written
    out independently here, holds the compressed arrays and their CRCs."""
    import struct
    import zlib
    if dtype == 0:
        x = synth.normal_bf16(n, seed=3)
    elif dtype == 1:
        x = synth.normal_fp8(n, seed=3)
    else:
        x = np.random.default_rng(3).integers(0, 256, n).astype(np.uint8)
    c = oracle.compress(dtype, x, chunk=chunk)
    idx = oracle.value_index(dtype, x, c.code_len, chunk=chunk) if with_index else None
    buf = oracle.container(c, idx)
    assert buf[:4] == b"EXHF"
    version, dt, lmax, ch, flags, n_, C, bits = struct.unpack_from("<HBBIIQQQ", buf, 4)
    assert (version, dt, lmax, ch, flags, n_, bits) == (1, dtype, 32, chunk, int(with_index), n, c.bits)
    assert C == -(-n // chunk)
    parts = [c.code_len.tobytes(), c.code.astype("<u4").tobytes(), c.chunk_bit_off.astype("<u8").tobytes(),
             c.stream.tobytes(), c.sign_mant.tobytes(), idx.astype("<u4").tobytes() if with_index else b""]
    pos = 192
    for i, part in enumerate(parts):
        off, ln, crc, zero = struct.unpack_from("<QQII", buf, 40 + 24 * i)
        assert (off, ln, zero) == (pos, len(part), 0)
        assert buf[off:off + ln] == part and crc == zlib.crc32(part)
        end = -(-(off + ln) // 16) * 16
        assert buf[off + ln:end] == bytes(end - off - ln)  # zero padding
        pos = end
    assert len(buf) == pos
    assert struct.unpack_from("<II", buf, 184) == (zlib.crc32(buf[:184]), 0)


# ------------------------------------------------------------ randomized
# Random tensors of the three alphabets with skewed (geometric) exponent
# distributions, random sizes, chunk sizes and code-length limits: the stored
# form must obey its definition and round-trip.

from hypothesis import HealthCheck, given, settings, strategies as st  # noqa: E402


def _skewed(dtype, n, rng):
    g = rng.geometric(0.35, n)
    if dtype == 0:
        e = np.clip(121 - g, 0, 255).astype(np.uint16)
        return ((rng.integers(0, 2, n).astype(np.uint16) << 15) | (e << 7)
                | rng.integers(0, 128, n).astype(np.uint16)).astype(np.uint16)
    if dtype == 1:
        e = np.clip(9 - g, 0, 15).astype(np.uint8)
        m = rng.integers(0, 8, n).astype(np.uint8)
        m = np.where((e == 15) & (m == 7), 6, m).astype(np.uint8)  # no NaN patterns
        return ((rng.integers(0, 2, n).astype(np.uint8) << 7) | (e << 3) | m).astype(np.uint8)
    return np.clip(100 - g, 0, 255).astype(np.uint8)


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(dtype=st.sampled_from([0, 1, 2]), n=st.integers(0, 5000), chunk=st.sampled_from([1024, 2048, 4096]),
       lmax=st.integers(8, 32), seed=st.integers(0, 2 ** 31 - 1))
def test_random_tensors(oracle, dtype, n, chunk, lmax, seed):
    x = _skewed(dtype, n, np.random.default_rng(seed))
    c = oracle.compress(dtype, x, chunk=chunk, lmax=lmax)
    lens = c.code_len.astype(np.int64)
    used = lens[lens > 0]
    assert used.size == 0 or used.max() <= lmax
    if used.size >= 2:
        assert np.sum(2.0 ** -used) == 1.0  # a complete prefix code
    # symbols and their code lengths, straight from the definition
    if dtype == 0:
        e = (x.astype(np.int64) >> 7) & 0xFF
    elif dtype == 1:
        e = (x.astype(np.int64) >> 3) & 0xF
    else:
        e = x.astype(np.int64)
    assert np.all(lens[e] > 0)
    per_value = lens[e]
    C = -(-n // chunk)
    off = c.chunk_bit_off.astype(np.int64)
    assert off.size == C + 1 and off[0] == 0
    for k in range(C):
        assert off[k + 1] - off[k] == per_value[k * chunk:(k + 1) * chunk].sum()
    assert c.bits == per_value.sum() and c.stream.size == (c.bits + 7) // 8
    # sign and mantissa, stored raw
    xi = x.astype(np.int64)
    if dtype == 0:
        assert np.array_equal(c.sign_mant, (((xi >> 8) & 0x80) | (xi & 0x7F)).astype(np.uint8))
    elif dtype == 1:
        nib = ((xi >> 4) & 0x8) | (xi & 0x7)
        nib = np.concatenate([nib, np.zeros(n % 2, np.int64)])
        assert np.array_equal(c.sign_mant, (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8))
    else:
        assert c.sign_mant.size == 0
    assert np.array_equal(oracle.decompress(c), x)
