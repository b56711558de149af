"""Fixed-slot K/V page store on the GPU against the oracle.

Pages of a K cache are coded with the codebook of earlier pages (frozen) into
fixed slots; pages that do not fit, or that hold an exponent the frozen
codebook has no code for, go to the raw pool.  Every slot (its meaningful
bytes), page record, sign/mantissa array and raw page must equal the oracle's,
and reading the pages back (in any order) must return the input bits.
"""
import numpy as np
import pytest
import torch

from exponent_entropy_coding_b200 import synth

pytestmark = pytest.mark.gpu
PAGE = 65536


@pytest.fixture(scope="module")
def eh():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from exponent_entropy_coding_b200 import build, exphuff
    build.build()
    exphuff.lib()
    return exphuff


class _Book:
    def __init__(self, code_len, code):
        self.code_len, self.code = code_len, code


def _setup(eh, oracle, n_prefill=8, n_new=24, smooth=True):
    _, items = synth.workload("kv_layer", scale=32)      # 256 tokens: 32 pages per tensor
    k = items[0][1]
    prefill, new = k[: n_prefill * PAGE], k[n_prefill * PAGE: (n_prefill + n_new) * PAGE].copy()
    p = eh.plan(0)
    if smooth:
        # frozen codebook: prefill counts plus one for every exponent
        cnt = oracle.histogram(0, prefill) + np.uint64(1)
        code_len, code = eh.codebook_from_counts(p, torch.from_numpy(cnt.view(np.int64)).cuda())
        ref = oracle.code_lengths(cnt, 32)
        assert np.array_equal(code_len.cpu().numpy(), ref)
        assert np.array_equal(code.cpu().numpy().view(np.uint32), oracle.canonical_codes(ref))
        book = _Book(code_len, code)
    else:
        new[5 * PAGE + 123] = 0x7F00                     # exponent 254, absent from the prefill
        book = eh.compress(torch.from_numpy(prefill.view(np.int16)).cuda(), p)
    return p, book, prefill, new


def _check_against_oracle(eh, oracle, store, book, new, slot_ids, dtype=0):
    lens = book.code_len.cpu().numpy()
    codes = book.code.cpu().numpy().view(np.uint32)
    meta = store.page_meta.cpu().numpy().view(np.uint32)
    slots = store.slots.cpu().numpy().reshape(store.n_slots, store.slot_bytes)
    sm = store.sign_mant.cpu().numpy().reshape(store.n_slots, PAGE if dtype == 0 else PAGE // 2)
    pool = store.raw_pool.cpu().numpy()
    n_raw = 0
    for i, s in enumerate(slot_ids):
        page = new[i * PAGE:(i + 1) * PAGE]
        ref = oracle.page_encode(dtype, page, lens, codes, store.slot_bytes)
        assert np.array_equal(sm[s], ref.sign_mant)
        if ref.raw:
            n_raw += 1
            assert meta[s] & eh.EH_PAGE_RAW
            idx = int(meta[s]) & 0x7FFFFFFF
            assert np.array_equal(pool[idx * PAGE:(idx + 1) * PAGE], ref.raw_exps)
        else:
            assert meta[s] == ref.bits
            nb = (ref.bits + 7) // 8
            assert np.array_equal(slots[s, :nb], ref.slot[:nb])
    assert int(store.raw_used.item()) == n_raw
    return n_raw


@pytest.mark.parametrize("smooth", [True, False])
def test_pages_append_and_read(eh, oracle, smooth):
    p, book, prefill, new = _setup(eh, oracle, smooth=smooth)
    n_new = new.size // PAGE
    store = eh.PageStore(p, book.code_len, book.code, n_slots=40, slot_bytes=28 * 1024, raw_cap=24,
                         device="cuda")
    rng = np.random.default_rng(0)
    slot_ids = rng.permutation(40)[:n_new]
    store.append(torch.from_numpy(new.view(np.int16)).cuda(), torch.from_numpy(slot_ids))
    assert store.status() == eh.EH_OK
    n_raw = _check_against_oracle(eh, oracle, store, book, new, slot_ids)
    assert n_raw == 0 if smooth else n_raw >= 1          # the page with exponent 254
    order = rng.permutation(n_new)
    y = store.read(torch.from_numpy(slot_ids[order]))
    want = np.concatenate([new[i * PAGE:(i + 1) * PAGE] for i in order])
    assert np.array_equal(y.cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("smooth", [True, False])
def test_pages_one_cta_per_page(eh, oracle, smooth):
    # With a 256-byte workspace (no room for the part totals) every page is
    # coded by one CTA; slots, records and raw pages must be the same.
    p, book, prefill, new = _setup(eh, oracle, smooth=smooth)
    n_new = new.size // PAGE
    store = eh.PageStore(p, book.code_len, book.code, n_slots=40, slot_bytes=28 * 1024, raw_cap=24,
                         device="cuda")
    read_ws = store.workspace
    store.workspace = torch.empty(256, dtype=torch.uint8, device="cuda")
    slot_ids = np.random.default_rng(2).permutation(40)[:n_new]
    store.append(torch.from_numpy(new.view(np.int16)).cuda(), torch.from_numpy(slot_ids))
    assert store.status() == eh.EH_OK
    n_raw = _check_against_oracle(eh, oracle, store, book, new, slot_ids)
    assert n_raw == 0 if smooth else n_raw >= 1
    store.workspace = read_ws
    y = store.read(torch.from_numpy(slot_ids))
    assert np.array_equal(y.cpu().numpy().view(np.uint16), new)


def test_prepared_tables(eh, oracle):
    # The frozen codebook's decode tables built once (eh_pages_prepare) serve
    # every later read (eh_pages_read_prepared), in any page order; tables
    # prepared from an invalid codebook make reads report corruption.
    p, book, prefill, new = _setup(eh, oracle, n_new=12)
    store = eh.PageStore(p, book.code_len, book.code, n_slots=16, slot_bytes=28 * 1024, raw_cap=4,
                         device="cuda")
    slot_ids = np.random.default_rng(5).permutation(16)[:12]
    store.append(torch.from_numpy(new.view(np.int16)).cuda(), torch.from_numpy(slot_ids))
    assert store.status() == eh.EH_OK
    store.prepare()
    rng = np.random.default_rng(6)
    for _ in range(3):
        order = rng.permutation(12)[: rng.integers(1, 13)]
        y = store.read(torch.from_numpy(slot_ids[order]))
        want = np.concatenate([new[i * PAGE:(i + 1) * PAGE] for i in order])
        assert np.array_equal(y.cpu().numpy().view(np.uint16), want)
    good = store.code_len
    store.code_len = torch.ones_like(good)  # every symbol 1 bit long: Kraft sum far above 1
    store.prepare()
    store.code_len = good
    store.read(torch.from_numpy(slot_ids[:2]), check=False)
    assert store.status() == eh.EH_ERR_CORRUPT


def test_small_slots_go_raw(eh, oracle):
    p, book, prefill, new = _setup(eh, oracle, n_new=8)
    store = eh.PageStore(p, book.code_len, book.code, n_slots=8, slot_bytes=16 * 1024, raw_cap=8,
                         device="cuda")
    slot_ids = np.arange(8)
    store.append(torch.from_numpy(new.view(np.int16)).cuda(), torch.from_numpy(slot_ids))
    assert store.status() == eh.EH_OK
    assert _check_against_oracle(eh, oracle, store, book, new, slot_ids) == 8
    y = store.read(torch.from_numpy(slot_ids))
    assert np.array_equal(y.cpu().numpy().view(np.uint16), new)


def test_raw_pool_exhaustion_is_reported(eh, oracle):
    p, book, prefill, new = _setup(eh, oracle, n_new=6)
    store = eh.PageStore(p, book.code_len, book.code, n_slots=6, slot_bytes=16 * 1024, raw_cap=2,
                         device="cuda")
    store.append(torch.from_numpy(new.view(np.int16)).cuda(), torch.arange(6, dtype=torch.int32))
    assert store.status() == eh.EH_ERR_NOMEM
    y = store.read(torch.arange(6, dtype=torch.int32), check=False)
    assert store.status() == eh.EH_ERR_CORRUPT


def _fp8_cache(n_pages, seed):
    """FP8 E4M3 K/V-like values: normal with standard deviation 20, so that no
    value reaches 256 (exponent field 15) while subnormals occur."""
    w = np.random.default_rng(seed).standard_normal(n_pages * PAGE).astype(np.float32) * np.float32(20.0)
    return synth.to_fp8_e4m3_bits(w)


@pytest.mark.parametrize("smooth", [True, False])
def test_fp8_pages_append_and_read(eh, oracle, smooth):
    """The page store with FP8 E4M3 pages (16-symbol exponent alphabet,
    sign/mantissa nibbles packed two per byte)."""
    prefill, new = _fp8_cache(6, 11), _fp8_cache(20, 12)
    assert not ((prefill >> 3) & 0xF == 15).any()
    p = eh.plan(eh.EH_FP8_E4M3)
    if smooth:
        cnt = oracle.histogram(1, prefill) + np.uint64(1)
        code_len, code = eh.codebook_from_counts(p, torch.from_numpy(cnt.view(np.int64)).cuda())
        assert np.array_equal(code_len.cpu().numpy(), oracle.code_lengths(cnt, 32))
        book = _Book(code_len, code)
    else:
        new[7 * PAGE + 4321] = 0x78                     # 256.0: exponent 15, absent from the prefill
        book = eh.compress(torch.from_numpy(prefill).cuda(), p)
    n_new = new.size // PAGE
    # pages code to 21.15 - 21.30 KB (2.6 bits per exponent): with 21,248-byte
    # slots some fit and some go to the raw pool
    store = eh.PageStore(p, book.code_len, book.code, n_slots=32, slot_bytes=21248, raw_cap=n_new,
                         device="cuda")
    rng = np.random.default_rng(1)
    slot_ids = rng.permutation(32)[:n_new]
    store.append(torch.from_numpy(new).cuda(), torch.from_numpy(slot_ids))
    assert store.status() == eh.EH_OK
    n_raw = _check_against_oracle(eh, oracle, store, book, new, slot_ids, dtype=1)
    assert 0 < n_raw < n_new
    order = rng.permutation(n_new)
    y = store.read(torch.from_numpy(slot_ids[order]))
    want = np.concatenate([new[i * PAGE:(i + 1) * PAGE] for i in order])
    assert np.array_equal(y.cpu().numpy(), want)
