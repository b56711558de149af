"""ctypes wrapper around the CPU oracle (libehref.so).

Test infrastructure only.  Inputs and outputs are numpy arrays of raw bit
patterns: uint16 for BF16, uint8 for FP8 E4M3.  Errors raise OracleError with
the oracle's code.
"""
import ctypes as C
from dataclasses import dataclass

import numpy as np

from . import build as _build

BF16 = 0
FP8_E4M3 = 1
BYTES = 2

OK, EINVAL, EINFEASIBLE, ECAPACITY, ECORRUPT = 0, -1, -2, -3, -4
_NAMES = {EINVAL: "EINVAL", EINFEASIBLE: "EINFEASIBLE", ECAPACITY: "ECAPACITY",
          ECORRUPT: "ECORRUPT"}


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle returned {_NAMES.get(code, code)}")
        self.code = code


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(_build.build())
        u64, i32, u32, vp = C.c_uint64, C.c_int, C.c_uint32, C.c_void_p
        sig = {
            "ehref_alphabet": (i32, [i32]),
            "ehref_split": (i32, [i32, vp, u64, vp, vp]),
            "ehref_merge": (i32, [i32, vp, vp, u64, vp]),
            "ehref_histogram": (i32, [i32, vp, u64, vp]),
            "ehref_huffman_depths": (i32, [vp, i32, vp]),
            "ehref_package_merge": (i32, [vp, i32, i32, vp]),
            "ehref_code_lengths": (i32, [vp, i32, i32, vp]),
            "ehref_canonical_codes": (i32, [vp, i32, vp]),
            "ehref_sm_bytes": (u64, [i32, u64]),
            "ehref_pack_sm": (i32, [i32, vp, u64, vp]),
            "ehref_num_chunks": (u64, [u64, u32]),
            "ehref_encode": (i32, [i32, vp, u64, u32, vp, vp, vp, vp, u64, vp]),
            "ehref_compress": (i32, [i32, vp, u64, u32, i32, vp, vp, vp, vp, u64, vp, vp]),
            "ehref_decompress_chunks": (i32, [i32, u64, u32, vp, vp, vp, vp, u64, vp, u32, u32, vp]),
            "ehref_decompress": (i32, [i32, u64, u32, vp, vp, vp, vp, u64, vp, vp]),
            "ehref_page_encode": (i32, [i32, vp, u64, vp, vp, vp, u64, vp, vp, vp, vp]),
            "ehref_page_decode": (i32, [i32, u64, vp, vp, vp, u64, u64, i32, vp, vp, vp]),
            "ehref_value_index": (i32, [i32, vp, u64, u32, vp, vp]),
            "ehref_container_write": (i32, [i32, u64, u32, i32, vp, vp, vp, vp, u64, vp, vp, vp, u64, vp]),
            "ehref_crc32": (u32, [vp, u64]),
            "zfref_blocks": (u64, [u64]),
            "zfref_block_base": (i32, [vp, u32, vp, vp]),
            "zfref_compress": (i32, [vp, u64, vp, vp, vp, vp, vp, u64, vp]),
            "zfref_decompress": (i32, [u64, vp, vp, vp, vp, vp, u64, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(_lib, name)
            f.restype = res
            f.argtypes = args
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _check(rc):
    if rc != OK:
        raise OracleError(rc)


def elem_dtype(dtype):
    return np.uint16 if dtype == BF16 else np.uint8


def alphabet(dtype):
    return lib().ehref_alphabet(dtype)


def split(dtype, x):
    x = np.ascontiguousarray(x, dtype=elem_dtype(dtype))
    e = np.empty(x.size, np.uint8)
    sm = np.empty(x.size, np.uint8)
    _check(lib().ehref_split(dtype, _p(x), x.size, _p(e), _p(sm)))
    return e, sm


def merge(dtype, e, sm):
    e = np.ascontiguousarray(e, np.uint8)
    sm = np.ascontiguousarray(sm, np.uint8)
    out = np.empty(e.size, elem_dtype(dtype))
    _check(lib().ehref_merge(dtype, _p(e), _p(sm), e.size, _p(out)))
    return out


def histogram(dtype, x):
    x = np.ascontiguousarray(x, dtype=elem_dtype(dtype))
    cnt = np.zeros(alphabet(dtype), np.uint64)
    _check(lib().ehref_histogram(dtype, _p(x), x.size, _p(cnt)))
    return cnt


def huffman_depths(cnt):
    cnt = np.ascontiguousarray(cnt, np.uint64)
    d = np.zeros(cnt.size, np.uint8)
    rc = lib().ehref_huffman_depths(_p(cnt), cnt.size, _p(d))
    if rc < 0:
        raise OracleError(rc)
    return d


def package_merge(cnt, lmax):
    cnt = np.ascontiguousarray(cnt, np.uint64)
    ln = np.zeros(cnt.size, np.uint8)
    _check(lib().ehref_package_merge(_p(cnt), cnt.size, lmax, _p(ln)))
    return ln


def code_lengths(cnt, lmax=32):
    cnt = np.ascontiguousarray(cnt, np.uint64)
    ln = np.zeros(cnt.size, np.uint8)
    _check(lib().ehref_code_lengths(_p(cnt), cnt.size, lmax, _p(ln)))
    return ln


def canonical_codes(lengths):
    ln = np.ascontiguousarray(lengths, np.uint8)
    code = np.zeros(ln.size, np.uint32)
    _check(lib().ehref_canonical_codes(_p(ln), ln.size, _p(code)))
    return code


def sm_bytes(dtype, n):
    return lib().ehref_sm_bytes(dtype, n)


def pack_sm(dtype, x):
    x = np.ascontiguousarray(x, dtype=elem_dtype(dtype))
    out = np.empty(sm_bytes(dtype, x.size), np.uint8)
    _check(lib().ehref_pack_sm(dtype, _p(x), x.size, _p(out)))
    return out


def num_chunks(n, chunk):
    return lib().ehref_num_chunks(n, chunk)


@dataclass
class Compressed:
    dtype: int
    n: int
    chunk: int
    lmax: int
    code_len: np.ndarray     # uint8[A]
    code: np.ndarray         # uint32[A]
    chunk_bit_off: np.ndarray  # uint64[C+1]
    stream: np.ndarray       # uint8[ceil(bits/8)]
    sign_mant: np.ndarray    # uint8[n or ceil(n/2)]
    bits: int


def encode(dtype, x, chunk, lengths, codes):
    x = np.ascontiguousarray(x, dtype=elem_dtype(dtype))
    n = x.size
    ln = np.ascontiguousarray(lengths, np.uint8)
    cd = np.ascontiguousarray(codes, np.uint32)
    nc = num_chunks(n, chunk)
    off = np.zeros(nc + 1, np.uint64)
    cap = (n * 32 + 7) // 8
    stream = np.zeros(max(cap, 1), np.uint8)
    bits = C.c_uint64(0)
    _check(lib().ehref_encode(dtype, _p(x), n, chunk, _p(ln), _p(cd), _p(off), _p(stream),
                              cap, C.byref(bits)))
    return off, stream[: (bits.value + 7) // 8].copy(), bits.value


INDEX_STRIDE = 128


def value_index(dtype, x, lengths, chunk=65536):
    """Bit offset of every INDEX_STRIDE-th value of each chunk (format in ehref.h)."""
    x = np.ascontiguousarray(x, dtype=elem_dtype(dtype))
    nc = num_chunks(x.size, chunk)
    idx = np.zeros(max(nc * (chunk // INDEX_STRIDE), 1), np.uint32)
    _check(lib().ehref_value_index(dtype, _p(x), x.size, chunk,
                                   _p(np.ascontiguousarray(lengths, np.uint8)), _p(idx)))
    return idx[: nc * (chunk // INDEX_STRIDE)]


def compress(dtype, x, chunk=65536, lmax=32):
    x = np.ascontiguousarray(x, dtype=elem_dtype(dtype))
    n = x.size
    A = alphabet(dtype)
    ln = np.zeros(A, np.uint8)
    code = np.zeros(A, np.uint32)
    nc = num_chunks(n, chunk)
    off = np.zeros(nc + 1, np.uint64)
    cap = (n * lmax + 7) // 8
    stream = np.zeros(max(cap, 1), np.uint8)
    sm = np.zeros(max(sm_bytes(dtype, n), 1), np.uint8)
    bits = C.c_uint64(0)
    _check(lib().ehref_compress(dtype, _p(x), n, chunk, lmax, _p(ln), _p(code), _p(off),
                                _p(stream), cap, _p(sm), C.byref(bits)))
    return Compressed(dtype, n, chunk, lmax, ln, code, off,
                      stream[: (bits.value + 7) // 8].copy(),
                      sm[: sm_bytes(dtype, n)].copy(), bits.value)


def container(c: Compressed, index=None) -> bytes:
    """The stored form (ehref.h) of a compressed tensor; `index` is its
    optional value index (uint32 array)."""
    args = [c.dtype, c.n, c.chunk, c.lmax, _p(np.ascontiguousarray(c.code_len, np.uint8)),
            _p(np.ascontiguousarray(c.code, np.uint32)), _p(np.ascontiguousarray(c.chunk_bit_off, np.uint64)),
            _p(np.ascontiguousarray(c.stream, np.uint8)), c.bits, _p(np.ascontiguousarray(c.sign_mant, np.uint8)),
            _p(np.ascontiguousarray(index, np.uint32)) if index is not None else None]
    size = C.c_uint64(0)
    _check(lib().ehref_container_write(*args, None, 0, C.byref(size)))
    out = np.zeros(size.value, np.uint8)
    _check(lib().ehref_container_write(*args, _p(out), out.size, C.byref(size)))
    return out.tobytes()


def crc32(data: bytes) -> int:
    a = np.frombuffer(data, np.uint8)
    return int(lib().ehref_crc32(_p(np.ascontiguousarray(a)), a.size))


def decompress(c: Compressed, first=None, count=None):
    nc = num_chunks(c.n, c.chunk)
    if first is None:
        first, count = 0, nc
    i0 = first * c.chunk
    i1 = min(c.n, (first + count) * c.chunk)
    out = np.zeros(max(i1 - i0, 0), elem_dtype(c.dtype))
    stream = np.ascontiguousarray(c.stream, np.uint8)
    _check(lib().ehref_decompress_chunks(
        c.dtype, c.n, c.chunk, _p(np.ascontiguousarray(c.code_len, np.uint8)),
        _p(np.ascontiguousarray(c.code, np.uint32)),
        _p(np.ascontiguousarray(c.chunk_bit_off, np.uint64)), _p(stream), stream.size,
        _p(np.ascontiguousarray(c.sign_mant, np.uint8)), first, count, _p(out)))
    return out


@dataclass
class Page:
    slot: np.ndarray       # uint8[slot_bytes] (zero beyond the codes)
    bits: int
    raw: bool
    raw_exps: np.ndarray   # uint8[n] when raw
    sign_mant: np.ndarray


def page_encode(dtype, x, lengths, codes, slot_bytes):
    x = np.ascontiguousarray(x, dtype=elem_dtype(dtype))
    n = x.size
    slot = np.zeros(slot_bytes, np.uint8)
    sm = np.zeros(max(sm_bytes(dtype, n), 1), np.uint8)
    raw_exps = np.zeros(max(n, 1), np.uint8)
    bits = C.c_uint64(0)
    raw = C.c_int(0)
    _check(lib().ehref_page_encode(dtype, _p(x), n, _p(np.ascontiguousarray(lengths, np.uint8)),
                                   _p(np.ascontiguousarray(codes, np.uint32)), _p(slot), slot_bytes,
                                   _p(sm), _p(raw_exps), C.byref(bits), C.byref(raw)))
    return Page(slot, bits.value, bool(raw.value), raw_exps[:n], sm[:sm_bytes(dtype, n)])


def page_decode(dtype, n, lengths, codes, page: Page):
    out = np.zeros(max(n, 1), elem_dtype(dtype))
    _check(lib().ehref_page_decode(dtype, n, _p(np.ascontiguousarray(lengths, np.uint8)),
                                   _p(np.ascontiguousarray(codes, np.uint32)), _p(page.slot),
                                   page.slot.size, page.bits, int(page.raw),
                                   _p(np.ascontiguousarray(page.raw_exps, np.uint8)),
                                   _p(np.ascontiguousarray(page.sign_mant, np.uint8)), _p(out)))
    return out[:n]


# ---- ZipFloat comparison codec (BF16 only; format in zfref.h)
ZF_BLOCK = 2048


@dataclass
class ZfCompressed:
    n: int
    sign_mant: np.ndarray   # uint8[n]
    meta: np.ndarray        # uint32[B]: l_b | records << 8
    dense: np.ndarray       # uint32[B*192]: 3 bit planes of 64 words per block
    sparse_off: np.ndarray  # uint32[B]
    sparse: np.ndarray      # uint16[records]

    def nbytes(self):
        return self.sign_mant.size + 4 * self.meta.size + 4 * self.dense.size + 4 * self.sparse_off.size + \
            2 * self.sparse.size


def zf_blocks(n):
    return lib().zfref_blocks(n)


def zf_block_base(x):
    x = np.ascontiguousarray(x, np.uint16)
    md, lb = C.c_uint32(0), C.c_uint32(0)
    _check(lib().zfref_block_base(_p(x), x.size, C.byref(md), C.byref(lb)))
    return md.value, lb.value


def zf_compress(x):
    x = np.ascontiguousarray(x, np.uint16)
    n = x.size
    B = zf_blocks(n)
    sm = np.zeros(max(n, 1), np.uint8)
    meta = np.zeros(max(B, 1), np.uint32)
    dense = np.zeros(max(B * 192, 1), np.uint32)
    off = np.zeros(max(B, 1), np.uint32)
    sparse = np.zeros(max(n, 1), np.uint16)
    nrec = C.c_uint64(0)
    _check(lib().zfref_compress(_p(x), n, _p(sm), _p(meta), _p(dense), _p(off), _p(sparse), n, C.byref(nrec)))
    return ZfCompressed(n, sm[:n], meta[:B], dense[:B * 192], off[:B], sparse[:nrec.value].copy())


def zf_decompress(c: ZfCompressed):
    out = np.zeros(max(c.n, 1), np.uint16)
    sp = np.ascontiguousarray(c.sparse, np.uint16)
    _check(lib().zfref_decompress(c.n, _p(np.ascontiguousarray(c.sign_mant, np.uint8)),
                                  _p(np.ascontiguousarray(c.meta, np.uint32)),
                                  _p(np.ascontiguousarray(c.dense, np.uint32)),
                                  _p(np.ascontiguousarray(c.sparse_off, np.uint32)),
                                  _p(sp) if sp.size else None, sp.size, _p(out)))
    return out[:c.n]
