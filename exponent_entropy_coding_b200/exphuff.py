"""Python binding of libexphuff (include/exphuff.h).

Argument marshalling only: every step of compression and decompression runs
in the library's CUDA kernels.  PyTorch provides device memory and streams.
The library must have been built (``python -m exponent_entropy_coding_b200.build``
or ``__graft_entry__.build()``); if it is missing, loading raises instead of
falling back to anything else.
"""
import ctypes as C
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libexphuff.so")

EH_BF16 = 0
EH_FP8_E4M3 = 1
EH_BYTES = 2     # every byte a symbol, no sign/mantissa (FP4 block scale factors)
EH_DEFAULT_CHUNK_ELEMS = 65536
EH_MAX_CODE_LEN = 32
EH_MAX_BATCH = 16
EH_NOALLOC_MAX_BATCH = 8

STATUS = {0: "EH_OK", 1: "EH_ERR_INVALID_ARG", 2: "EH_ERR_UNSUPPORTED", 3: "EH_ERR_INFEASIBLE",
          4: "EH_ERR_CUDA", 5: "EH_ERR_CORRUPT", 6: "EH_ERR_TIMEOUT", 7: "EH_ERR_NOMEM"}
EH_OK, EH_ERR_INVALID_ARG, EH_ERR_UNSUPPORTED, EH_ERR_INFEASIBLE = 0, 1, 2, 3
EH_ERR_CUDA, EH_ERR_CORRUPT, EH_ERR_TIMEOUT, EH_ERR_NOMEM = 4, 5, 6, 7

EXPORTED = ["eh_plan", "eh_compress_bound", "eh_compress_batch_workspace", "eh_compress",
            "eh_compress_batch", "eh_compress_shard_begin", "eh_compress_shard_finish",
            "eh_decompress_workspace", "eh_decompress", "eh_decompress_batch",
            "eh_decompress_chunks", "eh_decompress_batch_noalloc", "eh_codebook_from_counts",
            "eh_pages_append", "eh_pages_read", "eh_pages_prepare", "eh_pages_read_prepared",
            "eh_prefetch_workspace", "eh_prefetch_create", "eh_prefetch_submit",
            "eh_prefetch_acquire", "eh_prefetch_release", "eh_prefetch_status",
            "eh_prefetch_destroy",
            "eh_zf_bound", "eh_zf_compress", "eh_zf_decompress",
            "eh_get_status", "eh_status_str", "eh_version", "eh_debug_set_fixup_rounds",
            "eh_container_size", "eh_container_write", "eh_container_read"]
EH_PREFETCH_MAX_DEPTH = 8
EH_PAGE_RAW = 0x80000000


class EhError(RuntimeError):
    def __init__(self, code, what=""):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}")


class eh_plan_t(C.Structure):
    _fields_ = [("dtype", C.c_int32), ("chunk_elems", C.c_uint32),
                ("max_code_len", C.c_uint32), ("reserved", C.c_uint32)]


class eh_compressed_t(C.Structure):
    _fields_ = [("dtype", C.c_int32), ("n_chunks", C.c_uint32), ("n", C.c_uint64),
                ("code_len", C.c_void_p), ("code", C.c_void_p), ("chunk_bit_off", C.c_void_p),
                ("exp_stream", C.c_void_p), ("exp_stream_cap", C.c_uint64),
                ("sign_mant", C.c_void_p), ("exp_stream_bits", C.c_uint64),
                ("value_index", C.c_void_p)]


class eh_zf_t(C.Structure):
    _fields_ = [("n", C.c_uint64), ("sign_mant", C.c_void_p), ("meta", C.c_void_p), ("dense", C.c_void_p),
                ("sparse_off", C.c_void_p), ("sparse", C.c_void_p), ("sparse_cap", C.c_uint64),
                ("n_records", C.c_uint64)]


class eh_page_store_t(C.Structure):
    _fields_ = [("code_len", C.c_void_p), ("code", C.c_void_p), ("slots", C.c_void_p),
                ("slot_bytes", C.c_uint64), ("n_slots", C.c_uint32), ("raw_cap", C.c_uint32),
                ("sign_mant", C.c_void_p), ("page_meta", C.c_void_p), ("raw_pool", C.c_void_p),
                ("raw_used", C.c_void_p)]


_lib = None


def lib():
    """Loads libexphuff.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libexphuff.so not built ({LIB_PATH}); run "
                               "python -m exponent_entropy_coding_b200.build")
        L = C.CDLL(LIB_PATH)
        P, u64, i32, u32, vp = C.POINTER, C.c_uint64, C.c_int32, C.c_uint32, C.c_void_p
        sig = {
            "eh_plan": [P(eh_plan_t), i32, u32, u32],
            "eh_compress_bound": [P(eh_plan_t), u64, P(u64), P(u64), P(u64)],
            "eh_compress_batch_workspace": [P(eh_plan_t), C.c_int, P(u64), P(u64)],
            "eh_compress": [P(eh_plan_t), vp, u64, P(eh_compressed_t), vp, u64, vp],
            "eh_compress_batch": [P(eh_plan_t), C.c_int, P(vp), P(eh_compressed_t), vp, vp, u64, vp],
            "eh_compress_shard_begin": [P(eh_plan_t), vp, P(eh_compressed_t), vp, vp, u64, vp],
            "eh_compress_shard_finish": [P(eh_plan_t), vp, P(eh_compressed_t), vp, vp, vp, u64, vp],
            "eh_decompress_workspace": [P(eh_plan_t), C.c_int, P(u64)],
            "eh_decompress": [P(eh_plan_t), P(eh_compressed_t), vp, vp, u64, vp],
            "eh_decompress_batch": [P(eh_plan_t), C.c_int, P(eh_compressed_t), P(vp), vp, u64, vp],
            "eh_decompress_chunks": [P(eh_plan_t), P(eh_compressed_t), u32, u32, vp, vp, u64, vp],
            "eh_decompress_batch_noalloc": [P(eh_plan_t), C.c_int, P(eh_compressed_t), P(vp), vp],
            "eh_debug_set_fixup_rounds": [u32],
            "eh_container_size": [P(eh_plan_t), u64, u64, C.c_int, P(u64)],
            "eh_container_write": [P(eh_plan_t), P(eh_compressed_t), vp, u64],
            "eh_container_read": [vp, u64, P(eh_plan_t), P(eh_compressed_t)],
            "eh_codebook_from_counts": [P(eh_plan_t), vp, vp, vp, vp, u64, vp],
            "eh_pages_append": [P(eh_plan_t), P(eh_page_store_t), vp, u32, vp, vp, u64, vp],
            "eh_pages_read": [P(eh_plan_t), P(eh_page_store_t), vp, u32, vp, vp, u64, vp],
            "eh_pages_prepare": [P(eh_plan_t), P(eh_page_store_t), vp, u64, vp],
            "eh_pages_read_prepared": [P(eh_plan_t), P(eh_page_store_t), vp, vp, u32, vp, vp, u64, vp],
            "eh_prefetch_workspace": [P(eh_plan_t), C.c_int, P(u64)],
            "eh_prefetch_create": [P(eh_plan_t), C.c_int, P(vp), u64, vp, u64, vp, u32, P(vp)],
            "eh_prefetch_submit": [vp, C.c_int, P(eh_compressed_t), P(u64), P(C.c_int)],
            "eh_prefetch_acquire": [vp, C.c_int, vp],
            "eh_prefetch_release": [vp, C.c_int, vp],
            "eh_prefetch_status": [vp, C.c_int],
            "eh_prefetch_destroy": [vp],
            "eh_zf_bound": [u64, P(u64), P(u64)],
            "eh_zf_compress": [vp, P(eh_zf_t), vp, u64, C.c_int, vp],
            "eh_zf_decompress": [P(eh_zf_t), vp, vp, u64, vp],
            "eh_get_status": [vp, vp],
            "eh_status_str": [C.c_int],
            "eh_version": [],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = C.c_char_p if name in ("eh_status_str", "eh_version") else C.c_int
        _lib = L
    return _lib


def _check(rc, what):
    if rc != EH_OK:
        raise EhError(rc, what)


def _stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def dtype_code(torch_dtype) -> int:
    if torch_dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return EH_BF16
    if torch_dtype in (torch.float8_e4m3fn, torch.uint8):
        return EH_FP8_E4M3
    raise ValueError(f"unsupported dtype {torch_dtype}")


def alphabet(dtype: int) -> int:
    return 16 if dtype == EH_FP8_E4M3 else 256


def plan(dtype: int, chunk_elems: int = 0, max_code_len: int = 0) -> eh_plan_t:
    p = eh_plan_t()
    _check(lib().eh_plan(C.byref(p), dtype, chunk_elems, max_code_len), "eh_plan")
    return p


def compress_bound(p: eh_plan_t, n: int):
    sc, sm, ws = C.c_uint64(), C.c_uint64(), C.c_uint64()
    _check(lib().eh_compress_bound(C.byref(p), n, C.byref(sc), C.byref(sm), C.byref(ws)),
           "eh_compress_bound")
    return sc.value, sm.value, ws.value


def compress_batch_workspace(p: eh_plan_t, ns: Sequence[int]) -> int:
    arr = (C.c_uint64 * len(ns))(*ns)
    out = C.c_uint64()
    _check(lib().eh_compress_batch_workspace(C.byref(p), len(ns), arr, C.byref(out)),
           "eh_compress_batch_workspace")
    return out.value


def decompress_workspace(p: eh_plan_t, k: int = 1) -> int:
    out = C.c_uint64()
    _check(lib().eh_decompress_workspace(C.byref(p), k, C.byref(out)), "eh_decompress_workspace")
    return out.value


@dataclass
class Compressed:
    """Device arrays of one compressed tensor (torch tensors own the memory)."""
    dtype: int
    n: int
    code_len: torch.Tensor       # uint8[A]
    code: torch.Tensor           # int32[A] (uint32 values)
    chunk_bit_off: torch.Tensor  # int64[C+1] (uint64 values)
    exp_stream: torch.Tensor     # uint8[cap]
    sign_mant: torch.Tensor      # uint8[n or ceil(n/2)]
    exp_stream_bits: int = 0
    value_index: Optional[torch.Tensor] = None  # int32[C * chunk / 128] (uint32 values) or None

    @property
    def n_chunks(self) -> int:
        return self.chunk_bit_off.numel() - 1

    def stream_bytes(self) -> int:
        return (self.exp_stream_bits + 7) // 8

    def compressed_bytes(self) -> int:
        """Stored size: exponent stream + sign/mantissa + offsets + codebook
        (+ the value index when there is one)."""
        return (self.stream_bytes() + self.sign_mant.numel() + 8 * self.chunk_bit_off.numel()
                + self.code_len.numel() + (4 * self.value_index.numel() if self.value_index is not None else 0))

    def struct(self) -> eh_compressed_t:
        s = eh_compressed_t()
        s.dtype = self.dtype
        s.n_chunks = self.n_chunks
        s.n = self.n
        s.code_len = self.code_len.data_ptr()
        s.code = self.code.data_ptr()
        s.chunk_bit_off = self.chunk_bit_off.data_ptr()
        s.exp_stream = self.exp_stream.data_ptr() if self.exp_stream.numel() else None
        s.exp_stream_cap = self.exp_stream.numel()
        s.sign_mant = self.sign_mant.data_ptr() if self.sign_mant.numel() else None
        s.exp_stream_bits = self.exp_stream_bits
        s.value_index = self.value_index.data_ptr() if self.value_index is not None else None
        return s


EH_INDEX_STRIDE = 128


def alloc_compressed(p: eh_plan_t, n: int, device, index: bool = False) -> Compressed:
    """Buffers for one compressed tensor; `index` adds the optional value
    index (4 bytes per EH_INDEX_STRIDE values)."""
    cap, smb, _ = compress_bound(p, n)
    A = alphabet(p.dtype)
    nc = -(-n // p.chunk_elems)
    dev = torch.device(device)
    return Compressed(
        dtype=p.dtype, n=n,
        code_len=torch.zeros(A, dtype=torch.uint8, device=dev),
        code=torch.zeros(A, dtype=torch.int32, device=dev),
        chunk_bit_off=torch.zeros(nc + 1, dtype=torch.int64, device=dev),
        exp_stream=torch.empty(cap if n else 0, dtype=torch.uint8, device=dev),
        sign_mant=torch.empty(smb, dtype=torch.uint8, device=dev),
        value_index=(torch.zeros(max(nc * (p.chunk_elems // EH_INDEX_STRIDE), 1), dtype=torch.int32, device=dev)
                     if index else None))


def _raw(x: torch.Tensor) -> torch.Tensor:
    if not x.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    return x.contiguous()


def compress_batch(p: eh_plan_t, xs: List[torch.Tensor], outs: List[Compressed], workspace: torch.Tensor,
                   bits_dev: Optional[torch.Tensor] = None, stream=None):
    """Calls eh_compress_batch on device tensors; fills outs[i].exp_stream_bits
    unless bits_dev (int64[k] on the device) is given."""
    k = len(xs)
    xs = [_raw(x) for x in xs]
    ins = (C.c_void_p * k)(*[x.data_ptr() if x.numel() else None for x in xs])
    structs = (eh_compressed_t * k)(*[o.struct() for o in outs])
    rc = lib().eh_compress_batch(C.byref(p), k, ins, structs,
                                 C.c_void_p(bits_dev.data_ptr()) if bits_dev is not None else None,
                                 C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream))
    _check(rc, "eh_compress_batch")
    if bits_dev is None:
        for o, s in zip(outs, structs):
            o.exp_stream_bits = s.exp_stream_bits
    return outs


def compress(x: torch.Tensor, p: Optional[eh_plan_t] = None, workspace: Optional[torch.Tensor] = None,
             stream=None, index: bool = False) -> Compressed:
    """Compresses one BF16 / FP8 E4M3 tensor (or its raw uint16 / uint8 bits);
    `index` also writes the optional value index."""
    x = _raw(x)
    if p is None:
        p = plan(dtype_code(x.dtype))
    n = x.numel()
    out = alloc_compressed(p, n, x.device, index=index)
    if workspace is None:
        workspace = torch.empty(compress_bound(p, n)[2], dtype=torch.uint8, device=x.device)
    s = out.struct()
    rc = lib().eh_compress(C.byref(p), C.c_void_p(x.data_ptr()) if n else None, n, C.byref(s),
                           C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream))
    _check(rc, "eh_compress")
    out.exp_stream_bits = s.exp_stream_bits
    return out


def compress_shard_begin(x: torch.Tensor, out: Compressed, counts: torch.Tensor, p: eh_plan_t,
                         workspace: torch.Tensor, stream=None):
    """Step 1 of sharded compression: local exponent counts (int64[A] on the
    device, uint64 values) and packed sign/mantissa of the shard."""
    x = _raw(x)
    s = out.struct()
    rc = lib().eh_compress_shard_begin(C.byref(p), C.c_void_p(x.data_ptr()) if x.numel() else None,
                                       C.byref(s), C.c_void_p(counts.data_ptr()),
                                       C.c_void_p(workspace.data_ptr()), workspace.numel(),
                                       _stream_ptr(stream))
    _check(rc, "eh_compress_shard_begin")


def compress_shard_finish(x: torch.Tensor, out: Compressed, counts: torch.Tensor, p: eh_plan_t,
                          workspace: torch.Tensor, bits_dev: Optional[torch.Tensor] = None, stream=None):
    """Step 2: codebook from the summed counts, shard offsets and stream."""
    x = _raw(x)
    s = out.struct()
    rc = lib().eh_compress_shard_finish(C.byref(p), C.c_void_p(x.data_ptr()) if x.numel() else None,
                                        C.byref(s), C.c_void_p(counts.data_ptr()),
                                        C.c_void_p(bits_dev.data_ptr()) if bits_dev is not None else None,
                                        C.c_void_p(workspace.data_ptr()), workspace.numel(),
                                        _stream_ptr(stream))
    _check(rc, "eh_compress_shard_finish")
    if bits_dev is None:
        out.exp_stream_bits = s.exp_stream_bits
    return out


def _elem_dtype(dtype):
    return torch.int16 if dtype == EH_BF16 else torch.uint8


def decompress_batch(p: eh_plan_t, cs: List[Compressed], outs: List[torch.Tensor], workspace: torch.Tensor,
                     stream=None):
    k = len(cs)
    structs = (eh_compressed_t * k)(*[c.struct() for c in cs])
    optrs = (C.c_void_p * k)(*[o.data_ptr() if o.numel() else None for o in outs])
    rc = lib().eh_decompress_batch(C.byref(p), k, structs, optrs, C.c_void_p(workspace.data_ptr()),
                                   workspace.numel(), _stream_ptr(stream))
    _check(rc, "eh_decompress_batch")
    return outs


def decompress_batch_noalloc(p: eh_plan_t, cs: List[Compressed], outs: List[torch.Tensor], stream=None) -> int:
    """Block decompression with the library's fixed scratch (no workspace, no
    allocation); waits for the stream and returns the call's status code."""
    k = len(cs)
    structs = (eh_compressed_t * k)(*[c.struct() for c in cs])
    optrs = (C.c_void_p * k)(*[o.data_ptr() if o.numel() else None for o in outs])
    return lib().eh_decompress_batch_noalloc(C.byref(p), k, structs, optrs, _stream_ptr(stream))


def decompress(c: Compressed, p: Optional[eh_plan_t] = None, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None, check: bool = True) -> torch.Tensor:
    """Decompresses into a raw-bits tensor (int16 for BF16, uint8 for FP8);
    with check=True waits for the stream and raises on a data error."""
    dev = c.code_len.device
    if p is None:
        p = plan(c.dtype)
    if out is None:
        out = torch.empty(c.n, dtype=_elem_dtype(c.dtype), device=dev)
    if workspace is None:
        workspace = torch.empty(decompress_workspace(p, 1), dtype=torch.uint8, device=dev)
    s = c.struct()
    rc = lib().eh_decompress(C.byref(p), C.byref(s), C.c_void_p(out.data_ptr()) if c.n else None,
                             C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream))
    _check(rc, "eh_decompress")
    if check:
        _check(get_status(workspace, stream), "eh_decompress (device status)")
    return out


def decompress_chunks(c: Compressed, first: int, count: int, p: Optional[eh_plan_t] = None,
                      out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                      stream=None, check: bool = True) -> torch.Tensor:
    dev = c.code_len.device
    if p is None:
        p = plan(c.dtype)
    K = p.chunk_elems
    n_out = max(0, min(c.n, (first + count) * K) - first * K)
    if out is None:
        out = torch.empty(n_out, dtype=_elem_dtype(c.dtype), device=dev)
    if workspace is None:
        workspace = torch.empty(decompress_workspace(p, 1), dtype=torch.uint8, device=dev)
    s = c.struct()
    rc = lib().eh_decompress_chunks(C.byref(p), C.byref(s), first, count,
                                    C.c_void_p(out.data_ptr()) if n_out else None,
                                    C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream))
    _check(rc, "eh_decompress_chunks")
    if check:
        _check(get_status(workspace, stream), "eh_decompress_chunks (device status)")
    return out


def container_size(p: eh_plan_t, n: int, exp_stream_bits: int, with_index: bool = False) -> int:
    out = C.c_uint64()
    _check(lib().eh_container_size(C.byref(p), n, exp_stream_bits, int(with_index), C.byref(out)),
           "eh_container_size")
    return out.value


def to_container(c: Compressed, p: eh_plan_t) -> bytes:
    """The stored form of a compressed tensor: its device arrays copied to the
    host and written by eh_container_write."""
    import numpy as np
    host = {k: getattr(c, k).cpu().numpy() for k in ("code_len", "code", "chunk_bit_off", "exp_stream", "sign_mant")}
    vi = c.value_index.cpu().numpy() if c.value_index is not None else None
    s = eh_compressed_t()
    s.dtype, s.n, s.n_chunks, s.exp_stream_bits = c.dtype, c.n, c.n_chunks, c.exp_stream_bits
    ptr = lambda a: a.ctypes.data_as(C.c_void_p) if a is not None and a.size else None
    s.code_len, s.code, s.chunk_bit_off = ptr(host["code_len"]), ptr(host["code"]), ptr(host["chunk_bit_off"])
    s.exp_stream, s.exp_stream_cap = ptr(host["exp_stream"]), host["exp_stream"].size
    s.sign_mant = ptr(host["sign_mant"])
    s.value_index = ptr(vi)
    size = container_size(p, c.n, c.exp_stream_bits, vi is not None)
    out = np.zeros(size, np.uint8)
    _check(lib().eh_container_write(C.byref(p), C.byref(s), out.ctypes.data_as(C.c_void_p), size),
           "eh_container_write")
    return out.tobytes()


def from_container(buf: bytes, device):
    """(Compressed on `device`, plan) from a stored container; raises EhError
    (EH_ERR_CORRUPT) if it fails its checks."""
    import numpy as np
    src = np.frombuffer(buf, np.uint8)
    p, v = eh_plan_t(), eh_compressed_t()
    _check(lib().eh_container_read(src.ctypes.data_as(C.c_void_p), src.size, C.byref(p), C.byref(v)),
           "eh_container_read")
    base = src.ctypes.data

    def arr(ptr, count, dtype):
        if not ptr or not count:
            return np.zeros(0, dtype)
        return src[ptr - base: ptr - base + count * np.dtype(dtype).itemsize].view(dtype)

    A = alphabet(p.dtype)
    nc = v.n_chunks
    c = alloc_compressed(p, v.n, device, index=bool(v.value_index))
    c.code_len.copy_(torch.from_numpy(arr(v.code_len, A, np.uint8).copy()))
    c.code.copy_(torch.from_numpy(arr(v.code, A, np.int32).copy()))
    c.chunk_bit_off.copy_(torch.from_numpy(arr(v.chunk_bit_off, nc + 1, np.int64).copy()))
    nb = v.exp_stream_cap
    if nb:
        c.exp_stream[:nb].copy_(torch.from_numpy(arr(v.exp_stream, nb, np.uint8).copy()))
    if c.sign_mant.numel():
        c.sign_mant.copy_(torch.from_numpy(arr(v.sign_mant, c.sign_mant.numel(), np.uint8).copy()))
    if c.value_index is not None:
        c.value_index.copy_(torch.from_numpy(arr(v.value_index, c.value_index.numel(), np.int32).copy()))
    c.exp_stream_bits = v.exp_stream_bits
    return c, p


def debug_set_fixup_rounds(rounds: int) -> None:
    """Test hook: the decoder's fix-up round limit for later calls (0: default)."""
    _check(lib().eh_debug_set_fixup_rounds(rounds), "eh_debug_set_fixup_rounds")


def get_status(workspace: torch.Tensor, stream=None) -> int:
    return lib().eh_get_status(C.c_void_p(workspace.data_ptr()), _stream_ptr(stream))


def version() -> str:
    return lib().eh_version().decode()


def codebook_from_counts(p: eh_plan_t, counts: torch.Tensor, stream=None, code_len: Optional[torch.Tensor] = None,
                         code: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """(code_len uint8[A], code int32[A]) on the counts' device from
    exponent counts (int64[A], uint64 values); the output arrays and the
    workspace may be passed in."""
    counts = counts.contiguous()
    A = alphabet(p.dtype)
    if code_len is None:
        code_len = torch.zeros(A, dtype=torch.uint8, device=counts.device)
    if code is None:
        code = torch.zeros(A, dtype=torch.int32, device=counts.device)
    ws = workspace
    if ws is None:
        ws = torch.empty(compress_bound(p, 0)[2], dtype=torch.uint8, device=counts.device)
    rc = lib().eh_codebook_from_counts(C.byref(p), C.c_void_p(counts.data_ptr()),
                                       C.c_void_p(code_len.data_ptr()), C.c_void_p(code.data_ptr()),
                                       C.c_void_p(ws.data_ptr()), ws.numel(), _stream_ptr(stream))
    _check(rc, "eh_codebook_from_counts")
    _check(get_status(ws, stream), "eh_codebook_from_counts (device status)")
    return code_len, code


class PageStore:
    """Fixed-slot page store (device arrays owned by torch) for online K/V
    compression with a frozen codebook."""

    def __init__(self, p: eh_plan_t, code_len: torch.Tensor, code: torch.Tensor, n_slots: int,
                 slot_bytes: int, raw_cap: int, device):
        dev = torch.device(device)
        n = p.chunk_elems
        sm_page = n if p.dtype == EH_BF16 else (n // 2 if p.dtype == EH_FP8_E4M3 else 0)
        self.plan = p
        self.code_len, self.code = code_len, code
        self.n_slots, self.slot_bytes, self.raw_cap = n_slots, slot_bytes, raw_cap
        self.slots = torch.zeros(n_slots * slot_bytes, dtype=torch.uint8, device=dev)
        self.sign_mant = torch.empty(n_slots * sm_page, dtype=torch.uint8, device=dev)
        self.page_meta = torch.zeros(n_slots, dtype=torch.int32, device=dev)
        self.raw_pool = torch.empty(max(raw_cap, 1) * n, dtype=torch.uint8, device=dev)
        self.raw_used = torch.zeros(1, dtype=torch.int32, device=dev)
        self.workspace = torch.empty(max(256, decompress_workspace(p, 1)), dtype=torch.uint8, device=dev)
        self.tables = None  # decode tables built once by prepare()

    def struct(self) -> eh_page_store_t:
        s = eh_page_store_t()
        s.code_len = self.code_len.data_ptr()
        s.code = self.code.data_ptr()
        s.slots = self.slots.data_ptr()
        s.slot_bytes = self.slot_bytes
        s.n_slots = self.n_slots
        s.raw_cap = self.raw_cap
        s.sign_mant = self.sign_mant.data_ptr() if self.sign_mant.numel() else None
        s.page_meta = self.page_meta.data_ptr()
        s.raw_pool = self.raw_pool.data_ptr()
        s.raw_used = self.raw_used.data_ptr()
        return s

    def append(self, x: torch.Tensor, slot_ids: torch.Tensor, stream=None):
        """Codes len(slot_ids) full pages of x into the given slots."""
        x = _raw(x)
        ids = slot_ids.to(device=x.device, dtype=torch.int32).contiguous()
        st = self.struct()
        rc = lib().eh_pages_append(C.byref(self.plan), C.byref(st), C.c_void_p(x.data_ptr()), ids.numel(),
                                   C.c_void_p(ids.data_ptr()), C.c_void_p(self.workspace.data_ptr()),
                                   self.workspace.numel(), _stream_ptr(stream))
        _check(rc, "eh_pages_append")
        return ids

    def prepare(self, stream=None):
        """Builds the frozen codebook's decode tables once; later reads use
        them (eh_pages_read_prepared) instead of building them every call."""
        self.tables = torch.empty(decompress_workspace(self.plan, 1), dtype=torch.uint8, device=self.slots.device)
        st = self.struct()
        _check(lib().eh_pages_prepare(C.byref(self.plan), C.byref(st), C.c_void_p(self.tables.data_ptr()),
                                      self.tables.numel(), _stream_ptr(stream)), "eh_pages_prepare")

    def read(self, slot_ids: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None,
             check: bool = True) -> torch.Tensor:
        ids = slot_ids.to(device=self.slots.device, dtype=torch.int32).contiguous()
        n = ids.numel() * self.plan.chunk_elems
        if out is None:
            out = torch.empty(n, dtype=_elem_dtype(self.plan.dtype), device=self.slots.device)
        st = self.struct()
        if self.tables is not None:
            rc = lib().eh_pages_read_prepared(C.byref(self.plan), C.byref(st), C.c_void_p(self.tables.data_ptr()),
                                              C.c_void_p(ids.data_ptr()), ids.numel(), C.c_void_p(out.data_ptr()),
                                              C.c_void_p(self.workspace.data_ptr()), self.workspace.numel(),
                                              _stream_ptr(stream))
            _check(rc, "eh_pages_read_prepared")
        else:
            rc = lib().eh_pages_read(C.byref(self.plan), C.byref(st), C.c_void_p(ids.data_ptr()), ids.numel(),
                                     C.c_void_p(out.data_ptr()), C.c_void_p(self.workspace.data_ptr()),
                                     self.workspace.numel(), _stream_ptr(stream))
            _check(rc, "eh_pages_read")
        if check:
            _check(get_status(self.workspace, stream), "eh_pages_read (device status)")
        return out

    def status(self, stream=None) -> int:
        return get_status(self.workspace, stream)


class Prefetcher:
    """Ring of `depth` decoded-operand slots (device memory owned by torch)
    filled on a decode stream ahead of the consumer stream.  submit() enqueues
    the decompression of a group of tensors (e.g. one transformer block) into
    the next slot and returns (slot, views); acquire()/release() bracket the
    consumer's use of a slot on the consumer stream."""

    def __init__(self, p: eh_plan_t, depth: int, slot_bytes: int, device, decode_stream=None,
                 max_ctas: int = 0):
        dev = torch.device(device)
        self.plan, self.depth = p, depth
        self.slot_bytes = (slot_bytes + 255) // 256 * 256
        self.slots = [torch.empty(self.slot_bytes, dtype=torch.uint8, device=dev) for _ in range(depth)]
        wsb = C.c_uint64(0)
        _check(lib().eh_prefetch_workspace(C.byref(p), depth, C.byref(wsb)), "eh_prefetch_workspace")
        self.workspace = torch.empty(wsb.value, dtype=torch.uint8, device=dev)
        self.stream = decode_stream if decode_stream is not None else torch.cuda.Stream(device=dev)
        ptrs = (C.c_void_p * depth)(*[t.data_ptr() for t in self.slots])
        h = C.c_void_p()
        _check(lib().eh_prefetch_create(C.byref(p), depth, ptrs, self.slot_bytes,
                                        C.c_void_p(self.workspace.data_ptr()), self.workspace.numel(),
                                        C.c_void_p(self.stream.cuda_stream), max_ctas, C.byref(h)),
               "eh_prefetch_create")
        self._h = h
        self._keep = [None] * depth  # the compressed inputs of each slot's decode, alive until reuse

    def submit(self, cs: List[Compressed]):
        k = len(cs)
        structs = (eh_compressed_t * k)(*[c.struct() for c in cs])
        offs = (C.c_uint64 * k)()
        slot = C.c_int(-1)
        _check(lib().eh_prefetch_submit(self._h, k, structs, offs, C.byref(slot)), "eh_prefetch_submit")
        s = slot.value
        self._keep[s] = list(cs)
        et = _elem_dtype(self.plan.dtype)
        size = 2 if self.plan.dtype == EH_BF16 else 1
        views = [self.slots[s][offs[i]:offs[i] + c.n * size].view(et) for i, c in enumerate(cs)]
        return s, views

    def acquire(self, slot: int, stream=None):
        _check(lib().eh_prefetch_acquire(self._h, slot, _stream_ptr(stream)), "eh_prefetch_acquire")

    def release(self, slot: int, stream=None):
        _check(lib().eh_prefetch_release(self._h, slot, _stream_ptr(stream)), "eh_prefetch_release")

    def status(self, slot: int) -> int:
        return lib().eh_prefetch_status(self._h, slot)

    def close(self):
        if self._h:
            lib().eh_prefetch_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ZfCompressed:
    """ZipFloat comparison codec buffers (device, owned by torch)."""

    def __init__(self, n: int, device):
        blocks, cap = C.c_uint64(0), C.c_uint64(0)
        _check(lib().eh_zf_bound(n, C.byref(blocks), C.byref(cap)), "eh_zf_bound")
        dev = torch.device(device)
        B = blocks.value
        self.n = n
        self.sign_mant = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        self.meta = torch.empty(max(B, 1), dtype=torch.int32, device=dev)
        self.dense = torch.empty(max(B * 192, 4), dtype=torch.int32, device=dev)
        self.sparse_off = torch.empty(max(B, 1), dtype=torch.int32, device=dev)
        self.sparse = torch.empty(max(cap.value, 1), dtype=torch.int16, device=dev)
        self.workspace = torch.empty(256, dtype=torch.uint8, device=dev)
        self.blocks = B
        self.n_records = 0
        self._s = eh_zf_t()

    def struct(self) -> eh_zf_t:
        s = self._s
        s.n = self.n
        s.sign_mant = self.sign_mant.data_ptr()
        s.meta = self.meta.data_ptr()
        s.dense = self.dense.data_ptr()
        s.sparse_off = self.sparse_off.data_ptr()
        s.sparse = self.sparse.data_ptr()
        s.sparse_cap = self.sparse.numel()
        s.n_records = self.n_records
        return s

    def compressed_bytes(self) -> int:
        return self.n + 8 * self.blocks + 768 * self.blocks + 2 * self.n_records


def zf_compress(x: torch.Tensor, out: Optional[ZfCompressed] = None, wait: bool = True, stream=None) -> ZfCompressed:
    x = _raw(x)
    if out is None:
        out = ZfCompressed(x.numel(), x.device)
    st = out.struct()
    rc = lib().eh_zf_compress(C.c_void_p(x.data_ptr()), C.byref(st), C.c_void_p(out.workspace.data_ptr()),
                              out.workspace.numel(), int(wait), _stream_ptr(stream))
    _check(rc, "eh_zf_compress")
    if wait:
        out.n_records = st.n_records
    return out


def zf_decompress(c: ZfCompressed, out: Optional[torch.Tensor] = None, stream=None,
                  check: bool = True) -> torch.Tensor:
    if out is None:
        out = torch.empty(c.n, dtype=torch.int16, device=c.sign_mant.device)
    st = c.struct()
    rc = lib().eh_zf_decompress(C.byref(st), C.c_void_p(out.data_ptr()), C.c_void_p(c.workspace.data_ptr()),
                                c.workspace.numel(), _stream_ptr(stream))
    _check(rc, "eh_zf_decompress")
    if check:
        _check(get_status(c.workspace, stream), "eh_zf_decompress (device status)")
    return out
