"""The C-ABI library loads and exports every entry point the header declares.

CPU-only: only the host-side calls that touch no GPU are exercised (plans,
size queries, status strings).
"""
import ctypes as C
import os
import re
import subprocess
import sys

import pytest

from exponent_entropy_coding_b200 import build as eh_build
from exponent_entropy_coding_b200 import exphuff as eh

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "exphuff.h")


@pytest.fixture(scope="module")
def lib():
    eh_build.build()
    return eh.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"EH_API\s+[\w\s\*]*?\b(eh_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("eh_plan", "eh_compress", "eh_decompress", "eh_decompress_batch",
                 "eh_decompress_chunks", "eh_compress_bound", "eh_get_status"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", eh.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(lib, n)
    assert sorted(eh.EXPORTED) == names
    # nothing but the API is exported (the static CUDA runtime stays hidden)
    assert {n for n in exported if not n.startswith("eh_")} == set()


def test_plan_and_sizes(lib):
    p = eh.plan(eh.EH_BF16)
    assert (p.dtype, p.chunk_elems, p.max_code_len) == (0, 65536, 32)
    p8 = eh.plan(eh.EH_FP8_E4M3, 4096, 12)
    assert (p8.dtype, p8.chunk_elems, p8.max_code_len) == (1, 4096, 12)
    for bad in [(eh.EH_BF16, 1000, 32), (eh.EH_BF16, 65536, 33), (7, 65536, 32),
                (eh.EH_BF16, 131072, 32)]:
        with pytest.raises(eh.EhError) as ei:
            eh.plan(*bad)
        assert ei.value.code == eh.EH_ERR_UNSUPPORTED
    n = 3 * 65536 + 5
    cap, smb, ws = eh.compress_bound(p, n)
    assert cap == ((n * 32 + 7) // 8 + 15) // 16 * 16 + 16
    assert smb == n
    assert ws > 0 and ws % 256 == 0
    cap8, smb8, _ = eh.compress_bound(p8, 7)
    assert smb8 == 4 and cap8 == 16 + 16   # ceil(7*12/8)=11 -> 16, +16
    assert eh.compress_batch_workspace(p, [n, 1, 0]) > ws
    assert eh.decompress_workspace(p, 16) > eh.decompress_workspace(p, 1)
    with pytest.raises(eh.EhError):
        eh.decompress_workspace(p, 17)


def test_status_strings(lib):
    for code in range(8):
        s = lib.eh_status_str(code)
        assert s and s.decode()
    assert lib.eh_version().decode().startswith("libexphuff")


def test_invalid_arguments_rejected_before_any_launch(lib):
    p = eh.plan(eh.EH_BF16)
    s = eh.eh_compressed_t()
    s.dtype = 0
    s.n = 10
    # null device pointers: rejected on the host, no CUDA call is made
    assert lib.eh_compress(C.byref(p), None, 10, C.byref(s), None, 0, None) == eh.EH_ERR_INVALID_ARG
    assert lib.eh_decompress(C.byref(p), C.byref(s), None, None, 0, None) == eh.EH_ERR_INVALID_ARG
    assert lib.eh_get_status(None, None) == eh.EH_ERR_INVALID_ARG


def test_missing_library_fails_loudly():
    """Without libexphuff.so the binding raises; there is no CPU fallback."""
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from exponent_entropy_coding_b200 import exphuff as eh\n"
            "eh.LIB_PATH = '/nonexistent/libexphuff.so'\n"
            "try:\n"
            "    eh.plan(0)\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n"
            "    sys.exit(0)\n"
            "sys.exit(3)\n") % ROOT
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.stdout, r.stderr)
    assert "not built" in r.stdout


def test_python_constants_match_the_header():
    """The binding's copies of the header's macros (batch limits, index
    stride, chunk default) are the header's values."""
    text = open(HEADER).read()
    macros = dict(re.findall(r"#define\s+(EH_\w+)\s+(\w+)", text))
    for name in ("EH_NOALLOC_MAX_BATCH", "EH_MAX_BATCH", "EH_INDEX_STRIDE", "EH_PREFETCH_MAX_DEPTH",
                 "EH_DEFAULT_CHUNK_ELEMS", "EH_MAX_CODE_LEN", "EH_PAGE_RAW"):
        if hasattr(eh, name):
            assert int(macros[name].rstrip("u"), 0) == getattr(eh, name), name


def test_noalloc_scratch_size_documented(lib):
    """The no-allocation entry point's fixed array is 256 bytes plus one
    decompression workspace's tables per tensor: the documented 37,888 bytes
    per tensor is what eh_decompress_workspace reports per tensor."""
    p = eh.plan(eh.EH_BF16)
    per_tensor = eh.decompress_workspace(p, 2) - eh.decompress_workspace(p, 1)
    assert per_tensor == 37888
    assert "256 +\n * EH_NOALLOC_MAX_BATCH * 37,888 bytes" in open(HEADER).read()
