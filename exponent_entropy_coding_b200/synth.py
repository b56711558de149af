"""Seeded synthetic tensors shaped like the pages' workloads.

This module only draws random floats and rounds them to the storage format
(round-to-nearest-even through torch's own casts).  It holds none of the
codec's arithmetic, so both the CUDA path and the CPU oracle can consume its
output.  Every generator returns raw bit patterns as numpy arrays: ``uint16``
for BF16, ``uint8`` for FP8 E4M3.

Workloads (the pages measure on real checkpoints and K/V caches, which are not
available; these stand in for them):

* ``bf16_1m``   one BF16 1024x1024 tensor, N(0, 0.02^2), seed 0.
* ``fp8_16m``   one FP8 E4M3 4096x4096 tensor: N(0, 0.02^2) scaled per tensor so
  that amax maps to 448, then rounded to E4M3, seed 1.
* ``llama8b_block``  the seven BF16 weight matrices of one Llama-3.1-8B block
  (q 4096x4096, k 1024x4096, v 1024x4096, o 4096x4096, gate/up 14336x4096,
  down 4096x14336; 218,103,808 values), Student-t with 5 degrees of freedom
  scaled to standard deviation 0.02, seed 2.
* ``kv_layer``  one layer's BF16 K and V caches, [batch 8, tokens 8192,
  kv heads 8, head dim 128] each: N(0, 1) times a per-channel lognormal(0, 0.5)
  scale, with 4 outlier channels per head scaled by 20, seed 3.  A 64-token
  page of one tensor is 64*8*128 = 65,536 values.
* ``lm_head``   one BF16 128256x4096 tensor, N(0, 0.02^2), seed 4.
* ``nvfp4_scales`` / ``mxfp4_scales``  the block scale bytes of the
  ``llama8b_block`` weights quantised to FP4: E4M3 scales per 16 values
  (13,631,488 bytes) or E8M0 scales per 32 values (6,815,744 bytes).
"""
import math

import numpy as np
import torch

LLAMA8B_BLOCK_SHAPES = [
    ("q_proj", (4096, 4096)),
    ("k_proj", (1024, 4096)),
    ("v_proj", (1024, 4096)),
    ("o_proj", (4096, 4096)),
    ("gate_proj", (14336, 4096)),
    ("up_proj", (14336, 4096)),
    ("down_proj", (4096, 14336)),
]

WORKLOADS = ("bf16_1m", "fp8_16m", "llama8b_block", "kv_layer", "lm_head")
SCALE_WORKLOADS = ("nvfp4_scales", "mxfp4_scales")


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32/float64 -> BF16 bit patterns (uint16), round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).reshape(a.shape)


def to_fp8_e4m3_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> FP8 E4M3 (fn variant) bit patterns (uint8), round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().reshape(a.shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(n: int, seed: int, std: float = 0.02) -> np.ndarray:
    rng = np.random.default_rng(seed)
    w = rng.standard_normal(n, dtype=np.float32)
    w *= np.float32(std)
    return to_bf16_bits(w)


def normal_fp8(n: int, seed: int, std: float = 0.02) -> np.ndarray:
    rng = np.random.default_rng(seed)
    w = rng.standard_normal(n, dtype=np.float32)
    w *= np.float32(std)
    w *= np.float32(448.0) / np.abs(w).max()
    return to_fp8_e4m3_bits(w)


def fibonacci_symbols(m: int, seed: int, chunk: int = 65536) -> np.ndarray:
    """Symbol indices 0 .. m-1 occurring F(1), F(2), ..., F(m) times
    (Fibonacci numbers): the histogram that gives a Huffman code its largest
    depth, m - 1.  Placement: the first chunk holds one of the two rarest
    symbols, the next 14 rarest and common ones; the second chunk holds the
    other rarest symbol and symbols of middle rarity (long codes on
    average); the rest is shuffled."""
    rng = np.random.default_rng(seed)
    fib = [1, 1]
    while len(fib) < m:
        fib.append(fib[-1] + fib[-2])
    fib = fib[:m]
    pools = [np.full(c, i, dtype=np.int64) for i, c in enumerate(fib)]
    take = lambda i, k: (pools.__setitem__(i, pools[i][k:]), np.full(k, i, dtype=np.int64))[1]
    c0 = [take(0, 1)] + [take(i, len(pools[i])) for i in range(2, 16)]
    n0 = sum(len(a) for a in c0)
    c0.append(take(m - 1, chunk - n0))
    c1 = [take(1, 1)]
    left = chunk - 1
    for i in range(16, m):
        k = min(left, len(pools[i]))
        c1.append(take(i, k))
        left -= k
        if left == 0:
            break
    head = np.concatenate(c0)
    head = head[rng.permutation(head.size)]
    second = np.concatenate(c1)
    second = second[rng.permutation(second.size)]
    rest = np.concatenate(pools)
    rest = rest[rng.permutation(rest.size)]
    return np.concatenate([head, second, rest])


def fibonacci_bf16(m: int, seed: int, first_field: int = 60, chunk: int = 65536) -> np.ndarray:
    """BF16 values whose exponent fields first_field .. first_field+m-1 follow
    fibonacci_symbols(m, seed, chunk).  Each value is
    +-(1 + k/128) * 2^(field - 127) with random sign and k."""
    idx = fibonacci_symbols(m, seed, chunk)
    rng = np.random.default_rng(seed + 1000)
    field = (idx + first_field).astype(np.float64)
    mant = rng.integers(0, 128, idx.size)
    sign = np.where(rng.integers(0, 2, idx.size) == 1, -1.0, 1.0)
    v = sign * (1.0 + mant / 128.0) * np.exp2(field - 127.0)
    return to_bf16_bits(v.astype(np.float32))


def student_t_f32(shape, rng: np.random.Generator, df: float = 5.0,
                  std: float = 0.02) -> np.ndarray:
    # a t(df) draw has variance df/(df-2); rescale to the requested std
    w = rng.standard_t(df, size=shape).astype(np.float32)
    w *= np.float32(std / math.sqrt(df / (df - 2.0)))
    return w


def student_t_bf16(shape, rng: np.random.Generator, df: float = 5.0,
                   std: float = 0.02) -> np.ndarray:
    return to_bf16_bits(student_t_f32(shape, rng, df, std))


def nvfp4_block_scales(w: np.ndarray, block: int = 16) -> np.ndarray:
    """E4M3 scale bytes of NVFP4-style quantisation: one scale per block of
    `block` values, amax/6 (6 = largest FP4 E2M1 value) divided by a
    per-tensor factor that maps the largest block scale to 448."""
    a = np.abs(w.reshape(-1, block)).max(axis=1).astype(np.float32) / np.float32(6.0)
    g = a.max() / np.float32(448.0) if a.max() > 0 else np.float32(1.0)
    return to_fp8_e4m3_bits(a / g)


def mxfp4_block_scales(w: np.ndarray, block: int = 32) -> np.ndarray:
    """E8M0 scale bytes of MXFP4-style quantisation: one power-of-two scale
    per block of `block` values, 2^(floor(log2(amax)) - 2) (2 = largest FP4
    E2M1 exponent), stored as the biased exponent (+127)."""
    a = np.abs(w.reshape(-1, block)).max(axis=1).astype(np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126))) - 2
    return np.clip(e + 127, 0, 254).astype(np.uint8)


def llama8b_block(seed: int = 2, scale: int = 1, count: int = 7):
    """[(name, bits)] for the first ``count`` of the seven matrices; ``scale``
    divides the row count (scale=1 is the full block)."""
    rng = np.random.default_rng(seed)
    out = []
    for name, (r, c) in LLAMA8B_BLOCK_SHAPES[:count]:
        out.append((name, student_t_bf16((max(1, r // scale), c), rng).reshape(-1)))
    return out


def kv_tensor(rng: np.random.Generator, batch: int, tokens: int, heads: int = 8,
              head_dim: int = 128, outliers: int = 4) -> np.ndarray:
    scale = rng.lognormal(0.0, 0.5, size=(heads, head_dim)).astype(np.float32)
    for h in range(heads):
        idx = rng.choice(head_dim, outliers, replace=False)
        scale[h, idx] *= np.float32(20.0)
    x = rng.standard_normal((batch, tokens, heads, head_dim), dtype=np.float32)
    x *= scale[None, None, :, :]
    return to_bf16_bits(x).reshape(-1)


def kv_layer(seed: int = 3, batch: int = 8, tokens: int = 8192):
    """[("k", bits), ("v", bits)], layout [batch, token, head, dim]."""
    rng = np.random.default_rng(seed)
    k = kv_tensor(rng, batch, tokens)
    v = kv_tensor(rng, batch, tokens)
    return [("k", k), ("v", v)]


def fp4_scales(kind: str = "nv", seed: int = 2, scale: int = 1):
    """[(name, scale bytes)] of the Llama-8B block's seven matrices (the same
    Student-t weights as `llama8b_block`) quantised block-wise to FP4:
    kind "nv" = E4M3 scales per 16 values, "mx" = E8M0 scales per 32 values."""
    rng = np.random.default_rng(seed)
    out = []
    for name, (r, c) in LLAMA8B_BLOCK_SHAPES:
        w = student_t_f32((max(1, r // scale), c), rng).reshape(-1)
        out.append((name, nvfp4_block_scales(w) if kind == "nv" else mxfp4_block_scales(w)))
    return out


def workload(name: str, scale: int = 1):
    """Returns (dtype_name, [(item_name, bits)]).  ``scale`` > 1 shrinks the
    workload (fewer rows / tokens) for quick parity runs."""
    if name == "bf16_1m":
        return "bf16", [("w", normal_bf16((1 << 20) // scale, seed=0))]
    if name == "fp8_16m":
        return "fp8_e4m3", [("w", normal_fp8((4096 * 4096) // scale, seed=1))]
    if name == "llama8b_block":
        return "bf16", llama8b_block(seed=2, scale=scale)
    if name == "kv_layer":
        return "bf16", kv_layer(seed=3, tokens=max(64, 8192 // scale))
    if name == "lm_head":
        return "bf16", [("w", normal_bf16((128256 // scale) * 4096, seed=4))]
    if name == "nvfp4_scales":
        return "bytes", fp4_scales("nv", seed=2, scale=scale)
    if name == "mxfp4_scales":
        return "bytes", fp4_scales("mx", seed=2, scale=scale)
    raise KeyError(name)
