"""Seeded synthetic inputs for block-quantized attention.

This module draws random numbers and rounds them to storage types. It holds
none of the attention or quantization arithmetic, so the CPU oracle and the
CUDA path can both be fed from it without sharing any of the method.

Generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used counter-style: output i of stream s
under seed k is mix(base + (i + 1) * GAMMA) with base = mix(k * 2^32 + s).
Normals come from the Box-Muller transform in float64. Values are rounded to
float32 (round-to-nearest-even) and then to bfloat16 or float16
(round-to-nearest-even).

Workload shapes follow the five attention problems stated on the pages
(block quantized FP8/INT8 prefill and INT8/INT4 KV-cache decode).
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser (in place on a fresh array)."""
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def raw_u64(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """n SplitMix64 outputs of (seed, stream), starting at counter `start`."""
    with np.errstate(over="ignore"):
        base = _mix(np.array([(seed << 32) + stream], dtype=np.uint64))[0]
        z = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        z *= _GAMMA
        z += base
        return _mix(z)


_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        from concurrent.futures import ThreadPoolExecutor
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))
    return _POOL


def _chunked(n: int, dtype, fill, chunk: int = 1 << 22) -> np.ndarray:
    """Fill an n-element array by fill(out_slice, start) over independent
    chunks in a thread pool (numpy releases the GIL inside ufuncs). The result
    does not depend on the chunking: every element is a function of its
    counter alone."""
    out = np.empty(n, dtype=dtype)
    futs = [_pool().submit(fill, out[s:s + chunk], s) for s in range(0, n, chunk)]
    for f in futs:
        f.result()
    return out


def _u01(seed: int, stream: int, m: int, start: int) -> np.ndarray:
    u = raw_u64(seed, stream, m, start) >> np.uint64(11)
    return (u.astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def uniform01(seed: int, stream: int, n: int) -> np.ndarray:
    """Uniform float64 in (0, 1): 53 high bits, offset by half a step."""
    def fill(o, s):
        o[:] = _u01(seed, stream, len(o), s)
    return _chunked(n, np.float64, fill)


def normal(seed: int, stream: int, n: int) -> np.ndarray:
    """Standard normal float64 via Box-Muller (cosine branch only). Uses the
    uniform streams 1000 + 2*stream and 1001 + 2*stream, disjoint from the
    streams that uniform01 is called with directly."""
    def fill(o, s):
        u1 = _u01(seed, 1000 + 2 * stream, len(o), s)
        u2 = _u01(seed, 1001 + 2 * stream, len(o), s)
        o[:] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return _chunked(n, np.float64, fill)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64/float32 -> bfloat16 bit patterns (via float32, both steps RNE)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def f64_to_f16_bits(x: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def int8_uniform(seed: int, stream: int, n: int, lo: int = -127, hi: int = 127) -> np.ndarray:
    """n integers in [lo, hi]: each 64-bit draw gives four 16-bit chunks c
    (little-endian), mapped to lo + floor(c * (hi - lo + 1) / 2^16)."""
    span = hi - lo + 1

    def fill(o, s):                    # s is a multiple of 4 (chunk size is)
        c = raw_u64(seed, stream, (len(o) + 3) // 4, start=s // 4).view(np.uint16)[:len(o)]
        c = c.astype(np.uint32)
        c *= np.uint32(span)
        c >>= np.uint32(16)
        o[:] = (c.astype(np.int32) + lo).astype(np.int8)
    return _chunked(n, np.int8, fill)


def random_bytes(seed: int, stream: int, n: int) -> np.ndarray:
    """n uniform bytes (eight per 64-bit draw, little-endian)."""
    def fill(o, s):                    # s is a multiple of 8
        o[:] = raw_u64(seed, stream, (len(o) + 7) // 8, start=s // 8).view(np.uint8)[:len(o)]
    return _chunked(n, np.uint8, fill)


def haar_orthogonal(seed: int, stream: int, d: int) -> np.ndarray:
    """Seeded random orthogonal d x d matrix (float32): QR of a Gaussian matrix
    with the signs of R's diagonal folded into Q (Mezzadri 2007)."""
    g = normal(seed, stream, d * d).reshape(d, d)
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return np.ascontiguousarray(q.astype(np.float32))


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

BNSD, BSND = 0, 1
F16, BF16, INT8, FP8_E4M3, INT4_PACKED = 0, 1, 2, 3, 4


@dataclass
class PrefillProblem:
    name: str
    B: int
    H: int
    N: int
    D: int
    in_dtype: int            # F16 or BF16 (bit patterns stored as uint16)
    code_dtype: int          # INT8 or FP8_E4M3
    layout: int              # BNSD or BSND
    causal: bool
    rotate: bool
    seed: int
    outlier_frac: float = 0.0
    outlier_gain: float = 20.0
    lognormal_sigma: float = 0.0
    q_block: int = 128
    kv_block: int = 256

    def shape(self):
        if self.layout == BNSD:
            return (self.B, self.H, self.N, self.D)
        return (self.B, self.N, self.H, self.D)


@dataclass
class DecodeProblem:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    D: int
    kv_dtype: int            # INT8 or INT4_PACKED
    seed: int
    kv_block: int = 256
    group: int = 128
    scale_lo: float = 0.005
    scale_hi: float = 0.02


# The five problems: sizes, dtypes and distributions as stated for the method.
TINY_FP8 = PrefillProblem("tiny_fp8_b1h2n256d64", 1, 2, 256, 64, F16, FP8_E4M3, BNSD,
                          causal=False, rotate=False, seed=1)
INT8_CAUSAL = PrefillProblem("int8_causal_b1h32n4096d128", 1, 32, 4096, 128, BF16, INT8, BNSD,
                             causal=True, rotate=True, seed=2, outlier_frac=0.01)
FP8_LONG = PrefillProblem("fp8_bsnd_b1h24n16384d128", 1, 24, 16384, 128, BF16, FP8_E4M3, BSND,
                          causal=False, rotate=True, seed=3, lognormal_sigma=0.5)
INT8_KV_DECODE = DecodeProblem("int8kv_decode_b64hq32hkv8l8192d128", 64, 32, 8, 8192, 128, INT8,
                               seed=4, scale_lo=0.005, scale_hi=0.02)
INT4_KV_DECODE = DecodeProblem("int4kv_decode_b16hq32hkv8l32768d128", 16, 32, 8, 32768, 128,
                               INT4_PACKED, seed=5, scale_lo=0.01, scale_hi=0.05)

PROBLEMS = {p.name: p for p in (TINY_FP8, INT8_CAUSAL, FP8_LONG, INT8_KV_DECODE, INT4_KV_DECODE)}


def make_prefill(p: PrefillProblem) -> dict:
    """Q, K, V bit patterns (uint16, layout p.layout) and the rotation (or None).

    Streams: Q=1, K=2, V=3, rotation=4, outlier channel draw=5, per-token
    magnitudes 6..8 (Q, K, V)."""
    n = p.B * p.H * p.N * p.D
    out = {"problem": p}
    outliers = None
    if p.outlier_frac > 0:
        n_out = int(round(p.outlier_frac * p.H * p.D))
        u = uniform01(p.seed, 5, 4 * n_out + 64)
        picks = []
        for v in (u * (p.H * p.D)).astype(np.int64):
            if v not in picks:
                picks.append(int(v))
            if len(picks) == n_out:
                break
        outliers = np.array(sorted(picks), dtype=np.int64)      # flat (h * D + d)
        out["outlier_channels"] = outliers
    for name, stream in (("q", 1), ("k", 2), ("v", 3)):
        x = normal(p.seed, stream, n).reshape(p.shape())
        if outliers is not None:
            gain = np.ones(p.H * p.D)
            gain[outliers] = p.outlier_gain
            g = gain.reshape(p.H, p.D)
            if p.layout == BNSD:
                x = x * g[None, :, None, :]
            else:
                x = x * g[None, None, :, :]
        if p.lognormal_sigma > 0:
            mag = np.exp(p.lognormal_sigma * normal(p.seed, 5 + stream, p.B * p.N)).reshape(p.B, p.N)
            if p.layout == BNSD:
                x = x * mag[:, None, :, None]
            else:
                x = x * mag[:, :, None, None]
        bits = f32_to_bf16_bits(x) if p.in_dtype == BF16 else f64_to_f16_bits(x)
        out[name] = bits.reshape(p.shape())
    out["rot"] = haar_orthogonal(p.seed, 4, p.D) if p.rotate else None
    return out


def make_decode(p: DecodeProblem) -> dict:
    """Query bits, KV codes and scales for a decode problem.

    INT8: k/v int8 [B,Hkv,L,D]; scales float32 [B,Hkv,ceil(L/kv_block)].
    INT4: k/v uint8 [B,Hkv,L,D/2], element 2i in the low nibble and 2i+1 in
    the high nibble; scales float16 bits [B,Hkv,L,D/group].
    Streams: q=1, K=2, V=3, K scales=4, V scales=5."""
    q = f32_to_bf16_bits(normal(p.seed, 1, p.B * p.Hq * p.D)).reshape(p.B, p.Hq, 1, p.D)
    out = {"problem": p, "q": q}
    if p.kv_dtype == INT8:
        nblk = -(-p.L // p.kv_block)
        for name, stream in (("k", 2), ("v", 3)):
            out[name] = int8_uniform(p.seed, stream, p.B * p.Hkv * p.L * p.D).reshape(
                p.B, p.Hkv, p.L, p.D)
        for name, stream in (("k_scales", 4), ("v_scales", 5)):
            u = uniform01(p.seed, stream, p.B * p.Hkv * nblk)
            out[name] = (p.scale_lo + (p.scale_hi - p.scale_lo) * u).astype(np.float32).reshape(
                p.B, p.Hkv, nblk)
    else:
        ngroups = p.D // p.group
        # Uniform random bytes are exactly two independent uniform 4-bit
        # two's-complement codes in [-8, 7] per byte, whatever the nibble order.
        for name, stream in (("k", 2), ("v", 3)):
            nbytes = p.B * p.Hkv * p.L * p.D // 2
            out[name] = random_bytes(p.seed, stream, nbytes).reshape(p.B, p.Hkv, p.L, p.D // 2)
        for name, stream in (("k_scales", 4), ("v_scales", 5)):
            u = uniform01(p.seed, stream, p.B * p.Hkv * p.L * ngroups)
            s = p.scale_lo + (p.scale_hi - p.scale_lo) * u
            out[name] = f64_to_f16_bits(s).reshape(p.B, p.Hkv, p.L, ngroups)
    return out


def scaled(p, **kw):
    """A copy of problem p with some fields replaced (smaller test sizes)."""
    from dataclasses import replace
    return replace(p, **kw)
