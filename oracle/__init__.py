"""CPU oracle for block-quantized attention (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package. It wraps `qattn_oracle.c` (plain C, compiled with gcc)
through ctypes and shares no code with the CUDA library. Work over several
(batch, head) pairs is spread over Python threads; ctypes releases the GIL
for the duration of each C call, so the threads run in parallel.

See qattn_oracle.c for the arithmetic and for where each step is stated.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qattn_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

BNSD, BSND = 0, 1
F16, BF16, INT8, FP8_E4M3, INT4_PACKED = 0, 1, 2, 3, 4
F32 = 100

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
                               "-Wall", "-shared", "-fPIC", "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = C.CDLL(LIB)
        P = C.c_void_p
        i, f, d = C.c_int, C.c_float, C.c_double
        L.orc_e4m3_from_f32.argtypes, L.orc_e4m3_from_f32.restype = [f], C.c_uint8
        L.orc_e4m3_to_f32.argtypes, L.orc_e4m3_to_f32.restype = [C.c_uint8], f
        L.orc_e4m3_encode_n.argtypes = [P, C.c_int64, P]
        L.orc_e4m3_decode_n.argtypes = [P, C.c_int64, P]
        L.orc_f64_to_bf16.argtypes, L.orc_f64_to_bf16.restype = [d], C.c_uint16
        L.orc_f16_to_f32.argtypes, L.orc_f16_to_f32.restype = [C.c_uint16], f
        L.orc_bf16_to_f32.argtypes, L.orc_bf16_to_f32.restype = [C.c_uint16], f
        L.orc_int4_pack.argtypes, L.orc_int4_pack.restype = [i, i], C.c_uint8
        L.orc_int4_lo.argtypes, L.orc_int4_lo.restype = [C.c_uint8], i
        L.orc_int4_hi.argtypes, L.orc_int4_hi.restype = [C.c_uint8], i
        L.orc_rotate_row.argtypes = [P, P, i, P]
        L.orc_quant_block.argtypes = [P, i, i, i, i, i, i, P, i, i, i, i, i, P, P]
        L.orc_quant_head.argtypes = [P, i, i, i, i, i, i, P, i, i, i, i, P, P]
        L.orc_prefill_rows.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, i, i, i, i, i, i, f, i,
                                       i, i, P, i, P, P, P]
        L.orc_exact_rows.argtypes = [P, P, P, i, i, i, i, i, i, i, i, d, i, i, P, i, P]
        L.orc_decode_one.argtypes = [P, P, P, P, P, i, i, i, i, i, i, i, i, f, i, i, i, P, P]
        L.orc_f32_to_f16.argtypes, L.orc_f32_to_f16.restype = [f], C.c_uint16
        L.orc_kv_append_int8.argtypes = [P, i, i, i, i, i, i, i, P, P, i, i]
        L.orc_kv_append_int4.argtypes = [P, i, i, i, i, i, i, i, P, P, i, i]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


_POOL = None


def pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=threads())
    return _POOL


def threads() -> int:
    return int(os.environ.get("QATTN_ORACLE_THREADS", os.cpu_count() or 1))


def _run_all(jobs):
    futs = [pool().submit(j) for j in jobs]
    for f in futs:
        rc = f.result()
        if rc:
            raise RuntimeError("oracle call failed with code %d" % rc)


# ---------------------------------------------------------------------------
# Codecs
# ---------------------------------------------------------------------------

def e4m3_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_n(_p(x), x.size, _p(out))
    return out


def e4m3_decode(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float32)
    lib().orc_e4m3_decode_n(_p(c), c.size, _p(out))
    return out


def int4_pack(w0: int, w1: int) -> int:
    return int(lib().orc_int4_pack(int(w0), int(w1)))


def int4_unpack(b: int):
    return int(lib().orc_int4_lo(b)), int(lib().orc_int4_hi(b))


# ---------------------------------------------------------------------------
# Rotation + block quantization
# ---------------------------------------------------------------------------

def rotate_row(x: np.ndarray, rot) -> np.ndarray:
    """float32 y = x R for one row (sequential float32 FMA chain)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    R = None if rot is None else np.ascontiguousarray(rot, dtype=np.float32)
    y = np.empty_like(x)
    lib().orc_rotate_row(_p(x), _p(R), x.size, _p(y))
    return y


def rotate_block_quant(x_bits: np.ndarray, x_dtype: int, layout: int, rot, block: int,
                       code_dtype: int, heads=None, blocks=None):
    """Codes (uint8, same shape as x; INT4_PACKED: [..., D/2], two codes per
    byte, element 2i in the low nibble) and scales float32 [B, H, nblk].

    heads: optional list of (b, h) to compute (others are left zero).
    blocks: optional list of (b, h, blk) to compute (overrides heads)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if layout == BNSD:
        B, H, N, D = x_bits.shape
    else:
        B, N, H, D = x_bits.shape
    nblk = -(-N // block)
    codes = np.zeros(x_bits.shape, dtype=np.uint8)
    scales = np.zeros((B, H, nblk), dtype=np.float32)
    R = None if rot is None else np.ascontiguousarray(rot, dtype=np.float32)
    L = lib()
    if blocks is not None:
        jobs = [(lambda b=b, h=h, k=k: L.orc_quant_block(_p(x_bits), x_dtype, layout, B, H, N, D, _p(R),
                                                         block, code_dtype, b, h, k, _p(codes), _p(scales)))
                for (b, h, k) in blocks]
    else:
        hs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
        jobs = [(lambda b=b, h=h: L.orc_quant_head(_p(x_bits), x_dtype, layout, B, H, N, D, _p(R),
                                                   block, code_dtype, b, h, _p(codes), _p(scales)))
                for (b, h) in hs]
    _run_all(jobs)
    if code_dtype == INT4_PACKED:
        c = codes & 0xF                                    # two's complement nibbles
        codes = (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)
    return codes, scales


# ---------------------------------------------------------------------------
# Prefill attention
# ---------------------------------------------------------------------------

def prefill_rows(qc, qs, kc, ks, vc, vs, code_dtype: int, layout: int, causal: bool,
                 rows_by_head: dict, q_block=128, kv_block=256, kv_tile=128,
                 softmax_scale=0.0, p_quant=True, Nkv=None, want_f64=False, want_lse=False,
                 row_chunk=None, v_dtype=None):
    """Output rows of quantized attention.

    qc/kc/vc: codes (uint8 for INT8/FP8 -- INT8 codes as their byte pattern --
    or float32 for F32), shaped like the layout; Q and K have code_dtype, V
    has v_dtype (default code_dtype; INT4_PACKED: [..., D/2] packed bytes).
    rows_by_head: {(b, h): [rows]}.
    row_chunk: optional number of rows per parallel job (default: one job per
    head). Returns {(b, h): (bf16 bits [n, D], f64 [n, D] or None, lse [n] or
    None)}.
    """
    if layout == BNSD:
        B, H, Nq, D = qc.shape
        Nk = kc.shape[2]
    else:
        B, Nq, H, D = qc.shape
        Nk = kc.shape[1]
    if Nkv is not None:
        Nk = Nkv
    if code_dtype == INT4_PACKED:                          # packed: D/2 bytes per row
        D *= 2
    arrs = [np.ascontiguousarray(a) for a in (qc, qs, kc, ks, vc, vs)]
    for a in arrs[1::2]:
        assert a.dtype == np.float32
    L = lib()
    res = {}
    jobs = []
    for (b, h), rows in rows_by_head.items():
        r = np.ascontiguousarray(rows, dtype=np.int32)
        ob = np.empty((len(r), D), dtype=np.uint16)
        of = np.empty((len(r), D), dtype=np.float64) if want_f64 else None
        ls = np.empty(len(r), dtype=np.float64) if want_lse else None
        res[(b, h)] = (ob, of, ls)
        step = row_chunk or max(1, len(r))
        for s0 in range(0, len(r), step):
            s1 = min(len(r), s0 + step)
            rr = r[s0:s1]
            obs = ob[s0:s1]
            ofs = of[s0:s1] if of is not None else None
            lss = ls[s0:s1] if ls is not None else None
            jobs.append(lambda b=b, h=h, rr=rr, obs=obs, ofs=ofs, lss=lss: L.orc_prefill_rows(
                _p(arrs[0]), _p(arrs[1]), _p(arrs[2]), _p(arrs[3]), _p(arrs[4]), _p(arrs[5]),
                code_dtype, code_dtype if v_dtype is None else v_dtype, layout, B, H, Nq, Nk, D, q_block,
                kv_block, kv_tile, int(causal),
                float(softmax_scale), int(p_quant), b, h, _p(rr), len(rr), _p(obs), _p(ofs), _p(lss)))
    _run_all(jobs)
    return res


def exact_rows(q_bits, k_bits, v_bits, in_dtype: int, layout: int, causal: bool,
               rows_by_head: dict, softmax_scale=0.0):
    """float64 softmax(q k^T * scale) v on the unquantized inputs."""
    if layout == BNSD:
        B, H, Nq, D = q_bits.shape
        Nk = k_bits.shape[2]
    else:
        B, Nq, H, D = q_bits.shape
        Nk = k_bits.shape[1]
    arrs = [np.ascontiguousarray(a, dtype=np.uint16) for a in (q_bits, k_bits, v_bits)]
    L = lib()
    res, jobs = {}, []
    for (b, h), rows in rows_by_head.items():
        r = np.ascontiguousarray(rows, dtype=np.int32)
        o = np.empty((len(r), D), dtype=np.float64)
        res[(b, h)] = o
        jobs.append(lambda b=b, h=h, r=r, o=o: L.orc_exact_rows(
            _p(arrs[0]), _p(arrs[1]), _p(arrs[2]), in_dtype, layout, B, H, Nq, Nk, D, int(causal),
            float(softmax_scale), b, h, _p(r), len(r), _p(o)))
    _run_all(jobs)
    return res


# ---------------------------------------------------------------------------
# Decode
# ---------------------------------------------------------------------------

def decode(q_bits, k, v, k_scales, v_scales, kv_dtype: int, Hkv: int, heads=None, kv_block=256,
           group=128, softmax_scale=0.0, splits=1, want_f64=False):
    """Decode outputs for the listed (b, h_q) pairs (default: all).

    Returns (bf16 bits [B, Hq, 1, D] with unlisted rows zero, f64 or None)."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    B, Hq, _, D = q_bits.shape
    L_ = k.shape[2]
    arrs = [np.ascontiguousarray(a) for a in (k, v, k_scales, v_scales)]
    out = np.zeros((B, Hq, 1, D), dtype=np.uint16)
    of = np.zeros((B, Hq, 1, D), dtype=np.float64) if want_f64 else None
    hs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    Lb = lib()
    jobs = []
    for (b, h) in hs:
        ob = out[b, h, 0]
        fb = of[b, h, 0] if of is not None else None
        jobs.append(lambda b=b, h=h, ob=ob, fb=fb: Lb.orc_decode_one(
            _p(q_bits), _p(arrs[0]), _p(arrs[1]), _p(arrs[2]), _p(arrs[3]), kv_dtype, B, Hq, Hkv, L_,
            D, kv_block, group, float(softmax_scale), splits, b, h, _p(ob), _p(fb)))
    _run_all(jobs)
    return out, of


# ---------------------------------------------------------------------------
# KV-cache quantize-on-append
# ---------------------------------------------------------------------------

def f32_to_f16_bits(x: float) -> int:
    return int(lib().orc_f32_to_f16(float(x)))


def kv_append(x_bits: np.ndarray, cache: np.ndarray, scales: np.ndarray, L: int, kv_dtype: int,
              kv_block: int = 256, group: int = 128):
    """Appends x (bf16 bits [B, H_kv, n, D]) at token L of a quantized cache.

    INT8: cache int8 [B, H_kv, L_max, D], scales float32 [B, H_kv, nblk].
    INT4_PACKED: cache uint8 [B, H_kv, L_max, D/2], scales fp16 bits (uint16)
    [B, H_kv, L_max, D/group]. Returns updated copies (cache, scales)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    B, Hkv, n, D = x_bits.shape
    Lmax = cache.shape[2]
    cache = np.ascontiguousarray(cache).copy()
    scales = np.ascontiguousarray(scales).copy()
    L_ = lib()
    if kv_dtype == INT8:
        assert cache.dtype == np.int8 and scales.dtype == np.float32
        fn = lambda b, h: L_.orc_kv_append_int8(_p(x_bits), B, Hkv, n, D, L, Lmax, kv_block, _p(cache),
                                                 _p(scales), b, h)
    else:
        assert cache.dtype == np.uint8 and scales.dtype == np.uint16
        fn = lambda b, h: L_.orc_kv_append_int4(_p(x_bits), B, Hkv, n, D, L, Lmax, group, _p(cache),
                                                 _p(scales), b, h)
    jobs = [(lambda b=b, h=h: fn(b, h)) for b in range(B) for h in range(Hkv)]
    _run_all(jobs)
    return cache, scales
