"""Shared helpers for the GPU parity tests: move synthetic inputs to the
device, run the CUDA path through the C ABI, run the oracle on the same
inputs, compare."""
import numpy as np
import torch

import block_quantized_precision_b200 as qa
import synth

# Attention tolerance (relative to max |V| of the head, V dequantized).
MAX_ABS_TOL = 1e-2
MEAN_ABS_TOL = 1e-3


def dev_bits(bits: np.ndarray, in_dtype: int) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16 if in_dtype == synth.BF16 else torch.float16)


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_quant_all(d: dict):
    """CUDA path: rotate+quantize Q (blocks of 128), K (256), V (256, no
    rotation). Returns device tensors (codes, scales) x 3."""
    p = d["problem"]
    rot = dev(d["rot"]) if d["rot"] is not None else None
    out = []
    for name, blk, r in (("q", p.q_block, rot), ("k", p.kv_block, rot), ("v", p.kv_block, None)):
        x = dev_bits(d[name], p.in_dtype)
        out.append(qa.qattn_rotate_block_quant(x, p.layout, r, blk, p.code_dtype))
    torch.cuda.synchronize()
    return out


def head_rows(x, layout, b, h):
    return x[b, h] if layout == synth.BNSD else x[b, :, h]


def dequant_v_max(vc: np.ndarray, vs: np.ndarray, code_dtype: int, layout: int, b: int, h: int, orc) -> float:
    codes = head_rows(vc, layout, b, h)
    if code_dtype == synth.INT8:
        vals = np.abs(codes.view(np.int8).astype(np.float64))
    elif code_dtype == synth.INT4_PACKED:
        lo = ((codes & 0xF).astype(np.int16) ^ 8) - 8
        hi = ((codes >> 4).astype(np.int16) ^ 8) - 8
        vals = np.abs(np.concatenate([lo, hi], axis=1).astype(np.float64))
    else:
        vals = np.abs(orc.e4m3_decode(codes).astype(np.float64))
    per_tok = vals.max(axis=1)
    n = len(per_tok)
    blk = np.arange(n) // 256
    return float((per_tok * vs[b, h, blk].astype(np.float64)).max())


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, vmax: float, what: str):
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS_TOL * vmax, "%s: max-abs %.3g > %.3g" % (what, err.max(), MAX_ABS_TOL * vmax)
    assert err.mean() <= MEAN_ABS_TOL * vmax, "%s: mean-abs %.3g > %.3g" % (what, err.mean(), MEAN_ABS_TOL * vmax)
    return float(err.max() / vmax), float(err.mean() / vmax)
