"""Python binding of libqattn (block-quantized attention for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/qattn.h. PyTorch provides device
memory and streams. There is no fallback: if libqattn.so is missing or a call
fails, an exception is raised.

Function names follow the C ABI:
    qattn_rotate_block_quant, qattn_rotate_block_quant_qkv, qattn_prefill, qattn_prefill_mixed,
    qattn_widen_int4, qattn_dequant_bf16,
    qattn_attention_bf16, qattn_decode_workspace_size,
    qattn_decode_kvq, qattn_decode_kvq_noalloc, qattn_kv_append, qattn_device_error,
    qattn_selftest_wait_timeout,
    qattn_abi_version, qattn_status_string.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqattn.so")

# Enumerations of include/qattn.h
QATTN_OK = 0
QATTN_ERR_INVALID_ARG = 1
QATTN_ERR_UNSUPPORTED = 2
QATTN_ERR_ALIGNMENT = 3
QATTN_ERR_WORKSPACE = 4
QATTN_ERR_CUDA = 5
QATTN_ERR_TIMEOUT = 6

QATTN_BNSD, QATTN_BSND = 0, 1
QATTN_F16, QATTN_BF16, QATTN_INT8, QATTN_FP8_E4M3, QATTN_INT4_PACKED = 0, 1, 2, 3, 4

EXPORTED = ("qattn_abi_version", "qattn_status_string", "qattn_rotate_block_quant", "qattn_rotate_block_quant_qkv",
            "qattn_prefill",
            "qattn_prefill_mixed", "qattn_widen_int4", "qattn_dequant_bf16", "qattn_attention_bf16",
            "qattn_decode_workspace_size", "qattn_decode_kvq", "qattn_decode_kvq_noalloc", "qattn_kv_append",
            "qattn_attention_path_host_workspace_size", "qattn_attention_path_host",
            "qattn_device_error", "qattn_selftest_wait_timeout")

# Fixed scratch of qattn_decode_kvq_noalloc (bytes).
NOALLOC_SCRATCH_BYTES = 16 << 20

_lib = None


class QAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


def lib() -> C.CDLL:
    """Loads libqattn.so from this package directory (raises if absent)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libqattn.so not built; run `python -m block_quantized_precision_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, i, f, z = C.c_void_p, C.c_int, C.c_float, C.c_size_t
        L.qattn_abi_version.restype = i
        L.qattn_status_string.argtypes, L.qattn_status_string.restype = [i], C.c_char_p
        L.qattn_rotate_block_quant.argtypes = [P, i, i, i, i, i, i, P, i, i, P, P, P]
        L.qattn_rotate_block_quant.restype = i
        L.qattn_rotate_block_quant_qkv.argtypes = [P, P, P, i, i, i, i, i, i, P, i, P, P, P, P, P, P, P]
        L.qattn_rotate_block_quant_qkv.restype = i
        L.qattn_prefill.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, i, i, i, i, f, P, P, P]
        L.qattn_prefill.restype = i
        L.qattn_prefill_mixed.argtypes = [P, P, P, P, P, P, i, i, i, i, i, i, i, i, i, i, i, f, P, P, P]
        L.qattn_prefill_mixed.restype = i
        L.qattn_widen_int4.argtypes, L.qattn_widen_int4.restype = [P, C.c_int64, P, P], i
        L.qattn_dequant_bf16.argtypes = [P, P, i, i, i, i, i, i, i, P, P]
        L.qattn_dequant_bf16.restype = i
        L.qattn_attention_bf16.argtypes = [P, P, P, i, i, i, i, i, i, i, f, P, P, P]
        L.qattn_attention_bf16.restype = i
        L.qattn_decode_workspace_size.argtypes, L.qattn_decode_workspace_size.restype = [i, i, i, i, i], z
        L.qattn_decode_kvq.argtypes = [P, P, P, P, P, i, i, i, i, i, i, i, i, f, P, P, z, P]
        L.qattn_decode_kvq.restype = i
        L.qattn_decode_kvq_noalloc.argtypes = [P, P, P, P, P, i, i, i, i, i, i, i, i, f, P, P]
        L.qattn_decode_kvq_noalloc.restype = i
        L.qattn_kv_append.argtypes = [P, i, i, i, i, i, i, i, P, P, i, i, P]
        L.qattn_kv_append.restype = i
        L.qattn_attention_path_host_workspace_size.argtypes = [i, i, i, i, i, i]
        L.qattn_attention_path_host_workspace_size.restype = z
        L.qattn_attention_path_host.argtypes = [P, P, P, i, i, i, i, i, i, P, i, i, f, P, i, P, z, P]
        L.qattn_attention_path_host.restype = i
        L.qattn_device_error.argtypes, L.qattn_device_error.restype = [P], i
        L.qattn_selftest_wait_timeout.argtypes, L.qattn_selftest_wait_timeout.restype = [i, P], i
        _lib = L
    return _lib


def qattn_abi_version() -> int:
    return int(lib().qattn_abi_version())


def status_string(status: int) -> str:
    return lib().qattn_status_string(int(status)).decode()


qattn_status_string = status_string


def _check(status: int, where: str):
    if status != QATTN_OK:
        raise QAttnError(status, where)


def _ptr(t) -> Optional[int]:
    """Address of a host tensor (or None)."""
    return None if t is None else t.data_ptr()


def _dptr(t) -> Optional[int]:
    """Address of a device tensor (or None). The kernels read and write the
    dense row-major extent from that address, so a tensor on the host or a
    strided view is refused here instead of being read out of bounds."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor, got one on %s" % t.device)
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor (shape %s, strides %s)" % (tuple(t.shape), t.stride()))
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dims(x, layout):
    if layout == QATTN_BNSD:
        B, H, N, D = x.shape
    else:
        B, N, H, D = x.shape
    return B, H, N, D


def qattn_rotate_block_quant(x, layout: int, rot, block_tokens: int, code_dtype: int,
                             codes=None, scales=None, stream=None):
    """Rotation (optional) + dynamic block quantization of one tensor.

    x: CUDA bfloat16/float16 tensor in `layout`; rot: CUDA float32 [D, D] or
    None. Returns (codes uint8 like x -- [..., D/2] for QATTN_INT4_PACKED --,
    scales float32 [B, H, nblk])."""
    import torch
    B, H, N, D = _dims(x, layout)
    x_dtype = {torch.bfloat16: QATTN_BF16, torch.float16: QATTN_F16}[x.dtype]
    nblk = -(-N // block_tokens)
    if codes is None:
        shape = tuple(x.shape[:-1]) + ((D // 2,) if code_dtype == QATTN_INT4_PACKED else (D,))
        codes = torch.empty(shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((B, H, nblk), dtype=torch.float32, device=x.device)
    st = lib().qattn_rotate_block_quant(_dptr(x), x_dtype, layout, B, H, N, D, _dptr(rot), block_tokens,
                                        code_dtype, _dptr(codes), _dptr(scales), _stream(stream))
    _check(st, "qattn_rotate_block_quant")
    return codes, scales


def qattn_rotate_block_quant_qkv(q, k, v, layout: int, rot, code_dtype: int, out=None, stream=None):
    """The quantizations of one prefill at once: Q (blocks of 128) and K
    (256) rotated by rot (or not, rot=None), V (256) not rotated; the two
    rotations run concurrently. Returns ((q codes, scales), (k ...), (v ...));
    `out` may pass those six tensors to fill instead."""
    import torch
    B, H, N, D = _dims(q, layout)
    x_dtype = {torch.bfloat16: QATTN_BF16, torch.float16: QATTN_F16}[q.dtype]
    for t in (k, v):
        if t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v must have one shape and dtype")
    if out is None:
        shape = tuple(q.shape[:-1]) + ((D // 2,) if code_dtype == QATTN_INT4_PACKED else (D,))
        out = []
        for blk in (128, 256, 256):
            out.append((torch.empty(shape, dtype=torch.uint8, device=q.device),
                        torch.empty((B, H, -(-N // blk)), dtype=torch.float32, device=q.device)))
    (qc, qs), (kc, ks), (vc, vs) = out
    st = lib().qattn_rotate_block_quant_qkv(_dptr(q), _dptr(k), _dptr(v), x_dtype, layout, B, H, N, D, _dptr(rot),
                                            code_dtype, _dptr(qc), _dptr(qs), _dptr(kc), _dptr(ks), _dptr(vc), _dptr(vs),
                                            _stream(stream))
    _check(st, "qattn_rotate_block_quant_qkv")
    return out


def qattn_prefill(q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, code_dtype: int, layout: int,
                  causal: bool, softmax_scale: float = 0.0, out=None, lse=None, q_block: int = 128,
                  kv_block: int = 256, stream=None):
    """Quantized attention over codes; returns the bfloat16 output (layout of Q)."""
    import torch
    B, H, Nq, D = _dims(q_codes, layout)
    Nkv = _dims(k_codes, layout)[2]
    if out is None:
        out = torch.empty(q_codes.shape, dtype=torch.bfloat16, device=q_codes.device)
    st = lib().qattn_prefill(_dptr(q_codes), _dptr(q_scales), _dptr(k_codes), _dptr(k_scales), _dptr(v_codes),
                             _dptr(v_scales), code_dtype, layout, B, H, Nq, Nkv, D, q_block, kv_block,
                             int(bool(causal)), float(softmax_scale), _dptr(out), _dptr(lse), _stream(stream))
    _check(st, "qattn_prefill")
    return out


def qattn_prefill_mixed(q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, qk_dtype: int, v_dtype: int,
                        layout: int, causal: bool, softmax_scale: float = 0.0, out=None, lse=None,
                        q_block: int = 128, kv_block: int = 256, stream=None):
    """Quantized attention with V in its own code type (packed INT4 codes:
    [..., D/2] bytes); returns the bfloat16 output (layout of Q, D channels)."""
    import torch
    B, H, Nq, D = _dims(q_codes, layout)
    if qk_dtype == QATTN_INT4_PACKED:
        D *= 2
    Nkv = _dims(k_codes, layout)[2]
    if out is None:
        out = torch.empty(tuple(q_codes.shape[:-1]) + (D,), dtype=torch.bfloat16, device=q_codes.device)
    st = lib().qattn_prefill_mixed(_dptr(q_codes), _dptr(q_scales), _dptr(k_codes), _dptr(k_scales), _dptr(v_codes),
                                   _dptr(v_scales), qk_dtype, v_dtype, layout, B, H, Nq, Nkv, D, q_block,
                                   kv_block, int(bool(causal)), float(softmax_scale), _dptr(out), _dptr(lse),
                                   _stream(stream))
    _check(st, "qattn_prefill_mixed")
    return out


def qattn_widen_int4(packed, out=None, stream=None):
    """Packed INT4 codes ([..., D/2] bytes) widened to INT8 codes ([..., D]
    bytes, int8 values -8..7, the same block scales apply)."""
    import torch
    if out is None:
        out = torch.empty(tuple(packed.shape[:-1]) + (2 * packed.shape[-1],), dtype=torch.uint8,
                          device=packed.device)
    n = packed.numel() * packed.element_size()
    if not (packed.is_contiguous() and out.is_contiguous()) or out.numel() * out.element_size() != 2 * n:
        raise ValueError("qattn_widen_int4: contiguous tensors of n and 2n bytes expected")
    st = lib().qattn_widen_int4(_dptr(packed), n, _dptr(out), _stream(stream))
    _check(st, "qattn_widen_int4")
    return out


def qattn_dequant_bf16(codes, scales, code_dtype: int, layout: int, block_tokens: int, out=None, stream=None):
    """The dequantize pass of the comparison path: bfloat16 code * block
    scale, same layout as the codes (INT8 or e4m3)."""
    import torch
    B, H, N, D = _dims(codes, layout)
    if out is None:
        out = torch.empty(codes.shape, dtype=torch.bfloat16, device=codes.device)
    st = lib().qattn_dequant_bf16(_dptr(codes), _dptr(scales), code_dtype, layout, B, H, N, D, block_tokens, _dptr(out),
                                  _stream(stream))
    _check(st, "qattn_dequant_bf16")
    return out


def qattn_attention_bf16(q, k, v, layout: int, causal: bool, softmax_scale: float = 0.0, out=None, lse=None,
                         stream=None):
    """Attention over bfloat16 Q/K/V on the 16-bit tensor-core path (the
    comparison path's second step); returns the bfloat16 output."""
    import torch
    B, H, Nq, D = _dims(q, layout)
    Nkv = _dims(k, layout)[2]
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    st = lib().qattn_attention_bf16(_dptr(q), _dptr(k), _dptr(v), layout, B, H, Nq, Nkv, D, int(bool(causal)),
                                    float(softmax_scale), _dptr(out), _dptr(lse), _stream(stream))
    _check(st, "qattn_attention_bf16")
    return out


def qattn_attention_path_host_workspace_size(B: int, H: int, N: int, D: int, layout: int, groups: int = 0) -> int:
    return int(lib().qattn_attention_path_host_workspace_size(B, H, N, D, layout, groups))


def qattn_attention_path_host(q, k, v, rot, layout: int, code_dtype: int, causal: bool, softmax_scale: float = 0.0,
                              out=None, groups: int = 0, workspace=None, stream=None):
    """The whole prefill path (rotate + quantize Q/K, quantize V, attention)
    from HOST tensors: q, k, v are CPU bfloat16/float16 tensors (pinned for
    the copies to overlap the compute), rot a CUDA float32 [D, D] tensor or
    None. Returns `out`, a CPU bfloat16 tensor in the layout of q, complete
    once `stream` has reached the end of the call's work."""
    import torch
    B, H, N, D = _dims(q, layout)
    x_dtype = {torch.bfloat16: QATTN_BF16, torch.float16: QATTN_F16}[q.dtype]
    for t in (q, k, v):
        if t.is_cuda or not t.is_contiguous() or t.shape != q.shape or t.dtype != q.dtype:
            raise ValueError("q, k, v must be contiguous CPU tensors of one shape and dtype")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=q.is_pinned())
    dev = rot.device if rot is not None else torch.device("cuda", torch.cuda.current_device())
    need = qattn_attention_path_host_workspace_size(B, H, N, D, layout, groups)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = lib().qattn_attention_path_host(_ptr(q), _ptr(k), _ptr(v), x_dtype, layout, B, H, N, D, _dptr(rot),
                                         code_dtype, int(bool(causal)), float(softmax_scale), _ptr(out),
                                         int(groups), _dptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "qattn_attention_path_host")
    return out


def qattn_decode_workspace_size(B: int, H_q: int, H_kv: int, L: int, D: int) -> int:
    return int(lib().qattn_decode_workspace_size(B, H_q, H_kv, L, D))


def qattn_decode_kvq(q, k_cache, v_cache, k_scales, v_scales, kv_dtype: int, kv_block: int = 256,
                     group: int = 128, softmax_scale: float = 0.0, out=None, workspace=None, stream=None):
    """One decode step against an INT8 / packed-INT4 KV cache.

    q: bfloat16 [B, H_q, 1, D]; caches [B, H_kv, L, D] (INT8) or
    [B, H_kv, L, D/2] (INT4). Returns the bfloat16 output [B, H_q, 1, D]."""
    import torch
    B, Hq, _, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty((B, Hq, 1, D), dtype=torch.bfloat16, device=q.device)
    need = qattn_decode_workspace_size(B, Hq, Hkv, L, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().qattn_decode_kvq(_dptr(q), _dptr(k_cache), _dptr(v_cache), _dptr(k_scales), _dptr(v_scales), kv_dtype,
                                B, Hq, Hkv, L, D, kv_block, group, float(softmax_scale), _dptr(out),
                                _dptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "qattn_decode_kvq")
    return out


def qattn_decode_kvq_noalloc(q, k_cache, v_cache, k_scales, v_scales, kv_dtype: int, kv_block: int = 256,
                             group: int = 128, softmax_scale: float = 0.0, out=None, stream=None):
    """qattn_decode_kvq with the split partials in the library's fixed 16 MiB
    device array instead of a caller workspace: for callers that cannot
    allocate device memory on their decode path. Calls must not overlap on
    the GPU (they share the array); make the first call on a device before
    any stream capture, and none after a cudaDeviceReset() on it. The output tensor is the caller's: pass `out` to
    avoid allocating it here."""
    import torch
    B, Hq, _, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty((B, Hq, 1, D), dtype=torch.bfloat16, device=q.device)
    st = lib().qattn_decode_kvq_noalloc(_dptr(q), _dptr(k_cache), _dptr(v_cache), _dptr(k_scales), _dptr(v_scales),
                                        kv_dtype, B, Hq, Hkv, L, D, kv_block, group, float(softmax_scale),
                                        _dptr(out), _stream(stream))
    _check(st, "qattn_decode_kvq_noalloc")
    return out


def qattn_kv_append(x_new, cache, scales, L: int, kv_dtype: int, kv_block: int = 256, group: int = 128,
                    stream=None):
    """Quantizes x_new (bf16 [B, H_kv, n, D]) into the cache at tokens
    [L, L + n), in place. INT8: cache int8 [B, H_kv, L_max, D], scales
    float32 [B, H_kv, ceil(L_max / kv_block)]. INT4_PACKED: cache uint8
    [B, H_kv, L_max, D/2], scales float16 [B, H_kv, L_max, D/group]."""
    B, Hkv, n, D = x_new.shape
    Lmax = cache.shape[2]
    st = lib().qattn_kv_append(_dptr(x_new), B, Hkv, n, D, kv_dtype, int(L), Lmax, _dptr(cache), _dptr(scales),
                               kv_block, group, _stream(stream))
    _check(st, "qattn_kv_append")
    return cache, scales


def qattn_device_error(stream=None) -> int:
    """Synchronises the stream; returns and clears the device error word."""
    return int(lib().qattn_device_error(_stream(stream)))


def qattn_selftest_wait_timeout(timeout_ms: int, stream=None):
    _check(lib().qattn_selftest_wait_timeout(int(timeout_ms), _stream(stream)), "qattn_selftest_wait_timeout")
