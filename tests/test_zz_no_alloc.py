"""qattn_decode_kvq_noalloc: decode with the split partials in the
library's fixed 16 MiB device array, for callers that cannot allocate device
memory on their decode path (memory reserved up front by an allocator they
do not own, or a decode loop where a cudaMalloc/cudaFree could synchronise
the device). It runs the same kernels with the same split count as
qattn_decode_kvq with a caller workspace, so its output must be the same
bytes, call after call, and it must refuse sizes whose partials do not fit.

The two calls in a row take different inputs and different split counts,
each compared with its own workspace run: a call that read partials left in
the array by the call before would show up here.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth

pytestmark = pytest.mark.gpu


def _inputs(p):
    d = synth.make_decode(p)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    q = dev(d["q"].view(np.int16)).view(torch.bfloat16)
    k, v = dev(d["k"]), dev(d["v"])
    if p.kv_dtype == synth.INT8:
        ks, vs, kv = dev(d["k_scales"]), dev(d["v_scales"]), qa.QATTN_INT8
    else:
        ks = dev(d["k_scales"].view(np.int16)).view(torch.float16)
        vs = dev(d["v_scales"].view(np.int16)).view(torch.float16)
        kv = qa.QATTN_INT4_PACKED
    return q, k, v, ks, vs, kv


def _noalloc_c(q, k, v, ks, vs, kv, p, out):
    """Direct call through the C ABI."""
    L = qa.lib()
    return L.qattn_decode_kvq_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), ks.data_ptr(), vs.data_ptr(), kv,
                                      p.B, p.Hq, p.Hkv, p.L, p.D, p.kv_block, p.group, C.c_float(0.0),
                                      out.data_ptr(), C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _bits(t):
    return t.view(torch.int16).cpu().numpy()


def _check_against_workspace_call(p):
    q, k, v, ks, vs, kv = _inputs(p)
    ref = qa.qattn_decode_kvq(q, k, v, ks, vs, kv, kv_block=p.kv_block, group=p.group)
    torch.cuda.synchronize()
    out = torch.full_like(ref, float("nan"))
    assert _noalloc_c(q, k, v, ks, vs, kv, p, out) == qa.QATTN_OK
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    assert np.array_equal(_bits(out), _bits(ref))


@pytest.mark.parametrize("kv_dtype", [synth.INT8, synth.INT4_PACKED])
def test_noalloc_matches_workspace_entry_point_twice(kv_dtype):
    base = synth.INT8_KV_DECODE if kv_dtype == synth.INT8 else synth.INT4_KV_DECODE
    first = synth.scaled(base, B=8, L=3000, seed=90 + kv_dtype)
    second = synth.scaled(base, B=4, L=700, seed=190 + kv_dtype)      # fewer splits, other values
    for p in (first, second):
        _check_against_workspace_call(p)


def test_noalloc_full_size_int8_decode():
    """The stated INT8 decode problem (B=64, H_q=32, L=8192: 8.25 MiB of
    partials) fits the array and matches the workspace call bit for bit."""
    p = synth.INT8_KV_DECODE
    assert qa.qattn_decode_workspace_size(p.B, p.Hq, p.Hkv, p.L, p.D) <= qa.NOALLOC_SCRATCH_BYTES
    _check_against_workspace_call(p)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    p = synth.scaled(synth.INT8_KV_DECODE, B=1024, L=8192)   # partials: more than 16 MiB
    assert qa.qattn_decode_workspace_size(p.B, p.Hq, p.Hkv, p.L, p.D) > qa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((p.B, p.Hq, 1, p.D), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1,), dtype=torch.int8, device="cuda")      # never read: rejected first
    s = torch.zeros((1,), dtype=torch.float32, device="cuda")
    out = torch.zeros((p.B, p.Hq, 1, p.D), dtype=torch.bfloat16, device="cuda")
    assert _noalloc_c(q, k, k, s, s, qa.QATTN_INT8, p, out) == qa.QATTN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
