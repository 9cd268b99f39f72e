"""qattn_decode_kvq_noalloc: decode with the split partials in the
library's fixed device array, for callers that cannot allocate device memory
on their decode path (memory reserved up front by an allocator they do not
own, or a decode loop where a cudaMalloc/cudaFree could synchronise the
device). It must give the same output as qattn_decode_kvq with a caller
workspace, call after call, and refuse sizes whose partials do not fit.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import MAX_ABS_TOL, MEAN_ABS_TOL

pytestmark = pytest.mark.gpu


def _inputs(p):
    d = synth.make_decode(p)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    q = dev(d["q"].view(np.int16)).view(torch.bfloat16)
    k, v = dev(d["k"]), dev(d["v"])
    if p.kv_dtype == synth.INT8:
        ks, vs, kv = dev(d["k_scales"]), dev(d["v_scales"]), qa.QATTN_INT8
        vmax = float(np.abs(d["v"].astype(np.float64)).max() * d["v_scales"].max())
    else:
        ks = dev(d["k_scales"].view(np.int16)).view(torch.float16)
        vs = dev(d["v_scales"].view(np.int16)).view(torch.float16)
        kv = qa.QATTN_INT4_PACKED
        vmax = 8.0 * float(d["v_scales"].view(np.float16).astype(np.float64).max())
    return q, k, v, ks, vs, kv, vmax


def _noalloc_c(q, k, v, ks, vs, kv, p, out):
    """Direct call through the C ABI."""
    L = qa.lib()
    return L.qattn_decode_kvq_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), ks.data_ptr(), vs.data_ptr(), kv,
                                      p.B, p.Hq, p.Hkv, p.L, p.D, p.kv_block, p.group, C.c_float(0.0),
                                      out.data_ptr(), C.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("kv_dtype", [synth.INT8, synth.INT4_PACKED])
def test_noalloc_matches_workspace_entry_point_twice(kv_dtype):
    base = synth.INT8_KV_DECODE if kv_dtype == synth.INT8 else synth.INT4_KV_DECODE
    p = synth.scaled(base, B=8, L=3000, seed=90 + kv_dtype)
    q, k, v, ks, vs, kv, vmax = _inputs(p)
    assert qa.qattn_decode_workspace_size(p.B, p.Hq, p.Hkv, p.L, p.D) <= qa.NOALLOC_SCRATCH_BYTES
    ref = qa.qattn_decode_kvq(q, k, v, ks, vs, kv, kv_block=p.kv_block, group=p.group)
    torch.cuda.synchronize()
    for _ in range(2):                                    # two calls in a row share the array
        out = torch.full_like(ref, float("nan"))
        assert _noalloc_c(q, k, v, ks, vs, kv, p, out) == qa.QATTN_OK
        torch.cuda.synchronize()
        assert qa.qattn_device_error() == qa.QATTN_OK
        err = (out.float() - ref.float()).abs()
        assert float(err.max()) <= MAX_ABS_TOL * vmax
        assert float(err.mean()) <= MEAN_ABS_TOL * vmax


def test_noalloc_rejects_sizes_beyond_its_scratch():
    p = synth.scaled(synth.INT8_KV_DECODE, B=256, L=8192)    # partials need more than 4 MiB
    assert qa.qattn_decode_workspace_size(p.B, p.Hq, p.Hkv, p.L, p.D) > qa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((p.B, p.Hq, 1, p.D), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1,), dtype=torch.int8, device="cuda")      # never read: rejected first
    s = torch.zeros((1,), dtype=torch.float32, device="cuda")
    out = torch.zeros((p.B, p.Hq, 1, p.D), dtype=torch.bfloat16, device="cuda")
    pp = synth.scaled(p)
    assert _noalloc_c(q, k, k, s, s, qa.QATTN_INT8, pp, out) == qa.QATTN_ERR_WORKSPACE
    with pytest.raises(qa.QAttnError) as e:
        qa.qattn_decode_kvq_noalloc(q, torch.zeros((p.B, p.Hkv, p.L, 0), dtype=torch.int8, device="cuda"),
                                    k, s, s, qa.QATTN_INT8)
    assert e.value.status in (qa.QATTN_ERR_WORKSPACE, qa.QATTN_ERR_INVALID_ARG)
