"""qattn_attention_path_host: the prefill path from host buffers, with the
copies of one group of heads overlapped with the compute of another, gives
the same bytes as the four device calls (rotate + quantize Q and K, quantize
V, prefill) on the whole problem -- for both layouts, ragged N, uneven head
groups and groups that take part of the heads of one b. The device calls
themselves are compared with the oracle in test_gpu_prefill.py."""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import dev, dev_bits

pytestmark = pytest.mark.gpu


def _host(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


def _device_path(p, d):
    rot = dev(d["rot"]) if d["rot"] is not None else None
    qc = qa.qattn_rotate_block_quant(dev_bits(d["q"], p.in_dtype), p.layout, rot, 128, p.code_dtype)
    kc = qa.qattn_rotate_block_quant(dev_bits(d["k"], p.in_dtype), p.layout, rot, 256, p.code_dtype)
    vc = qa.qattn_rotate_block_quant(dev_bits(d["v"], p.in_dtype), p.layout, None, 256, p.code_dtype)
    out = qa.qattn_prefill(*qc, *kc, *vc, p.code_dtype, p.layout, p.causal)
    torch.cuda.synchronize()
    return out.cpu()


CASES = [
    # (B, H, N, D, layout, code, causal, groups)
    (2, 5, 700, 128, synth.BNSD, synth.INT8, True, [1, 3, 0, 10]),
    (2, 6, 300, 64, synth.BSND, synth.FP8_E4M3, False, [1, 2, 5, 12]),
    (3, 4, 129, 128, synth.BSND, synth.INT8, True, [2, 7]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dN%dD%d_%s" % (c[0], c[1], c[2], c[3],
                                                                          "bnsd" if c[4] == synth.BNSD else "bsnd"))
def test_same_bytes_as_device_calls(case):
    B, H, N, D, layout, code, causal, groups = case
    p = synth.PrefillProblem("host", B, H, N, D, synth.BF16, code, layout, causal=causal, rotate=True,
                             seed=900 + B + H + N + D, outlier_frac=0.01)
    d = synth.make_prefill(p)
    want = _device_path(p, d)
    q, k, v = _host(d["q"]), _host(d["k"]), _host(d["v"])
    rot = dev(d["rot"])
    for g in groups:
        out = qa.qattn_attention_path_host(q, k, v, rot, layout, code, causal, groups=g)
        torch.cuda.synchronize()
        assert out.shape == want.shape
        assert torch.equal(out.view(torch.int16), want.view(torch.int16)), "groups=%d" % g
    assert qa.qattn_device_error() == qa.QATTN_OK


def test_pageable_host_memory_and_no_rotation():
    p = synth.PrefillProblem("host", 1, 3, 260, 128, synth.BF16, synth.INT8, synth.BNSD, causal=False,
                             rotate=False, seed=950)
    d = synth.make_prefill(p)
    want = _device_path(p, d)
    q, k, v = (torch.from_numpy(np.ascontiguousarray(d[n]).view(np.int16)).view(torch.bfloat16)
               for n in ("q", "k", "v"))
    out = qa.qattn_attention_path_host(q, k, v, None, p.layout, p.code_dtype, p.causal, groups=2)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))


def test_f16_inputs():
    """fp16 Q/K/V through the host path: the same bytes as the device calls."""
    p = synth.PrefillProblem("host", 1, 4, 333, 128, synth.F16, synth.INT8, synth.BNSD, causal=True,
                             rotate=True, seed=960)
    d = synth.make_prefill(p)
    rot = dev(d["rot"])
    codes = [qa.qattn_rotate_block_quant(dev_bits(d[n], p.in_dtype), p.layout, r, blk, p.code_dtype)
             for n, blk, r in (("q", 128, rot), ("k", 256, rot), ("v", 256, None))]
    want = qa.qattn_prefill(*codes[0], *codes[1], *codes[2], p.code_dtype, p.layout, p.causal)
    torch.cuda.synchronize()
    host = [torch.from_numpy(np.ascontiguousarray(d[n]).view(np.int16)).view(torch.float16).pin_memory()
            for n in ("q", "k", "v")]
    out = qa.qattn_attention_path_host(*host, rot, p.layout, p.code_dtype, p.causal, groups=3)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), want.cpu().view(torch.int16))


def test_small_workspace_is_rejected():
    q = torch.zeros((1, 2, 128, 128), dtype=torch.bfloat16).pin_memory()
    need = qa.qattn_attention_path_host_workspace_size(1, 2, 128, 128, qa.QATTN_BNSD, 2)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(qa.QAttnError) as e:
        qa.qattn_attention_path_host(q, q, q, None, qa.QATTN_BNSD, qa.QATTN_INT8, True, groups=2, workspace=ws)
    assert e.value.status == qa.QATTN_ERR_WORKSPACE
