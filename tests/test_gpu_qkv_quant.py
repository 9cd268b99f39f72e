"""qattn_rotate_block_quant_qkv: the three quantizations of a prefill in one
call (the two rotations concurrently on internal streams) give the same
codes and scales, bit for bit, as three qattn_rotate_block_quant calls --
which test_gpu_rotate_quant.py compares with the oracle -- and are ordered
on the caller's stream like any stream-ordered call."""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import dev, dev_bits

pytestmark = pytest.mark.gpu


def _three_calls(x, rot, p, code):
    return [qa.qattn_rotate_block_quant(x[n], p.layout, rot if n != "v" else None, blk, code)
            for n, blk in (("q", 128), ("k", 256), ("v", 256))]


def _same(a, b):
    for (ca, sa), (cb, sb) in zip(a, b):
        assert torch.equal(ca, cb)
        assert np.array_equal(sa.cpu().numpy().view(np.uint32), sb.cpu().numpy().view(np.uint32))


@pytest.mark.parametrize("code", [synth.INT8, synth.FP8_E4M3, synth.INT4_PACKED])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("rotate", [True, False])
def test_same_bytes_as_three_calls(code, layout, rotate):
    p = synth.PrefillProblem("qkv", 2, 5, 700, 128, synth.BF16, synth.INT8, layout, causal=False, rotate=True,
                             seed=800 + code + 3 * layout + rotate, outlier_frac=0.01)
    d = synth.make_prefill(p)
    x = {n: dev_bits(d[n], p.in_dtype) for n in ("q", "k", "v")}
    rot = dev(d["rot"]) if rotate else None
    want = _three_calls(x, rot, p, code)
    got = qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], layout, rot, code)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    _same(got, want)


def test_full_size_int8_causal_problem():
    p = synth.INT8_CAUSAL
    d = synth.make_prefill(p)
    x = {n: dev_bits(d[n], p.in_dtype) for n in ("q", "k", "v")}
    rot = dev(d["rot"])
    want = _three_calls(x, rot, p, p.code_dtype)
    got = qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], p.layout, rot, p.code_dtype)
    torch.cuda.synchronize()
    _same(got, want)


def test_ordered_on_the_callers_stream():
    """On a side stream: the prefill enqueued after the call on the same
    stream sees the finished codes (the stream waits for the internal ones);
    repeated back to back, every result is the same."""
    p = synth.scaled(synth.INT8_CAUSAL, H=8, N=2048, seed=810)
    d = synth.make_prefill(p)
    x = {n: dev_bits(d[n], p.in_dtype) for n in ("q", "k", "v")}
    rot = dev(d["rot"])
    ref_codes = _three_calls(x, rot, p, p.code_dtype)
    ref = qa.qattn_prefill(*ref_codes[0], *ref_codes[1], *ref_codes[2], p.code_dtype, p.layout, p.causal)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(side):
        for _ in range(3):
            codes = qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], p.layout, rot, p.code_dtype, stream=side)
            outs.append(qa.qattn_prefill(*codes[0], *codes[1], *codes[2], p.code_dtype, p.layout, p.causal,
                                         stream=side))
    side.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))


def test_captured_in_a_cuda_graph():
    """The call and a prefill captured as one CUDA graph (the internal
    streams join the capture) and replayed: the same bytes as eager calls,
    replay after replay, on new inputs copied into the captured buffers."""
    p = synth.scaled(synth.INT8_CAUSAL, H=4, N=1024, seed=820)
    d = synth.make_prefill(p)
    x = {n: dev_bits(d[n], p.in_dtype) for n in ("q", "k", "v")}
    rot = dev(d["rot"])
    codes = qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], p.layout, rot, p.code_dtype)   # creates the streams
    out = qa.qattn_prefill(*codes[0], *codes[1], *codes[2], p.code_dtype, p.layout, p.causal)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = torch.cuda.current_stream()
        qa.qattn_rotate_block_quant_qkv(x["q"], x["k"], x["v"], p.layout, rot, p.code_dtype, out=codes, stream=st)
        qa.qattn_prefill(*codes[0], *codes[1], *codes[2], p.code_dtype, p.layout, p.causal, out=out, stream=st)
    for seed in (821, 822):
        d2 = synth.make_prefill(synth.scaled(p, seed=seed))
        x2 = {n: dev_bits(d2[n], p.in_dtype) for n in ("q", "k", "v")}
        want_codes = _three_calls(x2, rot, p, p.code_dtype)
        want = qa.qattn_prefill(*want_codes[0], *want_codes[1], *want_codes[2], p.code_dtype, p.layout, p.causal)
        for n in ("q", "k", "v"):
            x[n].copy_(x2[n])
        g.replay()
        torch.cuda.synchronize()
        assert qa.qattn_device_error() == qa.QATTN_OK
        _same(codes, want_codes)
        assert torch.equal(out.view(torch.int16), want.view(torch.int16))
