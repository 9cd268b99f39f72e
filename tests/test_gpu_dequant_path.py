"""The dequantize-first comparison path ("INT8 量化算子", ops-transformer
items 1-2: the standard INT8 path converts back to FP16 and multiplies in
FP16): qattn_dequant_bf16 then qattn_attention_bf16.

The dequantize pass is checked bit for bit against float32 code * scale
rounded to bfloat16 (numpy, on the oracle's codes). The attention is checked
against float64 attention on exactly those bfloat16 inputs (the oracle's
exact-attention rows): the GPU differs from it only by its float32
accumulation and the bfloat16 rounding of P as an MMA operand."""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import assert_close, bf16_to_f64, gpu_quant_all, head_rows

pytestmark = pytest.mark.gpu


def _dequant_ref(codes, scales, code_dtype, layout, block, orc):
    """bf16 bits of float32(code) * scale (one float32 rounding), RNE to bf16."""
    if code_dtype == synth.INT8:
        vals = codes.view(np.int8).astype(np.float32)
    else:
        vals = orc.e4m3_decode(codes).astype(np.float32)
    if layout == synth.BNSD:
        B, H, N, D = vals.shape
        s = np.repeat(scales, block, axis=2)[:, :, :N, None]
    else:
        B, N, H, D = vals.shape
        s = np.transpose(np.repeat(scales, block, axis=2)[:, :, :N], (0, 2, 1))[..., None]
    return synth.f32_to_bf16_bits((vals * s.astype(np.float32)).astype(np.float32))


@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
def test_dequant_pass_bit_exact(orc, code_dtype, layout):
    """The oracle's codes and scales in, bfloat16 values out, bit for bit."""
    p = synth.PrefillProblem("dq", 2, 3, 300, 128, synth.BF16, code_dtype, layout, causal=False, rotate=True,
                             seed=400 + code_dtype + layout)
    d = synth.make_prefill(p)
    for name, blk, rot in (("q", 128, d["rot"]), ("k", 256, d["rot"]), ("v", 256, None)):
        codes, scales = orc.rotate_block_quant(d[name], p.in_dtype, p.layout, rot, blk, code_dtype)
        got = qa.qattn_dequant_bf16(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(), code_dtype,
                                    layout, blk)
        torch.cuda.synchronize()
        want = _dequant_ref(codes, scales, code_dtype, layout, blk, orc)
        assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16), want)


def _oracle_codes(orc, p, d, heads):
    return (orc.rotate_block_quant(d["q"], p.in_dtype, p.layout, d["rot"], 128, p.code_dtype, heads=heads),
            orc.rotate_block_quant(d["k"], p.in_dtype, p.layout, d["rot"], 256, p.code_dtype, heads=heads),
            orc.rotate_block_quant(d["v"], p.in_dtype, p.layout, None, 256, p.code_dtype, heads=heads))


def _bf16_inputs(orc, p, codes):
    """Codes and scales of Q, K, V dequantized and rounded to bfloat16 (bit
    patterns, the layout of the problem)."""
    return tuple(_dequant_ref(c, s, p.code_dtype, p.layout, blk, orc) for (c, s), blk in zip(codes, (128, 256, 256)))


def _gpu_path(p, codes):
    """The GPU's dequantize pass and bfloat16 attention on the given codes."""
    deq = [qa.qattn_dequant_bf16(torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda(), p.code_dtype, p.layout, blk)
           for (c, s), blk in zip(codes, (128, 256, 256))]
    lse = torch.empty((p.B, p.H, p.N), dtype=torch.float32, device="cuda")
    out = qa.qattn_attention_bf16(*deq, p.layout, p.causal, lse=lse)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    return out.view(torch.int16).cpu().numpy().view(np.uint16), lse.cpu().numpy()


def _run(orc, p, d, rows=None):
    """The GPU's dequantize pass and bfloat16 attention, fed the oracle's
    codes, against float64 attention on the bfloat16 inputs they make (the
    oracle's codes x scales rounded to bfloat16): what the
    dequantize-first path computes, exactly up to its float32 accumulation
    and the bfloat16 rounding of P as an MMA operand. (The bfloat16 rounding
    of the dequantized inputs itself moves large scores -- the outlier
    channels -- by O(1), so the quantized-attention oracle is not the
    reference here.)"""
    heads = [(b, h) for b in range(p.B) for h in range(p.H)] if rows is None else list(rows)
    codes = _oracle_codes(orc, p, d, heads)
    out_bits, lse_np = _gpu_path(p, codes)
    qb_bits, kb_bits, vb_bits = _bf16_inputs(orc, p, codes)
    rbh = {bh: list(range(p.N)) for bh in heads} if rows is None else rows
    ref = orc.exact_rows(qb_bits, kb_bits, vb_bits, synth.BF16, p.layout, p.causal, rbh)
    qb, kb, vb = bf16_to_f64(qb_bits), bf16_to_f64(kb_bits), bf16_to_f64(vb_bits)
    for (b, h), rr in rbh.items():
        vmax = float(np.abs(head_rows(vb, p.layout, b, h)).max())
        got = bf16_to_f64(head_rows(out_bits, p.layout, b, h))[rr]
        assert_close(got, ref[(b, h)], vmax, "head (%d,%d)" % (b, h))
        # LSE: the float64 log-sum-exp of the scores of the same inputs
        s = head_rows(qb, p.layout, b, h)[rr] @ head_rows(kb, p.layout, b, h).T / np.sqrt(p.D)
        if p.causal:
            s = np.where(np.arange(s.shape[1])[None, :] <= np.asarray(rr)[:, None], s, -np.inf)
        mx = s.max(axis=1, keepdims=True)
        want = mx[:, 0] + np.log(np.exp(s - mx).sum(axis=1))
        assert np.abs(lse_np[b, h][rr] - want).max() < 1e-3


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("causal", [False, True])
def test_attention_bf16_small_shapes(orc, D, layout, causal):
    p = synth.PrefillProblem("abf", 2, 3, 300, D, synth.BF16, synth.INT8, layout, causal=causal, rotate=True,
                             seed=500 + D + layout * 3 + causal, outlier_frac=0.01)
    _run(orc, p, synth.make_prefill(p))


@pytest.mark.parametrize("N", [1, 64, 129, 640])
def test_attention_bf16_lengths(orc, N):
    p = synth.PrefillProblem("abfl", 1, 2, N, 128, synth.BF16, synth.FP8_E4M3, synth.BNSD, causal=True,
                             rotate=True, seed=600 + N)
    _run(orc, p, synth.make_prefill(p))


def test_attention_bf16_int8_causal_problem_sampled(orc):
    """The INT8 causal problem at full size: sampled rows of two heads."""
    p = synth.INT8_CAUSAL
    sample = list(range(0, 64)) + list(range(2000, 2032)) + list(range(4064, 4096))
    _run(orc, p, synth.make_prefill(p), rows={(0, 3): sample, (0, 30): sample})
