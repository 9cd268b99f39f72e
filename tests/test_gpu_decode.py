"""GPU parity of the split-KV decode kernel (INT8 and packed-INT4 caches)
against the oracle: outputs within max-abs <= 1e-2 max|V| and mean-abs <=
1e-3 max|V| (V dequantized, per KV head)."""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import assert_close, bf16_to_f64, dev

pytestmark = pytest.mark.gpu


def _vmax(d, p, b, hk):
    if p.kv_dtype == synth.INT8:
        blk = np.arange(p.L) // p.kv_block
        v = np.abs(d["v"][b, hk].astype(np.float64)).max(axis=1) * d["v_scales"][b, hk, blk]
        return float(v.max())
    byte = d["v"][b, hk]
    lo = ((byte & 0xF).astype(np.int16) ^ 8) - 8
    hi = (((byte >> 4) & 0xF).astype(np.int16) ^ 8) - 8
    m = np.maximum(np.abs(lo), np.abs(hi)).max(axis=1).astype(np.float64)
    sc = d["v_scales"][b, hk].view(np.float16).astype(np.float64).max(axis=1)
    return float((m * sc).max())


def _run(orc, p, d, heads, softmax_scale=0.0):
    q = dev(d["q"]).view(torch.bfloat16)
    k, v = dev(d["k"]), dev(d["v"])
    if p.kv_dtype == synth.INT8:
        ks, vs = dev(d["k_scales"]), dev(d["v_scales"])
        kv = qa.QATTN_INT8
    else:
        ks, vs = dev(d["k_scales"]).view(torch.float16), dev(d["v_scales"]).view(torch.float16)
        kv = qa.QATTN_INT4_PACKED
    out = qa.qattn_decode_kvq(q, k, v, ks, vs, kv, kv_block=p.kv_block, group=p.group, softmax_scale=softmax_scale)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    ref_bits, ref = orc.decode(d["q"], d["k"], d["v"], d["k_scales"], d["v_scales"], p.kv_dtype, p.Hkv,
                               heads=heads, kv_block=p.kv_block, group=p.group, softmax_scale=softmax_scale,
                               want_f64=True)
    g = p.Hq // p.Hkv
    for (b, h) in heads:
        # both sides round their output to bfloat16; compare those outputs
        assert_close(bf16_to_f64(got[b, h, 0]), bf16_to_f64(ref_bits[b, h, 0]), _vmax(d, p, b, h // g),
                     "(%d,%d)" % (b, h))


@pytest.mark.parametrize("kv_dtype", [synth.INT8, synth.INT4_PACKED])
@pytest.mark.parametrize("L", [1, 63, 64, 200, 1000, 4097])
def test_lengths(orc, kv_dtype, L):
    base = synth.INT8_KV_DECODE if kv_dtype == synth.INT8 else synth.INT4_KV_DECODE
    p = synth.scaled(base, B=2, L=L, seed=40 + L)
    d = synth.make_decode(p)
    _run(orc, p, d, [(b, h) for b in range(2) for h in range(p.Hq)])


@pytest.mark.parametrize("kv_dtype", [synth.INT8, synth.INT4_PACKED])
def test_explicit_softmax_scale(orc, kv_dtype):
    """A softmax scale other than 1/sqrt(D), given to both sides."""
    base = synth.INT8_KV_DECODE if kv_dtype == synth.INT8 else synth.INT4_KV_DECODE
    p = synth.scaled(base, B=2, Hq=8, Hkv=2, L=900, seed=61)
    d = synth.make_decode(p)
    _run(orc, p, d, [(b, h) for b in range(2) for h in range(p.Hq)], softmax_scale=0.21)


@pytest.mark.parametrize("kv_dtype", [synth.INT8, synth.INT4_PACKED])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (32, 8), (16, 2)])
def test_gqa_ratios(orc, kv_dtype, Hq, Hkv):
    base = synth.INT8_KV_DECODE if kv_dtype == synth.INT8 else synth.INT4_KV_DECODE
    p = synth.scaled(base, B=3, Hq=Hq, Hkv=Hkv, L=777, seed=50 + Hq + Hkv)
    d = synth.make_decode(p)
    _run(orc, p, d, [(b, h) for b in range(3) for h in range(Hq)])


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (8, 8), (8, 4), (16, 2)])
def test_int4_two_groups_per_row(orc, Hq, Hkv):
    """Scale groups of 64 channels (two per row) at every query-head ratio."""
    p = synth.scaled(synth.INT4_KV_DECODE, B=2, Hq=Hq, Hkv=Hkv, L=500, group=64, seed=61 + Hq + Hkv)
    d = synth.make_decode(p)
    _run(orc, p, d, [(b, h) for b in range(2) for h in range(p.Hq)])


def test_empty_cache_gives_zeros(orc):
    p = synth.scaled(synth.INT8_KV_DECODE, B=2, L=0)
    q = torch.randn(2, p.Hq, 1, 128, device="cuda").to(torch.bfloat16)
    k = torch.empty((2, p.Hkv, 0, 128), dtype=torch.int8, device="cuda")
    s = torch.empty((2, p.Hkv, 0), dtype=torch.float32, device="cuda")
    out = qa.qattn_decode_kvq(q, k, k, s, s, qa.QATTN_INT8)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.float()) == 0


@pytest.mark.parametrize("prob", ["int8kv_decode_b64hq32hkv8l8192d128", "int4kv_decode_b16hq32hkv8l32768d128"])
def test_full_size(orc, prob):
    p = synth.PROBLEMS[prob]
    d = synth.make_decode(p)
    rng = np.random.default_rng(12)
    heads = [(0, 0), (p.B - 1, p.Hq - 1)] + [(int(b), int(h)) for b, h in
                                             zip(rng.integers(0, p.B, 10), rng.integers(0, p.Hq, 10))]
    _run(orc, p, d, heads)
