"""GPU parity of the mixed-precision prefill (Q/K INT8 with V e4m3 or packed
INT4) and of the INT4 block quantizer, against the oracle.

INT4 block codes, widened to INT8 for the matmul: "FlashAttention 的
INT8/INT4 量化" page, 第二层; Q/K INT8 with V in a narrower format: same page,
第三层 (混合精度). Codes and scales must agree bit for bit; outputs within
max-abs <= 1e-2 max|V| and mean-abs <= 1e-3 max|V| (V dequantized, per head).
"""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import assert_close, bf16_to_f64, dequant_v_max, dev, dev_bits, head_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("D,block", [(64, 256), (128, 128), (128, 256)])
@pytest.mark.parametrize("in_dtype", [synth.BF16, synth.F16])
def test_int4_block_quant_bit_exact(orc, layout, D, block, in_dtype):
    N = 300                                                    # ragged last block
    rng = np.random.default_rng(D + block + layout + 7 * in_dtype)
    shape = (2, 3, N, D) if layout == synth.BNSD else (2, N, 3, D)
    x = rng.standard_normal(shape) * np.exp(rng.uniform(-2, 2, shape[:-1] + (1,)))
    bits = synth.f32_to_bf16_bits(x) if in_dtype == synth.BF16 else synth.f64_to_f16_bits(x)
    codes, scales = qa.qattn_rotate_block_quant(dev_bits(bits, in_dtype), layout, None, block, qa.QATTN_INT4_PACKED)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    oc, osc = orc.rotate_block_quant(bits, in_dtype, layout, None, block, synth.INT4_PACKED)
    assert codes.shape == oc.shape
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), osc.view(np.uint32))


def test_int4_block_quant_ties(orc):
    """Blocks whose quotients land exactly on half-integers (max 7 -> scale 1,
    values k + 1/2) and on their bf16 neighbours: the IEEE quotient decides."""
    B, H, N, D = 1, 4, 256, 128
    rng = np.random.default_rng(1)
    half = rng.integers(-7, 7, (B, H, N, D)) + 0.5
    x = np.where(rng.random((B, H, N, D)) < 0.5, half, rng.uniform(-7, 7, (B, H, N, D)))
    x[..., 0, 0] = 7.0                                         # the block max: scale exactly 1
    bits = synth.f32_to_bf16_bits(x)
    nb = bits.copy()
    nb[:, 1::2] = bits[:, 1::2] + np.where(rng.random(bits[:, 1::2].shape) < 0.5, 1, -1).astype(np.uint16)
    nb[..., 0, 0] = bits[..., 0, 0]
    codes, scales = qa.qattn_rotate_block_quant(dev_bits(nb, synth.BF16), synth.BNSD, None, 256,
                                                qa.QATTN_INT4_PACKED)
    torch.cuda.synchronize()
    oc, osc = orc.rotate_block_quant(nb, synth.BF16, synth.BNSD, None, 256, synth.INT4_PACKED)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), osc.view(np.uint32))


def _mixed(orc, p, d, v_dtype, rows_by_head, check_codes=True):
    rot = dev(d["rot"]) if d["rot"] is not None else None
    q = dev_bits(d["q"], p.in_dtype)
    k = dev_bits(d["k"], p.in_dtype)
    v = dev_bits(d["v"], p.in_dtype)
    qc, qs = qa.qattn_rotate_block_quant(q, p.layout, rot, 128, qa.QATTN_INT8)
    kc, ks = qa.qattn_rotate_block_quant(k, p.layout, rot, 256, qa.QATTN_INT8)
    vc, vs = qa.qattn_rotate_block_quant(v, p.layout, None, 256, v_dtype)
    lse = torch.empty((p.B, p.H, p.N), dtype=torch.float32, device="cuda")
    out = qa.qattn_prefill_mixed(qc, qs, kc, ks, vc, vs, qa.QATTN_INT8, v_dtype, p.layout, p.causal, lse=lse)
    runs = [(out, lse, "on chip")]
    if v_dtype == synth.INT4_PACKED:
        # V widened to INT8 codes first, then the INT8 prefill
        lse_w = torch.empty_like(lse)
        out_w = qa.qattn_prefill(qc, qs, kc, ks, qa.qattn_widen_int4(vc), vs, qa.QATTN_INT8, p.layout, p.causal,
                                 lse=lse_w)
        runs.append((out_w, lse_w, "widened first"))
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    heads = sorted(rows_by_head)
    oq = orc.rotate_block_quant(d["q"], p.in_dtype, p.layout, d["rot"], 128, synth.INT8, heads=heads)
    ok_ = orc.rotate_block_quant(d["k"], p.in_dtype, p.layout, d["rot"], 256, synth.INT8, heads=heads)
    ov = orc.rotate_block_quant(d["v"], p.in_dtype, p.layout, None, 256, v_dtype, heads=heads)
    if check_codes:
        for (g, o) in (((qc, qs), oq), ((kc, ks), ok_), ((vc, vs), ov)):
            gcodes, gsc = g[0].cpu().numpy(), g[1].cpu().numpy()
            for (b, h) in heads:
                assert np.array_equal(head_rows(gcodes, p.layout, b, h), head_rows(o[0], p.layout, b, h))
                assert np.array_equal(gsc[b, h], o[1][b, h])
    ref = orc.prefill_rows(*oq, *ok_, *ov, synth.INT8, p.layout, p.causal, rows_by_head, want_lse=True,
                           v_dtype=v_dtype)
    _check_runs(orc, p, runs, ref, ov, v_dtype, rows_by_head)


def _check_runs(orc, p, runs, ref, ov, v_dtype, rows_by_head):
    for (out, lse, how) in runs:
        out_bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
        lse_np = lse.cpu().numpy()
        for (b, h), rows in rows_by_head.items():
            got = bf16_to_f64(head_rows(out_bits, p.layout, b, h)[rows])
            vmax = dequant_v_max(ov[0], ov[1], v_dtype, p.layout, b, h, orc)
            assert_close(got, bf16_to_f64(ref[(b, h)][0]), vmax, "head (%d,%d), %s" % (b, h, how))
            assert np.abs(lse_np[b, h, rows] - ref[(b, h)][2]).max() < 1e-2, how


@pytest.mark.parametrize("v_dtype", [synth.INT4_PACKED, synth.FP8_E4M3])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("causal", [False, True])
def test_mixed_small_shapes(orc, v_dtype, D, layout, causal):
    """Several query and key tiles, ragged tails (N = 300), both layouts."""
    p = synth.PrefillProblem("mixed", 2, 3, 300, D, synth.BF16, synth.INT8, layout, causal=causal, rotate=True,
                             seed=400 + D + 3 * layout + 5 * causal + v_dtype)
    d = synth.make_prefill(p)
    _mixed(orc, p, d, v_dtype, {(b, h): list(range(p.N)) for b in range(p.B) for h in range(p.H)})


@pytest.mark.parametrize("N", [1, 129, 640])
def test_mixed_int4_sequence_lengths(orc, N):
    p = synth.PrefillProblem("len", 1, 2, N, 128, synth.BF16, synth.INT8, synth.BNSD, causal=True, rotate=True,
                             seed=500 + N, outlier_frac=0.01)
    d = synth.make_prefill(p)
    _mixed(orc, p, d, synth.INT4_PACKED, {(0, h): list(range(N)) for h in range(2)})


def test_mixed_int4_full_size(orc):
    """The INT8 causal problem (B1 H32 N4096 D128) with V in packed INT4, in
    the benchmark's launch configuration; sampled rows of sampled heads."""
    p = synth.INT8_CAUSAL
    d = synth.make_prefill(p)
    rng = np.random.default_rng(0)
    heads = [(0, int(h)) for h in rng.choice(p.H, 3, replace=False)]
    rows = sorted(set(rng.choice(p.N, 96, replace=False).tolist()) | {0, 127, 128, p.N - 1})
    _mixed(orc, p, d, synth.INT4_PACKED, {hd: rows for hd in heads})


@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("D,block", [(64, 128), (128, 128), (128, 256)])
def test_int4_rotated_block_quant_bit_exact(orc, layout, D, block):
    """Rotation + INT4 codes (the rotated values decide the codes as for
    INT8)."""
    N = 300
    rng = np.random.default_rng(D + block + 11 * layout)
    shape = (1, 3, N, D) if layout == synth.BNSD else (1, N, 3, D)
    bits = synth.f32_to_bf16_bits(rng.standard_normal(shape))
    R = synth.haar_orthogonal(3, 1, D)
    codes, scales = qa.qattn_rotate_block_quant(dev_bits(bits, synth.BF16), layout, dev(R), block,
                                                qa.QATTN_INT4_PACKED)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    oc, osc = orc.rotate_block_quant(bits, synth.BF16, layout, R, block, synth.INT4_PACKED)
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), osc.view(np.uint32))


def _int4_all(orc, p, d, rows_by_head, check_codes=True):
    rot = dev(d["rot"])
    c = {}
    for nm, blk, r in (("q", 128, rot), ("k", 256, rot), ("v", 256, None)):
        c[nm] = qa.qattn_rotate_block_quant(dev_bits(d[nm], p.in_dtype), p.layout, r, blk, qa.QATTN_INT4_PACKED)
    lse = torch.empty((p.B, p.H, p.N), dtype=torch.float32, device="cuda")
    out = qa.qattn_prefill_mixed(*c["q"], *c["k"], *c["v"], qa.QATTN_INT4_PACKED, qa.QATTN_INT4_PACKED, p.layout,
                                 p.causal, lse=lse)
    # every operand widened to INT8 codes first, then the INT8 prefill
    w = {nm: (qa.qattn_widen_int4(c[nm][0]), c[nm][1]) for nm in "qkv"}
    lse_w = torch.empty_like(lse)
    out_w = qa.qattn_prefill(*w["q"], *w["k"], *w["v"], qa.QATTN_INT8, p.layout, p.causal, lse=lse_w)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    assert out.shape == tuple(p.shape()) and out_w.shape == tuple(p.shape())
    heads = sorted(rows_by_head)
    o = {nm: orc.rotate_block_quant(d[nm], p.in_dtype, p.layout, d["rot"] if nm != "v" else None,
                                    128 if nm == "q" else 256, synth.INT4_PACKED, heads=heads) for nm in "qkv"}
    if check_codes:
        for nm in "qkv":
            gcodes, gsc = c[nm][0].cpu().numpy(), c[nm][1].cpu().numpy()
            for (b, h) in heads:
                assert np.array_equal(head_rows(gcodes, p.layout, b, h), head_rows(o[nm][0], p.layout, b, h))
                assert np.array_equal(gsc[b, h], o[nm][1][b, h])
    ref = orc.prefill_rows(*o["q"], *o["k"], *o["v"], synth.INT4_PACKED, p.layout, p.causal, rows_by_head,
                           want_lse=True)
    _check_runs(orc, p, [(out, lse, "on chip"), (out_w, lse_w, "widened first")], ref, o["v"], synth.INT4_PACKED,
                rows_by_head)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("causal", [False, True])
def test_int4_qkv_small_shapes(orc, D, layout, causal):
    p = synth.PrefillProblem("int4", 2, 3, 300, D, synth.BF16, synth.INT8, layout, causal=causal, rotate=True,
                             seed=600 + D + 3 * layout + 5 * causal)
    d = synth.make_prefill(p)
    _int4_all(orc, p, d, {(b, h): list(range(p.N)) for b in range(p.B) for h in range(p.H)})


@pytest.mark.parametrize("N", [1, 129, 640])
def test_int4_qkv_sequence_lengths(orc, N):
    p = synth.PrefillProblem("len4", 1, 2, N, 128, synth.BF16, synth.INT8, synth.BNSD, causal=True, rotate=True,
                             seed=700 + N, outlier_frac=0.01)
    d = synth.make_prefill(p)
    _int4_all(orc, p, d, {(0, h): list(range(N)) for h in range(2)})


def test_int4_qkv_full_size(orc):
    """The INT8 causal problem (B1 H32 N4096 D128) with Q, K and V in packed
    INT4; sampled rows of sampled heads."""
    p = synth.INT8_CAUSAL
    d = synth.make_prefill(p)
    rng = np.random.default_rng(1)
    heads = [(0, int(h)) for h in rng.choice(p.H, 3, replace=False)]
    rows = sorted(set(rng.choice(p.N, 96, replace=False).tolist()) | {0, 127, 128, p.N - 1})
    _int4_all(orc, p, d, {hd: rows for hd in heads})
