"""Pins for the oracle's INT4 block quantizer and its attention with Q/K and V
in different code types.

INT4 codes for attention inputs, widened to INT8 for the matmul:
"FlashAttention 的 INT8/INT4 量化" page, 第二层 (INT4); Q/K INT8 with V in a
narrower format: same page, 第三层 (混合精度). Packing (two codes per byte,
element 2i in the low nibble): "ops-transformer INT8/INT4 量化推理" page, 5.2.

The pins do not restate the oracle's loops: the INT4 codes are checked
against torch float32 division and rounding, an exact rotation (a
permutation matrix) and the INT4 error bound; the mixed attention against
the same oracle run in another code type that must give identical results
(INT4 codes are valid INT8 codes; small integers are exact e4m3 values), and
against a constant-V invariant.

CPU only.
"""
import numpy as np
import pytest
import torch

import synth


def _bf16(rng, shape, scale=1.0):
    return synth.f32_to_bf16_bits(rng.standard_normal(shape) * scale)


def _unpack(packed):
    lo = ((packed & 0xF).astype(np.int16) ^ 8) - 8
    hi = ((packed >> 4).astype(np.int16) ^ 8) - 8
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (packed.shape[-1] * 2,))


@pytest.mark.parametrize("layout,block", [(synth.BNSD, 256), (synth.BSND, 128)])
def test_int4_codes_match_torch_division(orc, layout, block):
    rng = np.random.default_rng(block)
    shape = (2, 3, 300, 64) if layout == synth.BNSD else (2, 300, 3, 64)
    x = _bf16(rng, shape)
    x.reshape(-1)[17] = synth.f32_to_bf16_bits(np.array([9.0]))[0]        # an outlier
    codes, scales = orc.rotate_block_quant(x, synth.BF16, layout, None, block, synth.INT4_PACKED)
    assert codes.shape == shape[:-1] + (32,)
    xf = torch.from_numpy(synth.bf16_bits_to_f32(x))
    if layout == synth.BSND:
        xf = xf.permute(0, 2, 1, 3)
        c = _unpack(codes).transpose(0, 2, 1, 3)
    else:
        c = _unpack(codes)
    N = xf.shape[2]
    nblk = -(-N // block)
    for k in range(nblk):
        xb = xf[:, :, k * block:(k + 1) * block]
        amax = xb.abs().amax(dim=(2, 3))
        s = (amax / 7.0).to(torch.float32)
        assert np.array_equal(scales[:, :, k].view(np.uint32), s.numpy().view(np.uint32))
        want = torch.where(s[:, :, None, None] > 0, torch.round(xb / s[:, :, None, None]).clamp(-7, 7),
                           torch.zeros(()))
        assert np.array_equal(c[:, :, k * block:(k + 1) * block], want.numpy().astype(np.int16))
        # the block maximum maps to +-7; every value is within s / 2
        cb = c[:, :, k * block:(k + 1) * block].astype(np.float64)
        sf = s.numpy().astype(np.float64)[:, :, None, None]
        assert np.all(np.abs(cb * sf - xb.numpy()) <= sf / 2 + 1e-7)
        assert np.all(np.abs(cb).max(axis=(2, 3)) == 7)


def test_int4_rotation_by_permutation_is_exact(orc):
    """A permutation matrix rotates exactly (every FMA chain adds zeros and one
    product by 1), so the codes are the unrotated codes with permuted columns."""
    rng = np.random.default_rng(3)
    x = _bf16(rng, (1, 2, 256, 64))
    perm = rng.permutation(64)
    R = np.zeros((64, 64), np.float32)
    R[perm, np.arange(64)] = 1.0                      # y[:, j] = x[:, perm[j]]
    c_rot, s_rot = orc.rotate_block_quant(x, synth.BF16, synth.BNSD, R, 256, synth.INT4_PACKED)
    c_ref, s_ref = orc.rotate_block_quant(x, synth.BF16, synth.BNSD, None, 256, synth.INT4_PACKED)
    assert np.array_equal(s_rot.view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(_unpack(c_rot), _unpack(c_ref)[..., perm])


def _qk_int8(orc, rng, B, H, N, D):
    x = {n: _bf16(rng, (B, H, N, D)) for n in ("q", "k", "v")}
    qc, qs = orc.rotate_block_quant(x["q"], synth.BF16, synth.BNSD, None, 128, synth.INT8)
    kc, ks = orc.rotate_block_quant(x["k"], synth.BF16, synth.BNSD, None, 256, synth.INT8)
    return x, qc, qs, kc, ks


@pytest.mark.parametrize("causal", [False, True])
def test_int4_v_equals_the_same_codes_held_as_int8(orc, causal):
    """INT4 codes in [-7, 7] are INT8 codes: V packed as INT4 and the same codes
    one per byte (INT8) with the same scales give identical outputs."""
    B, H, N, D = 1, 2, 384, 64
    rng = np.random.default_rng(5 + causal)
    x, qc, qs, kc, ks = _qk_int8(orc, rng, B, H, N, D)
    v4, vs = orc.rotate_block_quant(x["v"], synth.BF16, synth.BNSD, None, 256, synth.INT4_PACKED)
    v8 = _unpack(v4).astype(np.int8).view(np.uint8)
    rows = {(b, h): list(range(0, N, 7)) + [N - 1] for b in range(B) for h in range(H)}
    a = orc.prefill_rows(qc, qs, kc, ks, v4, vs, synth.INT8, synth.BNSD, causal, rows, want_f64=True,
                         v_dtype=synth.INT4_PACKED)
    b = orc.prefill_rows(qc, qs, kc, ks, v8, vs, synth.INT8, synth.BNSD, causal, rows, want_f64=True,
                         v_dtype=synth.INT8)
    for key in rows:
        assert np.array_equal(a[key][0], b[key][0])
        assert np.array_equal(a[key][1], b[key][1])


def test_int8_qk_with_e4m3_v_equals_e4m3_qk_for_small_codes(orc):
    """Integers up to 15 are exact e4m3 values: INT8 Q/K codes in [-15, 15]
    with e4m3 V give the same output as the all-e4m3 path whose Q/K codes
    encode the same integers."""
    B, H, N, D = 1, 2, 256, 64
    rng = np.random.default_rng(9)
    q8 = rng.integers(-15, 16, (B, H, N, D)).astype(np.int8)
    k8 = rng.integers(-15, 16, (B, H, N, D)).astype(np.int8)
    qs = rng.uniform(0.01, 0.03, (B, H, N // 128)).astype(np.float32)
    ks = rng.uniform(0.01, 0.03, (B, H, N // 256)).astype(np.float32)
    v = _bf16(rng, (B, H, N, D))
    vc, vs = orc.rotate_block_quant(v, synth.BF16, synth.BNSD, None, 256, synth.FP8_E4M3)
    q_e4 = orc.e4m3_encode(q8.astype(np.float32))
    k_e4 = orc.e4m3_encode(k8.astype(np.float32))
    assert np.array_equal(orc.e4m3_decode(q_e4), q8.astype(np.float32))
    rows = {(b, h): list(range(0, N, 5)) for b in range(B) for h in range(H)}
    a = orc.prefill_rows(q8.view(np.uint8), qs, k8.view(np.uint8), ks, vc, vs, synth.INT8, synth.BNSD, True,
                         rows, want_f64=True, v_dtype=synth.FP8_E4M3)
    b = orc.prefill_rows(q_e4, qs, k_e4, ks, vc, vs, synth.FP8_E4M3, synth.BNSD, True, rows, want_f64=True)
    for key in rows:
        assert np.array_equal(a[key][1], b[key][1])


@pytest.mark.parametrize("v_dtype", [synth.INT4_PACKED, synth.FP8_E4M3])
def test_constant_v_reproduces_the_row(orc, v_dtype):
    """All V rows equal: the weights are normalised by their own sum, so every
    output row is that V row (dequantized)."""
    B, H, N, D = 1, 1, 256, 64
    rng = np.random.default_rng(11)
    x, qc, qs, kc, ks = _qk_int8(orc, rng, B, H, N, D)
    row = synth.f32_to_bf16_bits(np.linspace(-1.0, 1.0, D))
    v = np.broadcast_to(row, (B, H, N, D)).copy()
    vc, vs = orc.rotate_block_quant(v, synth.BF16, synth.BNSD, None, 256, v_dtype)
    if v_dtype == synth.INT4_PACKED:
        deq = _unpack(vc)[0, 0, 0].astype(np.float64) * float(vs[0, 0, 0])
    else:
        deq = orc.e4m3_decode(vc[0, 0, 0]).astype(np.float64) * float(vs[0, 0, 0])
    rows = {(0, 0): list(range(0, N, 3))}
    out = orc.prefill_rows(qc, qs, kc, ks, vc, vs, synth.INT8, synth.BNSD, True, rows, want_f64=True,
                           v_dtype=v_dtype)[(0, 0)][1]
    assert np.allclose(out, deq[None, :], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_int4_qkv_equals_the_same_codes_held_as_int8(orc, causal):
    """INT4 Q, K and V (rotated Q/K): identical outputs to the INT8 path fed
    the same codes one per byte with the same scales -- INT4 codes widened to
    INT8 for the matmul, as the page's INT4 layer states."""
    B, H, N, D = 1, 2, 300, 64
    rng = np.random.default_rng(21 + causal)
    R = synth.haar_orthogonal(5, 0, D)
    x = {n: _bf16(rng, (B, H, N, D)) for n in ("q", "k", "v")}
    q4, qs = orc.rotate_block_quant(x["q"], synth.BF16, synth.BNSD, R, 128, synth.INT4_PACKED)
    k4, ks = orc.rotate_block_quant(x["k"], synth.BF16, synth.BNSD, R, 256, synth.INT4_PACKED)
    v4, vs = orc.rotate_block_quant(x["v"], synth.BF16, synth.BNSD, None, 256, synth.INT4_PACKED)
    as8 = lambda c: _unpack(c).astype(np.int8).view(np.uint8)
    rows = {(b, h): list(range(0, N, 4)) + [N - 1] for b in range(B) for h in range(H)}
    a = orc.prefill_rows(q4, qs, k4, ks, v4, vs, synth.INT4_PACKED, synth.BNSD, causal, rows, want_f64=True)
    b = orc.prefill_rows(as8(q4), qs, as8(k4), ks, as8(v4), vs, synth.INT8, synth.BNSD, causal, rows,
                         want_f64=True)
    for key in rows:
        assert np.array_equal(a[key][1], b[key][1])
