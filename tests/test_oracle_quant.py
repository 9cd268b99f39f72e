"""Pins for the oracle's rotation and dynamic block quantization.

Rotation: "MindIE-SD quantization" page, FA量化 / 技术特点 / 旋转.
Block quantization: same page, 块量化 (Q blocks of 128 tokens, K/V blocks of
256, float8_e4m3fn); symmetric INT8 with scale = max|x| / 127 and value =
round(x / scale): "INT8 量化算子" page, 对称量化.

CPU only.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth


def _round_f32(fr: Fraction) -> Fraction:
    """Exact round-to-nearest-even of a rational to float32."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = Fraction(2) ** max(e - 23, -149)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * q


def _fma_chain_exact(x, R, j):
    acc = Fraction(0)
    for k in range(len(x)):
        acc = _round_f32(Fraction(float(x[k])) * Fraction(float(R[k, j])) + acc)
    return float(acc)


def _bf16_values(rng, n):
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(rng.standard_normal(n) * 3))


@pytest.mark.parametrize("D", [16, 64])
def test_rotation_is_the_sequential_float32_fma_chain(orc, D):
    """Bit-exact against exact rational arithmetic rounded once per step."""
    rng = np.random.default_rng(D)
    R = synth.haar_orthogonal(7, 4, D)
    for _ in range(2):
        x = _bf16_values(rng, D)
        y = orc.rotate_row(x, R)
        ref = np.array([_fma_chain_exact(x, R, j) for j in range(D)], dtype=np.float32)
        assert np.array_equal(y.view(np.uint32), ref.view(np.uint32))


def test_rotation_identity_and_signed_permutation_are_exact(orc):
    D = 128
    rng = np.random.default_rng(3)
    x = _bf16_values(rng, D)
    assert np.array_equal(orc.rotate_row(x, np.eye(D, dtype=np.float32)), x)
    perm = rng.permutation(D)
    signs = rng.choice([-1.0, 1.0], D).astype(np.float32)
    P = np.zeros((D, D), dtype=np.float32)
    P[np.arange(D), perm] = signs        # x P moves x[k] to column perm[k]
    y = orc.rotate_row(x, P)
    ref = np.zeros(D, dtype=np.float32)
    ref[perm] = x * signs
    assert np.array_equal(y, ref)


def test_rotation_matches_float64_product_within_dot_bound(orc):
    D = 128
    rng = np.random.default_rng(4)
    R = synth.haar_orthogonal(9, 4, D)
    for _ in range(8):
        x = _bf16_values(rng, D)
        y = orc.rotate_row(x, R).astype(np.float64)
        exact = x.astype(np.float64) @ R.astype(np.float64)
        bound = D * 2.0 ** -24 * (np.abs(x).astype(np.float64) @ np.abs(R).astype(np.float64))
        assert np.all(np.abs(y - exact) <= bound)


def test_rotation_matrix_is_orthogonal_and_preserves_qk():
    D = 128
    R = synth.haar_orthogonal(2, 4, D).astype(np.float64)
    assert np.abs(R.T @ R - np.eye(D)).max() <= 1e-6
    rng = np.random.default_rng(5)
    Q = rng.standard_normal((64, D))
    K = rng.standard_normal((64, D))
    a = (Q @ R) @ (K @ R).T
    b = Q @ K.T
    assert np.abs(a - b).max() <= 1e-5 * np.abs(b).max()


def _torch_block_quant(y: np.ndarray, code_dtype: int):
    """Library reference: torch float32 absmax, division, round-half-even."""
    t = torch.from_numpy(np.ascontiguousarray(y, dtype=np.float32))
    qmax = 127.0 if code_dtype == synth.INT8 else 448.0
    s = t.abs().max() / qmax
    if float(s) == 0.0:
        return np.zeros(y.shape, np.uint8), np.float32(0)
    v = t / s
    if code_dtype == synth.INT8:
        c = torch.round(v).clamp(-127, 127).to(torch.int8).view(torch.uint8)
    else:
        c = v.to(torch.float8_e4m3fn).view(torch.uint8)
    return c.numpy(), np.float32(s.item())


def _rows(x_bits, layout, b, h, n0, n1):
    if layout == synth.BNSD:
        return x_bits[b, h, n0:n1]
    return x_bits[b, n0:n1, h]


@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("rotate", [False, True])
def test_block_quant_matches_torch_per_block(orc, code_dtype, layout, rotate):
    """Codes and scales of every block (including a ragged tail block) equal
    the torch reference applied to that block's rotated rows."""
    B, H, N, D, T = 2, 3, 300, 64, 128
    rng = np.random.default_rng(11)
    x = synth.f32_to_bf16_bits(rng.standard_normal((B, H, N, D) if layout == synth.BNSD
                                                   else (B, N, H, D)) * 2)
    R = synth.haar_orthogonal(5, 4, D) if rotate else None
    codes, scales = orc.rotate_block_quant(x, synth.BF16, layout, R, T, code_dtype)
    assert scales.shape == (B, H, 3)
    for b in range(B):
        for h in range(H):
            for blk in range(3):
                n0, n1 = blk * T, min(N, (blk + 1) * T)
                xr = synth.bf16_bits_to_f32(_rows(x, layout, b, h, n0, n1))
                y = np.stack([orc.rotate_row(r, R) for r in xr])
                c_ref, s_ref = _torch_block_quant(y, code_dtype)
                assert scales[b, h, blk].view(np.uint32) == s_ref.view(np.uint32)
                assert np.array_equal(_rows(codes, layout, b, h, n0, n1), c_ref)


@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3])
def test_quant_error_bounds_and_extremes(orc, code_dtype):
    B, H, N, D, T = 1, 2, 512, 128, 256
    rng = np.random.default_rng(12)
    x = synth.f32_to_bf16_bits(rng.standard_normal((B, H, N, D)) * np.exp(rng.standard_normal((B, H, N, 1))))
    R = synth.haar_orthogonal(6, 4, D)
    codes, scales = orc.rotate_block_quant(x, synth.BF16, synth.BNSD, R, T, code_dtype)
    for h in range(H):
        for blk in range(2):
            s = np.float64(scales[0, h, blk])
            y = np.stack([orc.rotate_row(r, R) for r in synth.bf16_bits_to_f32(x[0, h, blk * T:(blk + 1) * T])])
            c = codes[0, h, blk * T:(blk + 1) * T]
            if code_dtype == synth.INT8:
                deq = c.view(np.int8).astype(np.float64) * s
                assert np.all(np.abs(y - deq) <= s / 2 * (1 + 2.0 ** -20))
                peak = np.abs(c.view(np.int8).astype(np.int32)).max()
                assert peak == 127
            else:
                deq = orc.e4m3_decode(c).astype(np.float64)
                v = y.astype(np.float64) / s
                normal = np.abs(v) >= 2.0 ** -6
                assert np.all(np.abs(v - deq)[normal] <= 2.0 ** -4 * np.abs(v[normal]) * (1 + 1e-6))
                assert np.all(np.abs(v - deq)[~normal] <= 2.0 ** -10 * (1 + 1e-6))
                assert (c & 0x7F).max() == 0x7E          # the block max maps to +-448
            assert s == np.float32(np.abs(y).max()) / np.float32(127.0 if code_dtype == synth.INT8 else 448.0)


def test_zero_block_gives_zero_scale_and_codes(orc):
    x = np.zeros((1, 1, 256, 64), dtype=np.uint16)
    x[0, 0, 200:, :] = synth.f32_to_bf16_bits(np.ones((56, 64)))
    codes, scales = orc.rotate_block_quant(x, synth.BF16, synth.BNSD, None, 128, synth.INT8)
    assert scales[0, 0, 0] == 0.0 and not codes[0, 0, :128].any()
    assert scales[0, 0, 1] == np.float32(1.0) / np.float32(127.0)
    assert np.all(codes[0, 0, 200:].view(np.int8) == 127)


def test_layouts_agree(orc):
    B, H, N, D = 2, 3, 384, 64
    rng = np.random.default_rng(13)
    xb = synth.f32_to_bf16_bits(rng.standard_normal((B, H, N, D)))
    xs = np.ascontiguousarray(xb.transpose(0, 2, 1, 3))
    R = synth.haar_orthogonal(8, 4, D)
    c1, s1 = orc.rotate_block_quant(xb, synth.BF16, synth.BNSD, R, 256, synth.FP8_E4M3)
    c2, s2 = orc.rotate_block_quant(xs, synth.BF16, synth.BSND, R, 256, synth.FP8_E4M3)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1, c2.transpose(0, 2, 1, 3))


def test_f16_input_path(orc):
    rng = np.random.default_rng(14)
    x = synth.f64_to_f16_bits(rng.standard_normal((1, 2, 256, 64)))
    codes, scales = orc.rotate_block_quant(x, synth.F16, synth.BNSD, None, 128, synth.FP8_E4M3)
    xf = x.view(np.float16).astype(np.float32)
    for h in range(2):
        for blk in range(2):
            c_ref, s_ref = _torch_block_quant(xf[0, h, blk * 128:(blk + 1) * 128], synth.FP8_E4M3)
            assert scales[0, h, blk] == s_ref
            assert np.array_equal(codes[0, h, blk * 128:(blk + 1) * 128], c_ref)
