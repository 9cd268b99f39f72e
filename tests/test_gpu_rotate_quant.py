"""GPU parity of the rotation + block quantization kernels: codes and scales
must equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import dev, dev_bits

pytestmark = pytest.mark.gpu


def _check_all(orc, x_bits, in_dtype, layout, rot, block, code_dtype, blocks=None):
    x = dev_bits(x_bits, in_dtype)
    r = dev(rot) if rot is not None else None
    codes, scales = qa.qattn_rotate_block_quant(x, layout, r, block, code_dtype)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    oc, os_ = orc.rotate_block_quant(x_bits, in_dtype, layout, rot, block, code_dtype, blocks=blocks)
    if blocks is None:
        assert np.array_equal(gs.view(np.uint32), os_.view(np.uint32))
        bad = np.nonzero(gc != oc)
        assert bad[0].size == 0, "codes differ at %d places, first %s" % (bad[0].size, [b[:3] for b in bad])
    else:
        N = x_bits.shape[2] if layout == synth.BNSD else x_bits.shape[1]
        for (b, h, k) in blocks:
            assert gs[b, h, k].view(np.uint32) == os_[b, h, k].view(np.uint32)
            n0, n1 = k * block, min(N, (k + 1) * block)
            if layout == synth.BNSD:
                assert np.array_equal(gc[b, h, n0:n1], oc[b, h, n0:n1])
            else:
                assert np.array_equal(gc[b, n0:n1, h], oc[b, n0:n1, h])


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3, synth.INT4_PACKED])
@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("block", [128, 256])
def test_small_shapes_bit_exact(orc, D, layout, code_dtype, rotate, block):
    B, H, N = 2, 3, 300                     # ragged tail block
    rng = np.random.default_rng(D + 7 * layout + 13 * code_dtype + rotate + block)
    shape = (B, H, N, D) if layout == synth.BNSD else (B, N, H, D)
    x = synth.f32_to_bf16_bits(rng.standard_normal(shape) * np.exp(rng.standard_normal(shape[:-1] + (1,))))
    rot = synth.haar_orthogonal(17, 4, D) if rotate else None
    _check_all(orc, x, synth.BF16, layout, rot, block, code_dtype)


def test_rounding_ties_and_near_ties(orc):
    """Blocks whose scale is exactly 1 (block max 127 for INT8, 448 for e4m3)
    hold values on and next to the rounding boundaries of the codes (exact
    half-integers, exact e4m3 midpoints, and their bf16 neighbours), so the
    code decisions are exercised where a misrounded quotient would show; a
    block with a subnormal scale and a signed permutation as rotation (which
    moves values exactly) are included."""
    D, T = 128, 128
    for code, top in ((synth.INT8, 127.0), (synth.FP8_E4M3, 448.0)):
        if code == synth.INT8:
            base = np.arange(-126, 127) + 0.5
        else:
            import torch as _t
            grid = np.unique(_t.arange(0, 127, dtype=_t.uint8).view(_t.float8_e4m3fn).float().numpy())
            base = (grid[:-1].astype(np.float64) + grid[1:]) / 2
            base = np.concatenate([base, -base])
        bits = synth.f32_to_bf16_bits(base)
        nb = np.concatenate([bits, bits + 1, bits - 1]).astype(np.uint16)      # ties and bf16 neighbours
        vals = np.resize(nb, T * D).reshape(T, D)
        vals[0, 0] = synth.f32_to_bf16_bits(np.array([top]))[0]
        tiny = synth.f32_to_bf16_bits(np.random.default_rng(1).standard_normal((T, D)) * 1e-39)
        x = np.stack([vals, tiny])[None]                                          # [1, 2, T, D]
        perm = np.random.default_rng(2).permutation(D)
        P = np.zeros((D, D), dtype=np.float32)
        P[np.arange(D), perm] = 1.0
        _check_all(orc, x, synth.BF16, synth.BNSD, None, T, code)
        _check_all(orc, x, synth.BF16, synth.BNSD, P, T, code)


def test_f16_input_and_edge_blocks(orc):
    B, H, N, D = 1, 2, 257, 128               # last block holds one token
    rng = np.random.default_rng(3)
    x = synth.f64_to_f16_bits(rng.standard_normal((B, H, N, D)))
    x[0, 1, :128] = 0                         # an all-zero block: scale 0, codes 0
    rot = synth.haar_orthogonal(3, 4, D)
    for code in (synth.INT8, synth.FP8_E4M3):
        _check_all(orc, x, synth.F16, synth.BNSD, rot, 128, code)
        _check_all(orc, x, synth.F16, synth.BNSD, None, 128, code)


def test_outlier_channels_int8_config_small(orc):
    p = synth.scaled(synth.INT8_CAUSAL, H=4, N=512)
    d = synth.make_prefill(p)
    for name, blk, rot in (("q", 128, d["rot"]), ("k", 256, d["rot"]), ("v", 256, None)):
        _check_all(orc, d[name], p.in_dtype, p.layout, rot, blk, p.code_dtype)


@pytest.mark.parametrize("prob", ["tiny_fp8_b1h2n256d64", "int8_causal_b1h32n4096d128", "fp8_bsnd_b1h24n16384d128"])
def test_full_size_sampled_blocks(orc, prob):
    """Full-size problems in the launch configuration the benchmark uses;
    the oracle recomputes a sample of blocks (all of them for the tiny one)."""
    p = synth.PROBLEMS[prob]
    d = synth.make_prefill(p)
    rng = np.random.default_rng(5)
    for name, blk, rot in (("q", 128, d["rot"]), ("k", 256, d["rot"]), ("v", 256, None)):
        nblk = -(-p.N // blk)
        if p.N <= 256:
            blocks = None
        else:
            blocks = [(0, int(h), int(k)) for h, k in zip(rng.integers(0, p.H, 6), rng.integers(0, nblk, 6))]
            blocks += [(0, p.H - 1, nblk - 1), (0, 0, 0)]
        _check_all(orc, d[name], p.in_dtype, p.layout, rot, blk, p.code_dtype, blocks=blocks)


def test_signed_permutation_rotation_all_shapes(orc):
    """A signed permutation moves every value exactly: at both block sizes,
    both D and every code type."""
    rng = np.random.default_rng(21)
    for D in (64, 128):
        x = synth.f32_to_bf16_bits(rng.standard_normal((1, 2, 300, D)) * 4)
        P = np.zeros((D, D), dtype=np.float32)
        P[np.arange(D), rng.permutation(D)] = rng.choice([-1.0, 1.0], D)
        for T in (128, 256):
            for code in (synth.INT8, synth.FP8_E4M3, synth.INT4_PACKED):
                _check_all(orc, x, synth.BF16, synth.BNSD, P, T, code)


@pytest.mark.parametrize("in_dtype", [synth.BF16, synth.F16])
def test_wide_range_inputs_and_matrix(orc, in_dtype):
    """Inputs spanning many binades (f16 ones with subnormals) and a
    non-orthogonal R whose entries span many binades too, some far below the
    largest: the FMA chain of the rotation is reproduced bit for bit."""
    rng = np.random.default_rng(23 + in_dtype)
    D = 128
    mag = np.exp2(rng.integers(-16, 6, (1, 2, 300, D)))
    vals = rng.standard_normal((1, 2, 300, D)) * mag
    x = synth.f32_to_bf16_bits(vals) if in_dtype == synth.BF16 else synth.f64_to_f16_bits(vals)
    R = (rng.standard_normal((D, D)) * np.exp2(rng.integers(-30, 3, (D, D)))).astype(np.float32)
    for code in (synth.INT8, synth.FP8_E4M3, synth.INT4_PACKED):
        for T in (128, 256):
            _check_all(orc, x, in_dtype, synth.BNSD, R, T, code)
