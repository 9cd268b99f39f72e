"""GPU parity of KV-cache quantize-on-append: codes and scales must equal
the oracle's bit for bit after a sequence of appends (block-aligned, inside
a block, across block boundaries, with and without a growing INT8 block
scale), and at the size of the INT8 decode problem."""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import dev

pytestmark = pytest.mark.gpu


def _x(rng, shape, scale=1.0):
    return synth.f32_to_bf16_bits(rng.standard_normal(shape) * scale)


def _run_sequence(orc, kv_dtype, B, H, D, Lmax, pieces, group=128, seed=0):
    """pieces: list of (n, magnitude). Appends them one after another on the
    GPU and in the oracle; compares after every append."""
    rng = np.random.default_rng(seed)
    if kv_dtype == synth.INT8:
        oc = np.zeros((B, H, Lmax, D), np.int8)
        osc = np.zeros((B, H, -(-Lmax // 256)), np.float32)
    else:
        oc = np.zeros((B, H, Lmax, D // 2), np.uint8)
        osc = np.zeros((B, H, Lmax, D // group), np.uint16)
    gc, gs = dev(oc.copy()), dev(osc.copy())
    if kv_dtype == synth.INT4_PACKED:
        gs = gs.view(torch.float16)
    L = 0
    for n, mag in pieces:
        x = _x(rng, (B, H, n, D), mag)
        xg = dev(x.view(np.int16)).view(torch.bfloat16)
        qa.qattn_kv_append(xg, gc, gs, L, kv_dtype, group=group)
        torch.cuda.synchronize()
        oc, osc = orc.kv_append(x, oc, osc, L, kv_dtype, group=group)
        L += n
        got_c = gc.cpu().numpy()
        got_s = gs.cpu().numpy() if kv_dtype == synth.INT8 else gs.view(torch.int16).cpu().numpy().view(np.uint16)
        bad = np.nonzero(got_c.view(np.uint8) != oc.view(np.uint8))
        assert bad[0].size == 0, "codes differ at %d places after L=%d, first %s" % (
            bad[0].size, L, [v[:3] for v in bad])
        assert np.array_equal(got_s.view(np.uint16 if kv_dtype != synth.INT8 else np.uint32),
                              osc.view(np.uint16 if kv_dtype != synth.INT8 else np.uint32))


@pytest.mark.parametrize("D", [64, 128])
def test_int8_sequence(orc, D):
    # aligned block, partial block, growth inside a block, smaller piece,
    # a piece across a block boundary, a single token, a long run
    pieces = [(256, 1.0), (100, 1.0), (30, 4.0), (60, 0.5), (200, 1.0), (1, 8.0), (600, 2.0)]
    _run_sequence(orc, synth.INT8, 2, 3, D, 2048, pieces, seed=D)


def test_int8_zero_rows_and_tiny_values(orc):
    pieces = [(50, 0.0), (20, 1e-30), (10, 1.0)]
    _run_sequence(orc, synth.INT8, 1, 2, 128, 512, pieces, seed=3)


@pytest.mark.parametrize("group", [128, 64])
def test_int4_sequence(orc, group):
    pieces = [(1, 1.0), (37, 3.0), (256, 0.2), (5, 1e-6), (300, 1.0)]
    _run_sequence(orc, synth.INT4_PACKED, 2, 3, 128, 1024, pieces, group=group, seed=group)


def test_int8_decode_problem_size(orc):
    """The INT8 decode problem's cache (B64, H_kv 8, D 128) with its seeded
    codes and scales: append 4 tokens across the boundary of block 31 and a
    new block (the last block's scale grows and its earlier codes are
    requantized), and a 256-token chunk; the oracle checks every head."""
    p = synth.INT8_KV_DECODE
    dd = synth.make_decode(p)
    B, H, L0, D = dd["k"].shape
    Lmax = L0 + 512
    cache = np.zeros((B, H, Lmax, D), np.int8)
    cache[:, :, :L0] = dd["k"]
    sc = np.zeros((B, H, -(-Lmax // 256)), np.float32)
    sc[:, :, :dd["k_scales"].shape[2]] = dd["k_scales"]
    gc, gs = dev(cache.copy()), dev(sc.copy())
    rng = np.random.default_rng(9)
    L = L0 - 2
    for n in (4, 256):
        x = _x(rng, (B, H, n, D), 1.5)
        qa.qattn_kv_append(dev(x.view(np.int16)).view(torch.bfloat16), gc, gs, L, synth.INT8)
        torch.cuda.synchronize()
        cache, sc = orc.kv_append(x, cache, sc, L, synth.INT8)
        L += n
    assert np.array_equal(gc.cpu().numpy(), cache)
    assert np.array_equal(gs.cpu().numpy().view(np.uint32), sc.view(np.uint32))


@pytest.mark.parametrize("group", [128, 64])
def test_int4_ties_and_near_ties(orc, group):
    """Rows whose every group has maximum |x| = 7 exactly (fp16 scale exactly
    1) holding half-integers k + 1/2 (exact ties, decided to even) and their
    bf16 neighbours one unit away: every code as the IEEE quotient decides
    it, against the oracle."""
    B, H, n, D, Lmax = 1, 2, 64, 128, 128
    rng = np.random.default_rng(group)
    half = (rng.integers(-7, 7, (B, H, n, D)) + 0.5).astype(np.float32)
    x = np.where(rng.random((B, H, n, D)) < 0.6, half, rng.uniform(-6.9, 6.9, (B, H, n, D))).astype(np.float32)
    for g0 in range(0, D, group):
        x[..., g0] = np.where(rng.random((B, H, n)) < 0.5, 7.0, -7.0)
    bits = synth.f32_to_bf16_bits(x)
    step = np.where(rng.random(bits.shape) < 0.5, 1, -1).astype(np.int32)
    near = (rng.random(bits.shape) < 0.2) & (np.abs(x) < 6.9)
    bits = np.where(near, (bits.astype(np.int32) + step).astype(np.uint16), bits)
    oc = np.zeros((B, H, Lmax, D // 2), np.uint8)
    osc = np.zeros((B, H, Lmax, D // group), np.uint16)
    gc = dev(oc.copy())
    gs = dev(osc.copy()).view(torch.float16)
    xg = dev(bits.view(np.int16)).view(torch.bfloat16)
    qa.qattn_kv_append(xg, gc, gs, 0, synth.INT4_PACKED, group=group)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    oc, osc = orc.kv_append(bits, oc, osc, 0, synth.INT4_PACKED, group=group)
    assert np.array_equal(osc[:, :, :n], np.full((B, H, n, D // group), 0x3C00, np.uint16))   # scale 1.0
    assert np.array_equal(gc.cpu().numpy(), oc)
    assert np.array_equal(gs.view(torch.int16).cpu().numpy().view(np.uint16), osc)
