"""Pins for the oracle's KV-cache quantize-on-append.

INT8 cache written in the decode phase: "INT8 量化算子" page, ops-transformer
item 3 (KV Cache 也量化). Packed INT4 cache with one fp16 scale per group:
"ops-transformer INT8/INT4 量化推理" page, 5.1 and 5.2.

The pins do not restate the oracle's loops. They check it against the
already pinned block quantizer (a block appended in pieces whose first piece
holds the block's largest value must equal the block quantized at once),
against library routines (numpy float16 rounding, torch float32 division and
rounding for the INT4 codes), and against error bounds and invariants.

CPU only.
"""
import numpy as np
import pytest
import torch

import synth


def _bf16(rng, shape, scale=1.0):
    return synth.f32_to_bf16_bits(rng.standard_normal(shape) * scale)


def _int8_empty(B, H, Lmax, D, blk=256):
    return np.zeros((B, H, Lmax, D), np.int8), np.zeros((B, H, -(-Lmax // blk)), np.float32)


def test_f32_to_f16_matches_numpy(orc):
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.standard_normal(20000) * np.exp(rng.uniform(-25, 12, 20000)),
        np.float32(2.0) ** np.arange(-30, 17),
        [0.0, -0.0, 65504.0, 65519.0, 65520.0, 1e-8, 5.96e-8, 2.98e-8, 6.1e-5],
    ]).astype(np.float32)
    # exact float16 midpoints and their float32 neighbours
    h = np.arange(0, 0x7BFF, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = ((h[:-1] + h[1:]) / 2).astype(np.float32)
    xs = np.concatenate([xs, mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0))])
    got = np.array([orc.f32_to_f16_bits(v) for v in xs], dtype=np.uint16)
    with np.errstate(over="ignore"):                               # 65520 and above -> inf
        want = xs.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("splits", [[256], [100, 156], [1, 255], [7, 1, 80, 168]])
def test_int8_pieces_with_max_first_equal_block_quantizer(orc, splits):
    """Appending a 256-token block in pieces, the block's largest value in the
    first piece, gives exactly the codes and scale of quantizing the block at
    once (the scale never changes after the first piece)."""
    B, H, D = 2, 3, 128
    rng = np.random.default_rng(len(splits))
    x = _bf16(rng, (B, H, 256, D))
    # put the largest magnitude of every (b, h) into the first piece
    for b in range(B):
        for h in range(H):
            f = synth.bf16_bits_to_f32(x[b, h])
            t, d = np.unravel_index(np.argmax(np.abs(f)), f.shape)
            x[b, h, [0, t]] = x[b, h, [t, 0]]
    cache, sc = _int8_empty(B, H, 256, D)
    L = 0
    for n in splits:
        cache, sc = orc.kv_append(x[:, :, L:L + n], cache, sc, L, synth.INT8)
        L += n
    codes, scales = orc.rotate_block_quant(x, synth.BF16, synth.BNSD, None, 256, synth.INT8)
    assert np.array_equal(cache.view(np.uint8), codes)
    assert np.array_equal(sc.view(np.uint32), scales.view(np.uint32))


def test_int8_growing_scale_requantizes_old_tokens(orc):
    """When a later piece holds a larger value the block scale becomes that of
    the whole block (bit-exact), the later tokens' codes equal the block
    quantizer's, and the requantized earlier codes stay within the two
    rounding steps of their values."""
    B, H, D = 1, 4, 128
    rng = np.random.default_rng(7)
    x = _bf16(rng, (B, H, 300, D))
    x[:, :, 250] = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(x[:, :, 250]) * 8)   # late, large
    cache, sc = _int8_empty(B, H, 512, D)
    cache, sc = orc.kv_append(x[:, :, :200], cache, sc, 0, synth.INT8)
    s_first = sc[:, :, 0].copy()
    cache, sc = orc.kv_append(x[:, :, 200:300], cache, sc, 200, synth.INT8)
    full = np.zeros((B, H, 512, D), np.uint16)
    full[:, :, :300] = x
    codes, scales = orc.rotate_block_quant(full[:, :, :300], synth.BF16, synth.BNSD, None, 256, synth.INT8)
    # block 0: scale of tokens 0..255, later tokens exact
    assert np.array_equal(sc[:, :, 0].view(np.uint32), scales[:, :, 0].view(np.uint32))
    assert np.all(sc[:, :, 0] > s_first)
    assert np.array_equal(cache[:, :, 200:256].view(np.uint8), codes[:, :, 200:256])
    # block 1 (tokens 256..299) is new: equal to the quantizer on its own
    assert np.array_equal(cache[:, :, 256:300].view(np.uint8), codes[:, :, 256:300])
    assert np.array_equal(sc[:, :, 1].view(np.uint32), scales[:, :, 1].view(np.uint32))
    # requantized tokens 0..199: within s_first/2 + s/2 (+ float32 slack)
    xf = synth.bf16_bits_to_f32(x[:, :, :200]).astype(np.float64)
    s = sc[:, :, 0].astype(np.float64)[:, :, None, None]
    s0 = s_first.astype(np.float64)[:, :, None, None]
    err = np.abs(cache[:, :, :200].astype(np.float64) * s - xf)
    assert np.all(err <= s0 / 2 + s / 2 + 1e-6 * np.abs(xf))
    # tokens beyond the appended range are untouched
    assert not cache[:, :, 300:].any()
    assert not sc[:, :, 2:].any()


def test_int8_smaller_later_piece_keeps_codes(orc):
    B, H, D = 1, 2, 64
    rng = np.random.default_rng(11)
    a = _bf16(rng, (B, H, 40, D), 2.0)
    b = _bf16(rng, (B, H, 30, D), 0.5)
    cache, sc = _int8_empty(B, H, 256, D)
    cache, sc = orc.kv_append(a, cache, sc, 0, synth.INT8)
    c1, s1 = cache.copy(), sc.copy()
    cache, sc = orc.kv_append(b, cache, sc, 40, synth.INT8)
    if np.all(np.abs(synth.bf16_bits_to_f32(b)).max(axis=(2, 3)) <= s1[:, :, 0] * 127):
        assert np.array_equal(cache[:, :, :40], c1[:, :, :40])
        assert np.array_equal(sc, s1)
    # the new codes are RNE(x / s) by torch float32 arithmetic
    xt = torch.from_numpy(synth.bf16_bits_to_f32(b))
    st = torch.from_numpy(sc[:, :, 0])[:, :, None, None]
    want = torch.round(xt / st).clamp(-127, 127).to(torch.int8).numpy()
    assert np.array_equal(cache[:, :, 40:70], want)


@pytest.mark.parametrize("group", [128, 64])
def test_int4_append_codes_and_scales(orc, group):
    B, H, D, Lmax = 2, 2, 128, 64
    rng = np.random.default_rng(group)
    x = _bf16(rng, (B, H, 20, D), 3.0)
    x[0, 0, 3] = 0                                                  # an all-zero token
    cache = np.zeros((B, H, Lmax, D // 2), np.uint8)
    sc = np.zeros((B, H, Lmax, D // group), np.uint16)
    cache, sc = orc.kv_append(x[:, :, :5], cache, sc, 10, synth.INT4_PACKED, group=group)
    cache, sc = orc.kv_append(x[:, :, 5:], cache, sc, 15, synth.INT4_PACKED, group=group)
    xf = synth.bf16_bits_to_f32(x).reshape(B, H, 20, D // group, group)
    amax = np.abs(xf).max(axis=-1)
    # scale: float32 absmax / 7, rounded to fp16 by numpy
    want_s = (torch.from_numpy(amax) / 7.0).numpy().astype(np.float32).astype(np.float16).view(np.uint16)
    assert np.array_equal(sc[:, :, 10:30], want_s)
    # codes: independent unpacker (low nibble = even element), then torch RNE
    lo = ((cache[:, :, 10:30] & 0xF).astype(np.int16) ^ 8) - 8
    hi = ((cache[:, :, 10:30] >> 4).astype(np.int16) ^ 8) - 8
    codes = np.stack([lo, hi], axis=-1).reshape(B, H, 20, D // group, group)
    s = torch.from_numpy(want_s.view(np.float16).astype(np.float32))[..., None]
    want_c = torch.where(s > 0, torch.round(torch.from_numpy(xf) / s).clamp(-7, 7), torch.zeros(()))
    assert np.array_equal(codes, want_c.numpy().astype(np.int16))
    # the group maximum maps to +-7 and every value is within s/2
    sf = s.numpy().astype(np.float64)
    assert np.all(np.abs(codes * sf - xf) <= sf / 2 + 1e-7)
    nz = amax > 0
    assert np.all(np.abs(codes).max(axis=-1)[nz] == 7)
    assert not codes[0, 0, 3].any() and not sc[0, 0, 13].any()
    # untouched rows
    assert not cache[:, :, :10].any() and not cache[:, :, 30:].any()
