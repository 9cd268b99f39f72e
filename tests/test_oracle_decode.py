"""Pins for the oracle's decode against a quantized KV cache.

INT8 cache read directly with an INT8 query: "INT8 量化算子" page,
ops-transformer section, item 3 (KV Cache 也量化) and its Int8Attention
listing. Packed INT4 with one fp16 scale per group of 128 elements:
"ops-transformer INT8/INT4 量化推理" page, 5.1 and 5.2; the nibbles are
widened to INT8 and meet the same INT8 query codes ("FlashAttention 的
INT8/INT4 量化", 第二层).

CPU only.
"""
import numpy as np
import pytest
import torch

import synth


def _scale32(D):
    """Default softmax scale as the float32 value 1/sqrt(D) (the ABI passes
    the scale as a float32)."""
    return float(np.float32(1.0) / np.sqrt(np.float32(D)))


def _np_softmax_av(scores, vals):
    s = scores - scores.max()
    p = np.exp(s)
    return (p[:, None] * vals).sum(0) / p.sum()


def _q_codes(q_bits):
    """Per-head INT8 query codes and scale with torch float32 arithmetic
    (absmax / 127, division, round half to even, clamp)."""
    q = torch.from_numpy(synth.bf16_bits_to_f32(q_bits))
    sq = q.abs().max() / 127.0
    return torch.round(q / sq).clamp(-127, 127).numpy().astype(np.int64), float(sq)


def _unpack_int4(b):
    """Independent restatement of the nibble order: low nibble = even index."""
    lo = ((b & 0xF).astype(np.int16) ^ 8) - 8
    hi = (((b >> 4) & 0xF).astype(np.int16) ^ 8) - 8
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


@pytest.mark.parametrize("L", [1000, 512])
def test_int8_decode_matches_closed_form(orc, L):
    p = synth.scaled(synth.INT8_KV_DECODE, B=2, L=L)
    d = synth.make_decode(p)
    heads = [(0, 0), (0, 5), (1, 31), (1, 12)]
    out, of = orc.decode(d["q"], d["k"], d["v"], d["k_scales"], d["v_scales"], synth.INT8, p.Hkv,
                         heads=heads, want_f64=True)
    g = p.Hq // p.Hkv
    for (b, h) in heads:
        q = torch.from_numpy(synth.bf16_bits_to_f32(d["q"][b, h, 0]))
        sq = q.abs().max() / 127.0
        qc = torch.round(q / sq).clamp(-127, 127).numpy().astype(np.int64)
        kh = h // g
        dots = d["k"][b, kh].astype(np.int64) @ qc
        blk = np.arange(L) // 256
        s = dots * float(sq) * d["k_scales"][b, kh, blk].astype(np.float64) * _scale32(p.D)
        vals = d["v"][b, kh].astype(np.float64) * d["v_scales"][b, kh, blk, None].astype(np.float64)
        ref = _np_softmax_av(s, vals)
        assert np.abs(of[b, h, 0] - ref).max() <= 1e-12 * np.abs(vals).max()
        assert np.array_equal(out[b, h, 0], synth.f32_to_bf16_bits(of[b, h, 0]))


def test_int4_decode_matches_closed_form(orc):
    p = synth.scaled(synth.INT4_KV_DECODE, B=2, L=777)
    d = synth.make_decode(p)
    heads = [(0, 0), (0, 7), (1, 30)]
    out, of = orc.decode(d["q"], d["k"], d["v"], d["k_scales"], d["v_scales"], synth.INT4_PACKED,
                         p.Hkv, heads=heads, want_f64=True)
    g = p.Hq // p.Hkv
    for (b, h) in heads:
        qc, sq = _q_codes(d["q"][b, h, 0])
        kh = h // g
        kc = _unpack_int4(d["k"][b, kh]).astype(np.int64)
        vc = _unpack_int4(d["v"][b, kh]).astype(np.float64)
        ksc = d["k_scales"][b, kh].view(np.float16).astype(np.float64)      # [L, 1]
        vsc = d["v_scales"][b, kh].view(np.float16).astype(np.float64)
        s = (kc @ qc).astype(np.float64) * ksc[:, 0] * sq * _scale32(p.D)
        ref = _np_softmax_av(s, vc * vsc[:, [0]])
        assert np.abs(of[b, h, 0] - ref).max() <= 1e-12 * np.abs(vc * vsc[:, [0]]).max()


def test_int4_group_scales_apply_per_group(orc):
    """D = 256 with groups of 128: each half of a row uses its own scale."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, L, D, G = 1, 2, 1, 50, 256, 128
    q = synth.f32_to_bf16_bits(rng.standard_normal((B, Hq, 1, D)))
    k = rng.integers(0, 256, (B, Hkv, L, D // 2)).astype(np.uint8)
    v = rng.integers(0, 256, (B, Hkv, L, D // 2)).astype(np.uint8)
    ks = synth.f64_to_f16_bits(rng.uniform(0.01, 0.05, (B, Hkv, L, D // G)))
    vs = synth.f64_to_f16_bits(rng.uniform(0.01, 0.05, (B, Hkv, L, D // G)))
    _, of = orc.decode(q, k, v, ks, vs, synth.INT4_PACKED, Hkv, group=G, want_f64=True)
    kc = _unpack_int4(k[0, 0]).astype(np.int64)
    vc = _unpack_int4(v[0, 0]).astype(np.float64)
    ksg = ks[0, 0].view(np.float16).astype(np.float64)                        # [L, groups]
    vsc = np.repeat(vs[0, 0].view(np.float16).astype(np.float64), G, axis=1)
    for h in range(Hq):
        qc, sq = _q_codes(q[0, h, 0])
        part = np.stack([kc[:, g * G:(g + 1) * G] @ qc[g * G:(g + 1) * G] for g in range(D // G)], axis=1)
        s = (part.astype(np.float64) * ksg).sum(axis=1) * sq * _scale32(D)
        ref = _np_softmax_av(s, vc * vsc)
        assert np.abs(of[0, h, 0] - ref).max() <= 1e-12


@pytest.mark.parametrize("kv_dtype", [synth.INT8, synth.INT4_PACKED])
def test_split_merge_is_invariant(orc, kv_dtype):
    base = synth.INT8_KV_DECODE if kv_dtype == synth.INT8 else synth.INT4_KV_DECODE
    p = synth.scaled(base, B=1, L=1237)
    d = synth.make_decode(p)
    heads = [(0, 0), (0, 13), (0, 31)]
    _, ref = orc.decode(d["q"], d["k"], d["v"], d["k_scales"], d["v_scales"], kv_dtype, p.Hkv,
                        heads=heads, want_f64=True, splits=1)
    for splits in (2, 5, 16, 2000):
        _, got = orc.decode(d["q"], d["k"], d["v"], d["k_scales"], d["v_scales"], kv_dtype, p.Hkv,
                            heads=heads, want_f64=True, splits=splits)
        for (b, h) in heads:
            assert np.abs(got[b, h] - ref[b, h]).max() <= 1e-12 * np.abs(ref[b, h]).max()


def test_gqa_heads_share_their_kv_head(orc):
    """Query heads h and h' with h // (Hq/Hkv) == h' // (Hq/Hkv) and the same
    query give the same output; a different kv head gives another."""
    p = synth.scaled(synth.INT8_KV_DECODE, B=1, L=300)
    d = synth.make_decode(p)
    q = d["q"].copy()
    q[0, 1] = q[0, 0]
    q[0, 4] = q[0, 0]
    out, _ = orc.decode(q, d["k"], d["v"], d["k_scales"], d["v_scales"], synth.INT8, p.Hkv,
                        heads=[(0, 0), (0, 1), (0, 4)])
    assert np.array_equal(out[0, 0], out[0, 1])
    assert not np.array_equal(out[0, 0], out[0, 4])
