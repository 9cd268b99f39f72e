"""Pins for the oracle's quantized prefill attention.

The tiled loop with a running softmax follows "FlashAttention 的 INT8/INT4
量化" (三层实现详解 / 第一层), with the page's normalisation corrected to the
standard running-max form; FP8 attention with the output returned in the
original precision follows "MindIE-SD quantization" (FA量化 / FP8 Attention).

CPU only.
"""
import numpy as np
import pytest
import torch

import synth


def _np_layout(x, layout):
    """[B,H,N,D] view of a tensor stored in `layout`."""
    return x if layout == synth.BNSD else x.transpose(0, 2, 1, 3)


def _store(x_bhnd, layout):
    return np.ascontiguousarray(x_bhnd if layout == synth.BNSD else x_bhnd.transpose(0, 2, 1, 3))


def _ref_attention(qd, kd, vd, causal, scale):
    """float64 softmax(q k^T * scale) v, [N, D] per head."""
    s = (qd @ kd.T) * scale
    if causal:
        s = np.where(np.tril(np.ones(s.shape, bool)), s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return (p @ vd) / p.sum(axis=1, keepdims=True)


def _bf16_to_f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("causal", [False, True])
def test_running_softmax_equals_exact_softmax_without_quantization(orc, layout, causal):
    """float32 'codes', random per-block scales, probabilities not rounded:
    the tiled running softmax must equal the one-shot softmax (several key
    tiles and a ragged tail), and its LSE the float64 log-sum-exp of the
    scaled scores (natural log)."""
    B, H, N, D = 1, 2, 300, 64
    rng = np.random.default_rng(21)
    q = rng.standard_normal((B, H, N, D)).astype(np.float32)
    k = rng.standard_normal((B, H, N, D)).astype(np.float32)
    v = rng.standard_normal((B, H, N, D)).astype(np.float32)
    qs = rng.uniform(0.5, 2, (B, H, 3)).astype(np.float32)
    ks = rng.uniform(0.5, 2, (B, H, 2)).astype(np.float32)
    vs = rng.uniform(0.5, 2, (B, H, 2)).astype(np.float32)
    rows = list(range(N))
    res = orc.prefill_rows(_store(q, layout), qs, _store(k, layout), ks, _store(v, layout), vs,
                           orc.F32, layout, causal, {(0, h): rows for h in range(H)},
                           p_quant=False, want_f64=True, want_lse=True)
    tok = np.arange(N)
    for h in range(H):
        qd = q[0, h].astype(np.float64) * qs[0, h, tok // 128, None]
        kd = k[0, h].astype(np.float64) * ks[0, h, tok // 256, None]
        vd = v[0, h].astype(np.float64) * vs[0, h, tok // 256, None]
        ref = _ref_attention(qd, kd, vd, causal, 1.0 / np.sqrt(D))
        got = res[(0, h)][1]
        assert np.abs(got - ref).max() <= 2e-5 * np.abs(vd).max()
        sc = (qd @ kd.T) / np.sqrt(D)
        if causal:
            sc = np.where(np.tril(np.ones(sc.shape, bool)), sc, -np.inf)
        mx = sc.max(axis=1)
        ref_lse = mx + np.log(np.exp(sc - mx[:, None]).sum(axis=1))
        assert np.abs(res[(0, h)][2] - ref_lse).max() <= 1e-4 * max(1.0, np.abs(ref_lse).max())


def test_explicit_softmax_scale(orc):
    """A given softmax scale replaces 1/sqrt(D): float32 'codes', P not
    rounded, against float64 softmax at that scale."""
    B, H, N, D = 1, 1, 200, 64
    rng = np.random.default_rng(23)
    q = rng.standard_normal((B, H, N, D)).astype(np.float32)
    k = rng.standard_normal((B, H, N, D)).astype(np.float32)
    v = rng.standard_normal((B, H, N, D)).astype(np.float32)
    ones_q, ones_kv = np.ones((B, H, 2), np.float32), np.ones((B, H, 1), np.float32)
    rows = {(0, 0): list(range(N))}
    for scale in (0.37, 0.0):
        res = orc.prefill_rows(q, ones_q, k, ones_kv, v, ones_kv, orc.F32, synth.BNSD, False, rows,
                               softmax_scale=scale, p_quant=False, want_f64=True)
        want = _ref_attention(q[0, 0].astype(np.float64), k[0, 0].astype(np.float64), v[0, 0].astype(np.float64),
                              False, scale if scale > 0 else 1.0 / np.sqrt(D))
        assert np.abs(res[(0, 0)][1] - want).max() <= 2e-5 * np.abs(v).max()


@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3])
def test_constant_v_reproduces_v(orc, code_dtype):
    """Every value row equal: the output is that row whatever the weights,
    because the normaliser sums the same rounded probabilities."""
    B, H, N, D = 1, 1, 384, 64
    rng = np.random.default_rng(22)
    q = rng.integers(-127, 128, (B, H, N, D)).astype(np.int8).view(np.uint8)
    k = rng.integers(-127, 128, (B, H, N, D)).astype(np.int8).view(np.uint8)
    if code_dtype == synth.FP8_E4M3:
        q = (q & 0x77) | 0x20
        k = (k & 0x77) | 0x20
    row = rng.integers(-127, 128, D).astype(np.int8).view(np.uint8)
    if code_dtype == synth.FP8_E4M3:
        row = row & 0xF7          # avoid the NaN pattern
    v = np.broadcast_to(row, (B, H, N, D)).copy()
    qs = np.full((B, H, 3), 0.01, np.float32)
    ks = np.full((B, H, 2), 0.02, np.float32)
    vs = np.full((B, H, 2), 0.5, np.float32)
    for causal in (False, True):
        res = orc.prefill_rows(q, qs, k, ks, v, vs, code_dtype, synth.BNSD, causal,
                               {(0, 0): [0, 1, 127, 128, 200, 383]})
        if code_dtype == synth.INT8:
            val = row.view(np.int8).astype(np.float64) * 0.5
        else:
            val = orc.e4m3_decode(row).astype(np.float64) * 0.5
        expect = synth.f32_to_bf16_bits(val)
        for r in res[(0, 0)][0]:
            assert np.array_equal(r, expect)


def test_single_key_returns_that_value(orc):
    B, H, D = 1, 1, 64
    rng = np.random.default_rng(23)
    q = rng.integers(-127, 128, (B, H, 5, D)).astype(np.int8).view(np.uint8)
    k = rng.integers(-127, 128, (B, H, 1, D)).astype(np.int8).view(np.uint8)
    v = rng.integers(-127, 128, (B, H, 1, D)).astype(np.int8).view(np.uint8)
    res = orc.prefill_rows(q, np.ones((1, 1, 1), np.float32), k, np.ones((1, 1, 1), np.float32),
                           v, np.full((1, 1, 1), 0.25, np.float32), synth.INT8, synth.BNSD, False,
                           {(0, 0): list(range(5))})
    expect = synth.f32_to_bf16_bits(v[0, 0, 0].view(np.int8).astype(np.float64) * 0.25)
    for r in res[(0, 0)][0]:
        assert np.array_equal(r, expect)


def _quantize_p(p32: np.ndarray, code_dtype):
    if code_dtype == synth.INT8:
        return np.round(p32 * np.float32(127.0)).astype(np.float64) / 127.0    # half to even
    return torch.from_numpy(p32).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def _weights_brute_force(s32: np.ndarray, code_dtype, tile=128):
    """Effective weights of one query row, written directly from the rule
    'each key tile's probabilities are rounded relative to the running max
    at that tile, and earlier tiles are rescaled to the final max'."""
    n = len(s32)
    parts, m_run = [], -np.inf
    for t0 in range(0, n, tile):
        s = s32[t0:t0 + tile]
        m_run = max(m_run, float(s.max()))
        p = np.exp((s - np.float32(m_run)).astype(np.float64)).astype(np.float32)
        parts.append((m_run, _quantize_p(p, code_dtype)))
    m_fin = parts[-1][0]
    w = np.concatenate([pq * np.exp(m - m_fin) for m, pq in parts])
    return w / w.sum()


@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3])
@pytest.mark.parametrize("nkv", [100, 200, 128])
def test_weights_from_one_hot_values(orc, code_dtype, nkv):
    """With V = one-hot rows the output row is the vector of effective
    attention weights: they sum to one and equal the brute-force rule."""
    D = 256
    rng = np.random.default_rng(24 + nkv)
    q = rng.integers(-127, 128, (1, 1, 4, D)).astype(np.int8)
    k = rng.integers(-127, 128, (1, 1, nkv, D)).astype(np.int8)
    if code_dtype == synth.INT8:
        qb, kb = q.view(np.uint8), k.view(np.uint8)
        qv, kv = q.astype(np.float64), k.astype(np.float64)
        one = 1
    else:
        qb = ((q.view(np.uint8) & 0xD7) | 0x20).astype(np.uint8)   # no NaN pattern
        kb = ((k.view(np.uint8) & 0xD7) | 0x20).astype(np.uint8)
        qv, kv = orc.e4m3_decode(qb).astype(np.float64), orc.e4m3_decode(kb).astype(np.float64)
        one = 0x38                      # e4m3 code of 1.0
    v = np.zeros((1, 1, nkv, D), np.uint8)
    v[0, 0, np.arange(nkv), np.arange(nkv)] = one
    qs = np.array([[[0.013]]], np.float32)
    ks = np.array([[[0.011]]], np.float32)
    vs = np.ones((1, 1, 1), np.float32)
    res = orc.prefill_rows(qb, qs, kb, ks, v, vs, code_dtype, synth.BNSD, False,
                           {(0, 0): [0, 1, 2, 3]}, want_f64=True)
    w_all = res[(0, 0)][1]
    scale = np.float32(1.0 / np.sqrt(np.float32(D)))
    for r in range(4):
        w = w_all[r, :nkv]
        assert abs(w.sum() - 1.0) < 1e-12
        assert np.all(w_all[r, nkv:] == 0)
        dot = (qv[0, 0, r] @ kv[0, 0].T).astype(np.float32)
        s32 = dot * qs[0, 0, 0] * ks[0, 0, 0] * scale          # float32, same order
        ref = _weights_brute_force(s32.astype(np.float32), code_dtype)
        step = (1 / 127 if code_dtype == synth.INT8 else 1 / 16) / (1.0 / max(w.max(), 1e-30))
        assert np.abs(w - ref).max() <= step
        # all but rare rounding-boundary cases agree to float32 precision
        assert np.mean(np.abs(w - ref) <= 1e-6 * ref + 1e-15) >= 0.97


@pytest.mark.parametrize("code_dtype,tol", [(synth.INT8, 0.03), (synth.FP8_E4M3, 0.12)])
def test_quantized_pipeline_approximates_exact_attention(orc, code_dtype, tol):
    """Rotate Q and K with the same orthogonal matrix, quantize per block,
    attend: the result stays close to float64 attention on the original
    inputs; rotating only Q (a plausible slip) does not."""
    p = synth.scaled(synth.INT8_CAUSAL, H=2, N=512, D=64, code_dtype=code_dtype)
    d = synth.make_prefill(p)
    R = d["rot"]
    qc, qs = orc.rotate_block_quant(d["q"], p.in_dtype, p.layout, R, 128, code_dtype)
    kc, ks = orc.rotate_block_quant(d["k"], p.in_dtype, p.layout, R, 256, code_dtype)
    vc, vs = orc.rotate_block_quant(d["v"], p.in_dtype, p.layout, None, 256, code_dtype)
    rows = {(0, h): list(range(0, 512, 3)) for h in range(2)}
    got = orc.prefill_rows(qc, qs, kc, ks, vc, vs, code_dtype, p.layout, True, rows, want_f64=True)
    ref = orc.exact_rows(d["q"], d["k"], d["v"], p.in_dtype, p.layout, True, rows)
    vmax = np.abs(_bf16_to_f64(d["v"])).max()
    for key in rows:
        assert np.abs(got[key][1] - ref[key]).max() <= tol * vmax
    kc_bad, ks_bad = orc.rotate_block_quant(d["k"], p.in_dtype, p.layout, None, 256, code_dtype)
    bad = orc.prefill_rows(qc, qs, kc_bad, ks_bad, vc, vs, code_dtype, p.layout, True, rows, want_f64=True)
    assert max(np.abs(bad[k][1] - ref[k]).max() for k in rows) > 3 * tol * vmax


def test_exact_attention_is_rotation_invariant(orc):
    """softmax((QR)(KR)^T) V = softmax(Q K^T) V for orthogonal R."""
    rng = np.random.default_rng(26)
    N, D = 200, 64
    q = rng.standard_normal((N, D))
    k = rng.standard_normal((N, D))
    v = rng.standard_normal((N, D))
    R = synth.haar_orthogonal(3, 4, D).astype(np.float64)
    a = _ref_attention(q @ R, k @ R, v, True, 0.125)
    b = _ref_attention(q, k, v, True, 0.125)
    assert np.abs(a - b).max() < 1e-5
    bits = lambda x: synth.f32_to_bf16_bits(x)[None, None]
    res = orc.exact_rows(bits(q), bits(k), bits(v), synth.BF16, synth.BNSD, True, {(0, 0): list(range(N))})
    qf, kf, vf = (synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x)).astype(np.float64) for x in (q, k, v))
    assert np.abs(res[(0, 0)] - _ref_attention(qf, kf, vf, True, 1 / np.sqrt(D))).max() < 1e-12
