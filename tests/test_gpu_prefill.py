"""GPU parity of the tcgen05 prefill kernel against the oracle.

The CUDA path quantizes with its own kernel and attends; the oracle
quantizes with its own code and attends. Codes must agree bit for bit;
outputs within max-abs <= 1e-2 max|V| and mean-abs <= 1e-3 max|V| (V
dequantized, per head). The error against unquantized float64 attention is
reported as well.
"""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import (assert_close, bf16_to_f64, dequant_v_max, dev_bits, gpu_quant_all, head_rows)

pytestmark = pytest.mark.gpu


def _run(orc, p, d, rows_by_head, check_codes=True, report=None):
    (qc, qs), (kc, ks), (vc, vs) = gpu_quant_all(d)
    lse = torch.empty((p.B, p.H, p.N), dtype=torch.float32, device="cuda")
    out = qa.qattn_prefill(qc, qs, kc, ks, vc, vs, p.code_dtype, p.layout, p.causal, lse=lse)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    out_bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    lse_np = lse.cpu().numpy()
    heads = sorted({(b, h) for (b, h) in rows_by_head})
    oq = orc.rotate_block_quant(d["q"], p.in_dtype, p.layout, d["rot"], p.q_block, p.code_dtype, heads=heads)
    ok_ = orc.rotate_block_quant(d["k"], p.in_dtype, p.layout, d["rot"], p.kv_block, p.code_dtype, heads=heads)
    ov = orc.rotate_block_quant(d["v"], p.in_dtype, p.layout, None, p.kv_block, p.code_dtype, heads=heads)
    if check_codes:
        for (g, o) in (((qc, qs), oq), ((kc, ks), ok_), ((vc, vs), ov)):
            gcodes, gsc = g[0].cpu().numpy(), g[1].cpu().numpy()
            for (b, h) in heads:
                assert np.array_equal(head_rows(gcodes, p.layout, b, h), head_rows(o[0], p.layout, b, h))
                assert np.array_equal(gsc[b, h], o[1][b, h])
    ref = orc.prefill_rows(*oq, *ok_, *ov, p.code_dtype, p.layout, p.causal, rows_by_head,
                           want_f64=True, want_lse=True)
    exact = orc.exact_rows(d["q"], d["k"], d["v"], p.in_dtype, p.layout, p.causal, rows_by_head)
    worst = (0.0, 0.0)
    for (b, h), rows in rows_by_head.items():
        got = bf16_to_f64(head_rows(out_bits, p.layout, b, h)[rows])
        vmax = dequant_v_max(ov[0], ov[1], p.code_dtype, p.layout, b, h, orc)
        # both sides round their output to bfloat16; compare those outputs
        e = assert_close(got, bf16_to_f64(ref[(b, h)][0]), vmax, "head (%d,%d)" % (b, h))
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
        assert np.abs(lse_np[b, h, rows] - ref[(b, h)][2]).max() < 1e-2
        if report is not None:
            report.append(float(np.abs(got - exact[(b, h)]).max() / vmax))
    return worst


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3])
@pytest.mark.parametrize("causal", [False, True])
def test_small_shapes(orc, D, layout, code_dtype, causal):
    """Several query and key tiles, ragged tails (N = 300), both layouts."""
    p = synth.PrefillProblem("small", 2, 3, 300, D, synth.BF16, code_dtype, layout, causal=causal,
                             rotate=True, seed=100 + D + layout * 3 + code_dtype * 5 + causal)
    d = synth.make_prefill(p)
    rows = {(b, h): list(range(p.N)) for b in range(p.B) for h in range(p.H)}
    _run(orc, p, d, rows)


@pytest.mark.parametrize("N", [1, 100, 128, 129, 256, 640])
def test_sequence_lengths(orc, N):
    p = synth.PrefillProblem("len", 1, 2, N, 128, synth.BF16, synth.INT8, synth.BNSD, causal=True,
                             rotate=True, seed=200 + N, outlier_frac=0.01)
    d = synth.make_prefill(p)
    _run(orc, p, d, {(0, h): list(range(N)) for h in range(2)})


def test_cross_attention_lengths(orc):
    """N_q != N_kv (non-causal)."""
    p = synth.PrefillProblem("x", 1, 2, 200, 128, synth.BF16, synth.FP8_E4M3, synth.BNSD, causal=False,
                             rotate=True, seed=300)
    d = synth.make_prefill(p)
    pk = synth.PrefillProblem("x", 1, 2, 700, 128, synth.BF16, synth.FP8_E4M3, synth.BNSD, causal=False,
                              rotate=True, seed=301)
    dk = synth.make_prefill(pk)
    R = d["rot"]
    q = dev_bits(d["q"], p.in_dtype)
    k = dev_bits(dk["k"], p.in_dtype)
    v = dev_bits(dk["v"], p.in_dtype)
    r = torch.from_numpy(R).cuda()
    qc, qs = qa.qattn_rotate_block_quant(q, p.layout, r, 128, p.code_dtype)
    kc, ks = qa.qattn_rotate_block_quant(k, p.layout, r, 256, p.code_dtype)
    vc, vs = qa.qattn_rotate_block_quant(v, p.layout, None, 256, p.code_dtype)
    out = qa.qattn_prefill(qc, qs, kc, ks, vc, vs, p.code_dtype, p.layout, False)
    torch.cuda.synchronize()
    oq = orc.rotate_block_quant(d["q"], p.in_dtype, p.layout, R, 128, p.code_dtype)
    ok_ = orc.rotate_block_quant(dk["k"], p.in_dtype, p.layout, R, 256, p.code_dtype)
    ov = orc.rotate_block_quant(dk["v"], p.in_dtype, p.layout, None, 256, p.code_dtype)
    rows = {(0, h): list(range(200)) for h in range(2)}
    ref = orc.prefill_rows(*oq, *ok_, *ov, p.code_dtype, p.layout, False, rows, want_f64=True)
    got_bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for (b, h) in rows:
        vmax = dequant_v_max(ov[0], ov[1], p.code_dtype, p.layout, b, h, orc)
        assert_close(bf16_to_f64(got_bits[b, h]), bf16_to_f64(ref[(b, h)][0]), vmax, "cross")


@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3])
def test_explicit_softmax_scale(orc, code_dtype):
    """A softmax scale other than 1/sqrt(D), causal, ragged: CUDA path and
    oracle given the same scale."""
    p = synth.PrefillProblem("x", 1, 2, 300, 128, synth.BF16, code_dtype, synth.BNSD, causal=True,
                             rotate=True, seed=320)
    d = synth.make_prefill(p)
    (qc, qs), (kc, ks), (vc, vs) = gpu_quant_all(d)
    out = qa.qattn_prefill(qc, qs, kc, ks, vc, vs, code_dtype, p.layout, True, softmax_scale=0.37)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    oq = orc.rotate_block_quant(d["q"], p.in_dtype, p.layout, d["rot"], 128, code_dtype)
    ok_ = orc.rotate_block_quant(d["k"], p.in_dtype, p.layout, d["rot"], 256, code_dtype)
    ov = orc.rotate_block_quant(d["v"], p.in_dtype, p.layout, None, 256, code_dtype)
    rows = {(0, h): list(range(p.N)) for h in range(p.H)}
    ref = orc.prefill_rows(*oq, *ok_, *ov, code_dtype, p.layout, True, rows, softmax_scale=0.37, want_f64=True)
    got_bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for (b, h) in rows:
        vmax = dequant_v_max(ov[0], ov[1], code_dtype, p.layout, b, h, orc)
        assert_close(bf16_to_f64(got_bits[b, h]), bf16_to_f64(ref[(b, h)][0]), vmax, "scale 0.37")


@pytest.mark.parametrize("code_dtype", [synth.INT8, synth.FP8_E4M3])
def test_key_scales_beyond_the_shared_memory_cache(orc, code_dtype):
    """More than 512 K/V blocks (131072 keys): the block scales past the
    first 512 come from global memory. Per-token log-normal magnitudes give
    every block its own scale, and the last block is ragged."""
    nkv = 513 * 256 + 100
    p = synth.PrefillProblem("x", 1, 1, 200, 128, synth.BF16, code_dtype, synth.BNSD, causal=False,
                             rotate=True, seed=310)
    d = synth.make_prefill(p)
    pk = synth.PrefillProblem("x", 1, 1, nkv, 128, synth.BF16, code_dtype, synth.BNSD, causal=False,
                              rotate=True, seed=311, lognormal_sigma=0.7)
    dk = synth.make_prefill(pk)
    R = d["rot"]
    r = torch.from_numpy(R).cuda()
    qc, qs = qa.qattn_rotate_block_quant(dev_bits(d["q"], p.in_dtype), p.layout, r, 128, code_dtype)
    kc, ks = qa.qattn_rotate_block_quant(dev_bits(dk["k"], p.in_dtype), p.layout, r, 256, code_dtype)
    vc, vs = qa.qattn_rotate_block_quant(dev_bits(dk["v"], p.in_dtype), p.layout, None, 256, code_dtype)
    assert ks.shape[-1] == 514
    out = qa.qattn_prefill(qc, qs, kc, ks, vc, vs, code_dtype, p.layout, False)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    oq = orc.rotate_block_quant(d["q"], p.in_dtype, p.layout, R, 128, code_dtype)
    ok_ = orc.rotate_block_quant(dk["k"], p.in_dtype, p.layout, R, 256, code_dtype)
    ov = orc.rotate_block_quant(dk["v"], p.in_dtype, p.layout, None, 256, code_dtype)
    assert np.array_equal(ks.cpu().numpy(), ok_[1]) and np.array_equal(vs.cpu().numpy(), ov[1])
    rows = {(0, 0): [0, 57, 128, 199]}
    ref = orc.prefill_rows(*oq, *ok_, *ov, code_dtype, p.layout, False, rows, want_f64=True)
    got_bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
    vmax = dequant_v_max(ov[0], ov[1], code_dtype, p.layout, 0, 0, orc)
    assert_close(bf16_to_f64(got_bits[0, 0][rows[(0, 0)]]), bf16_to_f64(ref[(0, 0)][0]), vmax, "long kv")


@pytest.mark.parametrize("prob", ["tiny_fp8_b1h2n256d64", "int8_causal_b1h32n4096d128", "fp8_bsnd_b1h24n16384d128"])
def test_full_size(orc, prob):
    """The stated problems at full size, in the benchmark's launch
    configuration; the oracle computes sampled rows (all rows for the tiny
    problem) of sampled heads."""
    p = synth.PROBLEMS[prob]
    d = synth.make_prefill(p)
    rng = np.random.default_rng(11)
    if p.N <= 256:
        rows = {(0, h): list(range(p.N)) for h in range(p.H)}
    else:
        heads = [0, p.H - 1] + [int(x) for x in rng.integers(1, p.H - 1, 1)]
        rows = {}
        for h in heads:
            r = sorted(set([0, 1, 127, 128, p.N - 1] + [int(x) for x in rng.integers(0, p.N, 40)]))
            rows[(0, h)] = r
    report = []
    worst = _run(orc, p, d, rows, report=report)
    print("%s: worst max-abs/max|V| %.2e mean %.2e; vs fp64 exact %.2e" % (prob, worst[0], worst[1], max(report)))
