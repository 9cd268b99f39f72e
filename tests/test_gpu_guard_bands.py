"""Guard bands around every output of every kernel.

Each output, scale array and workspace lives inside a larger device buffer
whose bytes are all set to a pattern beforehand; the output starts at an
offset that is 16-byte aligned (the library's requirement) but on no tile
or 128-byte boundary. After the call every byte outside the output's own
extent must still hold the pattern, so a CTA that writes past its rows
(ragged tails, the last partial tile, the INT4 half-width rows, an append
that ends exactly at the cache's end, a decode workspace sized exactly)
fails here even when the values it does write are right. With
compute-sanitizer unavailable, this is the check on out-of-bounds stores.
"""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa
import synth
from parity_util import dev, dev_bits

pytestmark = pytest.mark.gpu

PATTERN = 0xA5
FRONT = 4096 + 48          # 16-byte aligned, not 128-byte aligned
BACK = 4096 + 80


class Guarded:
    """A tensor of `shape`/`dtype` inside a pattern-filled device (or pinned
    host) buffer with FRONT bytes before it and BACK bytes after it."""

    def __init__(self, shape, dtype, device="cuda"):
        esz = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape)) * esz
        kw = {"device": device} if device == "cuda" else {"pin_memory": True}
        self.buf = torch.full((FRONT + self.n + BACK,), PATTERN, dtype=torch.uint8, **kw)
        self.t = self.buf[FRONT:FRONT + self.n].view(dtype).view(shape)

    def check(self, what):
        b = self.buf.cpu().numpy()
        front, back = b[:FRONT], b[FRONT + self.n:]
        bad_f, bad_b = np.nonzero(front != PATTERN)[0], np.nonzero(back != PATTERN)[0]
        assert bad_f.size == 0, "%s: %d bytes written before the output (first at -%d)" % (
            what, bad_f.size, FRONT - bad_f[0])
        assert bad_b.size == 0, "%s: %d bytes written after the output (first at +%d)" % (what, bad_b.size, bad_b[0])
        inside = b[FRONT:FRONT + self.n]
        assert self.n == 0 or not np.all(inside == PATTERN), "%s: output never written" % what


def _problem(N, D, layout, code, causal, seed):
    return synth.PrefillProblem("guard", 2, 3, N, D, synth.BF16, code, layout, causal=causal, rotate=True,
                                seed=seed, outlier_frac=0.01)


@pytest.mark.parametrize("N", [1, 129, 300])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("code", [synth.INT8, synth.FP8_E4M3, synth.INT4_PACKED])
def test_rotate_block_quant(N, D, layout, code):
    p = _problem(N, D, layout, synth.INT8, False, 7000 + N + D + layout)
    d = synth.make_prefill(p)
    rot = dev(d["rot"])
    for name, blk, r in (("q", 128, rot), ("k", 256, rot), ("v", 256, None)):
        x = dev_bits(d[name], p.in_dtype)
        shape = tuple(x.shape[:-1]) + ((D // 2,) if code == synth.INT4_PACKED else (D,))
        codes = Guarded(shape, torch.uint8)
        scales = Guarded((p.B, p.H, -(-N // blk)), torch.float32)
        qa.qattn_rotate_block_quant(x, layout, r, blk, code, codes.t, scales.t)
        torch.cuda.synchronize()
        assert qa.qattn_device_error() == qa.QATTN_OK
        codes.check("%s codes" % name)
        scales.check("%s scales" % name)


def _codes(p, d, qk, v):
    rot = dev(d["rot"])
    return [qa.qattn_rotate_block_quant(dev_bits(d[n], p.in_dtype), p.layout, r, blk, t)
            for n, blk, r, t in (("q", 128, rot, qk), ("k", 256, rot, qk), ("v", 256, None, v))]


@pytest.mark.parametrize("N", [1, 129, 300])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
@pytest.mark.parametrize("codes", ["int8_causal", "fp8", "int8_q_k_int4_v", "int4_qkv"])
def test_prefill(N, D, layout, codes):
    qk, v, causal = {"int8_causal": (synth.INT8, synth.INT8, True), "fp8": (synth.FP8_E4M3, synth.FP8_E4M3, False),
                     "int8_q_k_int4_v": (synth.INT8, synth.INT4_PACKED, True),
                     "int4_qkv": (synth.INT4_PACKED, synth.INT4_PACKED, False)}[codes]
    p = _problem(N, D, layout, qk, causal, 7100 + N + D + layout)
    d = synth.make_prefill(p)
    (qc, qs), (kc, ks), (vc, vs) = _codes(p, d, qk, v)
    out = Guarded(p.shape(), torch.bfloat16)
    lse = Guarded((p.B, p.H, N), torch.float32)
    qa.qattn_prefill_mixed(qc, qs, kc, ks, vc, vs, qk, v, layout, causal, out=out.t, lse=lse.t)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    out.check("output")
    lse.check("lse")


@pytest.mark.parametrize("L", [1, 63, 4097])
@pytest.mark.parametrize("kv_dtype", [synth.INT8, synth.INT4_PACKED])
def test_decode(L, kv_dtype):
    base = synth.INT8_KV_DECODE if kv_dtype == synth.INT8 else synth.INT4_KV_DECODE
    p = synth.scaled(base, B=3, L=L, seed=7200 + L + kv_dtype)
    dd = synth.make_decode(p)
    q = dev(dd["q"].view(np.int16)).view(torch.bfloat16)
    k, v = dev(dd["k"]), dev(dd["v"])
    if kv_dtype == synth.INT8:
        ks, vs = dev(dd["k_scales"]), dev(dd["v_scales"])
    else:
        ks = dev(dd["k_scales"].view(np.int16)).view(torch.float16)
        vs = dev(dd["v_scales"].view(np.int16)).view(torch.float16)
    need = qa.qattn_decode_workspace_size(p.B, p.Hq, p.Hkv, p.L, p.D)
    ws = Guarded((need,), torch.uint8)
    out = Guarded((p.B, p.Hq, 1, p.D), torch.bfloat16)
    qa.qattn_decode_kvq(q, k, v, ks, vs, kv_dtype, out=out.t, workspace=ws.t)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    out.check("output")
    ws.check("workspace")


@pytest.mark.parametrize("kv_dtype", [synth.INT8, synth.INT4_PACKED])
def test_kv_append_to_the_end_of_the_cache(kv_dtype):
    """Appends that end exactly at L_max (a ragged L_max: the last INT8
    block is partial). Beyond the guard bands, cache rows the append does not
    own keep their bytes: INT8 may rewrite earlier rows of the block it
    grows, nothing else; INT4 rows [L, L + n) only."""
    B, H, D, Lmax = 2, 3, 128, 300
    rng = np.random.default_rng(kv_dtype)
    if kv_dtype == synth.INT8:
        cache = Guarded((B, H, Lmax, D), torch.int8)
        scales = Guarded((B, H, -(-Lmax // 256)), torch.float32)
    else:
        cache = Guarded((B, H, Lmax, D // 2), torch.uint8)
        scales = Guarded((B, H, Lmax, 1), torch.float16)
    before = cache.t.view(torch.uint8).cpu().numpy().copy()
    L = 0
    for n in (100, 170, 30):                     # the last piece ends at L_max = 300
        x = dev(synth.f32_to_bf16_bits(rng.standard_normal((B, H, n, D))).view(np.int16)).view(torch.bfloat16)
        qa.qattn_kv_append(x, cache.t, scales.t, L, kv_dtype)
        torch.cuda.synchronize()
        assert qa.qattn_device_error() == qa.QATTN_OK
        after = cache.t.view(torch.uint8).cpu().numpy()
        first = (L // 256) * 256 if kv_dtype == synth.INT8 else L
        untouched = np.ones(Lmax, bool)
        untouched[first:L + n] = False
        assert np.array_equal(after[:, :, untouched], before[:, :, untouched]), "rows outside the append changed"
        before = after.copy()
        L += n
        cache.check("cache")
        scales.check("scales")


def test_path_host_output():
    """The host-buffer path writes its output by device-to-host copies into
    a pinned host buffer: nothing beyond the output."""
    p = _problem(300, 128, synth.BSND, synth.INT8, True, 7300)
    d = synth.make_prefill(p)
    host = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).pin_memory()
    out = Guarded(p.shape(), torch.bfloat16, device="cpu")
    qa.qattn_attention_path_host(host(d["q"]), host(d["k"]), host(d["v"]), dev(d["rot"]), p.layout, p.code_dtype,
                                 p.causal, out=out.t, groups=4)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    out.check("host output")


@pytest.mark.parametrize("N", [1, 129, 300])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
def test_dequant_path(N, D, layout):
    """The dequantize-first comparison path: the dequantize pass and the
    bf16 attention write nothing beyond their outputs."""
    p = _problem(N, D, layout, synth.INT8, True, 7400 + N + D + layout)
    d = synth.make_prefill(p)
    deq = []
    for (c, s), blk in zip(_codes(p, d, synth.INT8, synth.INT8), (128, 256, 256)):
        g = Guarded(p.shape(), torch.bfloat16)
        qa.qattn_dequant_bf16(c, s, synth.INT8, layout, blk, out=g.t)
        torch.cuda.synchronize()
        g.check("dequantized")
        deq.append(g.t)
    out = Guarded(p.shape(), torch.bfloat16)
    lse = Guarded((p.B, p.H, N), torch.float32)
    qa.qattn_attention_bf16(*deq, layout, True, out=out.t, lse=lse.t)
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    out.check("output")
    lse.check("lse")


@pytest.mark.parametrize("N", [1, 300])
@pytest.mark.parametrize("code", [synth.INT8, synth.INT4_PACKED])
def test_rotate_block_quant_qkv(N, code):
    """The three quantizations in one call, two of them on internal streams:
    six outputs, each inside its own guard bands."""
    p = _problem(N, 128, synth.BSND, synth.INT8, False, 7500 + N + code)
    d = synth.make_prefill(p)
    x = [dev_bits(d[n], p.in_dtype) for n in ("q", "k", "v")]
    shape = tuple(x[0].shape[:-1]) + ((64,) if code == synth.INT4_PACKED else (128,))
    outs = [(Guarded(shape, torch.uint8), Guarded((p.B, p.H, -(-N // blk)), torch.float32)) for blk in (128, 256, 256)]
    qa.qattn_rotate_block_quant_qkv(*x, p.layout, dev(d["rot"]), code, out=[(c.t, s.t) for c, s in outs])
    torch.cuda.synchronize()
    assert qa.qattn_device_error() == qa.QATTN_OK
    for name, (c, s) in zip("qkv", outs):
        c.check("%s codes" % name)
        s.check("%s scales" % name)


@pytest.mark.parametrize("n", [17, 4096 + 7, 300 * 64])
def test_widen_int4(n):
    """The INT4 -> INT8 widening pass writes its 2n bytes and nothing else
    (byte tail beyond the last 16-byte vector included)."""
    rng = np.random.default_rng(n)
    packed = torch.from_numpy(rng.integers(0, 256, n, dtype=np.uint8)).cuda()
    out = Guarded((2 * n,), torch.uint8)
    qa.qattn_widen_int4(packed, out=out.t)
    torch.cuda.synchronize()
    out.check("widened codes")
