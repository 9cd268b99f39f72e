"""Pins for the oracle's number formats, against library routines, the OCP
FP8 specification and the packing formula printed on the pages.

CPU only.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def torch_e4m3_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_all_codes_match_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok].view(np.uint32), ref[ok].view(np.uint32))  # -0 included


def _e4m3_probe_values(rng):
    """Dense sample of float32 inputs: every binade from 2^-24 to 2^8 with
    random mantissas, every e4m3 value, every midpoint between adjacent e4m3
    values and the float32 neighbours of those midpoints, both signs."""
    vals = []
    for e in range(-24, 9):
        mant = rng.integers(0, 1 << 23, 4096, dtype=np.uint32)
        bits = ((e + 127) << 23) | mant
        vals.append(bits.astype(np.uint32).view(np.float32))
    grid = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    grid = np.unique(grid)
    mids = (grid[:-1].astype(np.float64) + grid[1:]) / 2
    mids = mids.astype(np.float32)
    vals += [grid, mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))]
    v = np.concatenate(vals).astype(np.float32)
    v = v[np.abs(v) < 464.0]     # beyond 464 torch's cast is non-saturating (NaN)
    return np.concatenate([v, -v])


def test_e4m3_encode_matches_torch_rne(orc):
    rng = np.random.default_rng(0)
    x = _e4m3_probe_values(rng)
    ours = orc.e4m3_encode(x)
    ref = torch_e4m3_bits(x)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(x[i]), hex(ours[i]), hex(ref[i])) for i in bad[:10]]


def test_e4m3_saturates_and_keeps_nan(orc):
    x = np.array([448.0, 449.0, 464.0, 465.0, 1e4, 3.0e38, np.inf, -470.0, -np.inf, np.nan, -np.nan],
                 dtype=np.float32)
    c = orc.e4m3_encode(x)
    assert list(c[:7]) == [0x7E] * 7
    assert list(c[7:9]) == [0xFE, 0xFE]
    assert c[9] & 0x7F == 0x7F and c[10] & 0x7F == 0x7F


def test_e4m3_spec_values(orc):
    for v, code in _read_golden("e4m3_spec.txt"):
        x = np.array([float(v)], dtype=np.float32)
        assert int(orc.e4m3_encode(x)[0]) == int(code, 16), v
        back = orc.e4m3_decode(np.array([int(code, 16)], dtype=np.uint8))[0]
        assert back == np.float32(v) and np.signbit(back) == np.signbit(np.float32(v))


def test_f16_decode_all_patterns(orc):
    L = orc.lib()
    pats = np.arange(1 << 16, dtype=np.uint32)
    ours = np.array([L.orc_f16_to_f32(int(p)) for p in pats[::7]], dtype=np.float32)
    ref = pats[::7].astype(np.uint16).view(np.float16).astype(np.float32)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok].view(np.uint32), ref[ok].view(np.uint32))


def _bf16_nearest_even(x: float) -> int:
    """bfloat16 bits nearest to x (ties to even), by exact rational search."""
    fx = Fraction(x)
    f32 = np.float32(x)
    cand = set()
    b = int(np.array([f32], dtype=np.float32).view(np.uint32)[0]) >> 16
    for d in range(-2, 3):
        cand.add((b + d) & 0xFFFF)
    best = None
    for c in cand:
        v = np.array([c << 16], dtype=np.uint32).view(np.float32)[0]
        if not np.isfinite(v):
            continue
        err = abs(Fraction(float(v)) - fx)
        key = (err, c & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return best[1]


def test_f64_to_bf16_rounds_from_the_exact_value(orc):
    L = orc.lib()
    rng = np.random.default_rng(1)
    xs = list(rng.standard_normal(3000) * np.exp(rng.uniform(-20, 20, 3000)))
    # exact ties and near-ties between bfloat16 neighbours
    for _ in range(300):
        b = int(rng.integers(0x3000, 0x5000))
        lo = np.array([b << 16], dtype=np.uint32).view(np.float32)[0]
        hi = np.array([(b + 1) << 16], dtype=np.uint32).view(np.float32)[0]
        mid = (float(lo) + float(hi)) / 2
        xs += [mid, np.nextafter(mid, 0.0), np.nextafter(mid, 1e300)]
    for x in xs:
        assert L.orc_f64_to_bf16(float(x)) == _bf16_nearest_even(float(x)), x


def test_int4_pack_golden_and_roundtrip(orc):
    for w0, w1, packed in _read_golden("int4_pack.txt"):
        assert orc.int4_pack(int(w0), int(w1)) == int(packed, 16)
        assert orc.int4_unpack(int(packed, 16)) == (int(w0), int(w1))
    for w0 in range(-8, 8):
        for w1 in range(-8, 8):
            assert orc.int4_unpack(orc.int4_pack(w0, w1)) == (w0, w1)
    for byte in range(256):
        assert orc.int4_pack(*orc.int4_unpack(byte)) == byte


def test_int4_storage_closed_form():
    """Packed INT4 with one fp16 scale per G elements costs 0.5 + 2/G bytes
    per element (page 3, section 5.1); for the long-context decode cache
    (D = 128, G = 128) that is 66 bytes per token, head and tensor."""
    (G, per_elem, frac), = _read_golden("int4_storage.txt")
    G = int(G)
    D = 128
    bytes_per_token = D // 2 + 2 * (D // G)
    assert bytes_per_token == 66
    assert bytes_per_token / D == pytest.approx(float(per_elem))
    assert (bytes_per_token / D) / 2.0 == pytest.approx(float(frac))
    assert abs(float(frac) - 0.26) < 0.005      # "about 26% of fp16"
