"""The seeded input generators (synth/): the counter-style SplitMix64 against
the sequential form of the published generator, independence of the values
from the chunking, the distributions the workloads ask for, and the storage
rounding against torch. CPU only."""
import numpy as np
import pytest
import torch

import synth

MASK = (1 << 64) - 1


def _splitmix64_sequential(state: int, n: int):
    """The published SplitMix64 step (Steele, Lea, Flood, OOPSLA 2014) as a
    sequential generator: add the golden gamma to the state, then mix."""
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        out.append(z ^ (z >> 31))
    return out


def _mix(z: int) -> int:
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
    return z ^ (z >> 31)


@pytest.mark.parametrize("seed,stream", [(0, 0), (1, 2), (7, 1001), (123456, 5)])
def test_counter_form_equals_the_sequential_generator(seed, stream):
    base = _mix(((seed << 32) + stream) & MASK)
    want = _splitmix64_sequential(base, 40)
    got = synth.raw_u64(seed, stream, 40).tolist()
    assert got == want
    # any counter offset continues the same sequence
    assert synth.raw_u64(seed, stream, 10, start=30).tolist() == want[30:]


def test_values_do_not_depend_on_the_chunking():
    """Element i is a function of (seed, stream, i) alone, also across the
    chunk boundary of the threaded fill."""
    n = (1 << 22) + 1000
    u = synth.uniform01(3, 7, n)
    g = synth.normal(3, 7, n)
    b = synth.random_bytes(3, 9, n)
    c = synth.int8_uniform(3, 11, n)
    for i in (0, 1, (1 << 22) - 1, 1 << 22, n - 1):
        assert u[i] == synth.uniform01(3, 7, i + 1)[i]
        assert g[i] == synth.normal(3, 7, i + 1)[i]
        assert b[i] == synth.random_bytes(3, 9, i + 1)[i]
        assert c[i] == synth.int8_uniform(3, 11, i + 1)[i]
    assert np.array_equal(synth.normal(3, 7, 1000), g[:1000])


def test_distributions():
    n = 1 << 20
    u = synth.uniform01(5, 1, n)
    assert u.min() > 0.0 and u.max() < 1.0 and abs(u.mean() - 0.5) < 5 / np.sqrt(12 * n)
    g = synth.normal(5, 1, n)
    assert abs(g.mean()) < 5 / np.sqrt(n) and abs(g.var() - 1.0) < 5 * np.sqrt(2.0 / n)
    c = synth.int8_uniform(5, 2, n)
    assert c.min() == -127 and c.max() == 127
    counts = np.bincount(c.astype(np.int64) + 127, minlength=255)
    assert np.all(np.abs(counts - n / 255) < 6 * np.sqrt(n / 255))
    b = synth.random_bytes(5, 3, n)
    counts = np.bincount(b, minlength=256)
    assert np.all(np.abs(counts - n / 256) < 6 * np.sqrt(n / 256))
    # different streams and seeds give different values
    assert not np.array_equal(synth.normal(5, 1, 64), synth.normal(5, 2, 64))
    assert not np.array_equal(synth.normal(5, 1, 64), synth.normal(6, 1, 64))


def test_storage_rounding_matches_torch():
    x = np.concatenate([synth.normal(8, 1, 1 << 16) * 10.0 ** synth.uniform01(8, 2, 1 << 16) * 3,
                        [0.0, -0.0, 1.0, -2.5, 65504.0, 1e-8, 3.0e38]])
    x32 = torch.from_numpy(x.astype(np.float32))
    assert np.array_equal(synth.f32_to_bf16_bits(x), x32.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    small = x[np.abs(x) < 60000]
    assert np.array_equal(synth.f64_to_f16_bits(small),
                          torch.from_numpy(small.astype(np.float32)).to(torch.float16).view(torch.int16).numpy()
                          .view(np.uint16))
    bits = synth.f32_to_bf16_bits(x)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), x32.to(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("layout", [synth.BNSD, synth.BSND])
def test_prefill_workload_recipe(layout):
    p = synth.PrefillProblem("recipe", 2, 8, 96, 64, synth.BF16, synth.INT8, layout, causal=True, rotate=True,
                             seed=21, outlier_frac=0.05)
    d = synth.make_prefill(p)
    for n in ("q", "k", "v"):
        assert d[n].shape == tuple(p.shape()) and d[n].dtype == np.uint16
    assert d["rot"].shape == (p.D, p.D) and d["rot"].dtype == np.float32
    oc = d["outlier_channels"]
    assert len(oc) == int(round(p.outlier_frac * p.H * p.D)) and len(set(oc.tolist())) == len(oc)
    # the outlier channels carry the larger magnitudes
    x = synth.bf16_bits_to_f32(d["k"]).astype(np.float64)
    per = np.abs(x).mean(axis=(0, 2)) if layout == synth.BNSD else np.abs(x).mean(axis=(0, 1))
    per = per.reshape(-1)
    mask = np.zeros(p.H * p.D, bool)
    mask[oc] = True
    assert per[mask].min() > 2 * per[~mask].max()
    again = synth.make_prefill(p)
    assert all(np.array_equal(d[n], again[n]) for n in ("q", "k", "v", "rot"))
