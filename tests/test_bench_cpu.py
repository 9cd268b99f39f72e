"""The benchmark's roofline arithmetic and clock summary, checked on the CPU:
the operation count of a prefill against a brute-force count of the
(query, key) pairs it computes, the bytes of a decode step against the
arrays the step reads and writes, and the throttle reasons and load clock
taken from nvidia-smi samples (a recorded sample file, no GPU)."""
import itertools
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 7, 64])
def test_prefill_ops_counts_every_unmasked_pair(causal, N):
    """4 D operations (a multiply-add in Q K^T and one in P V, per channel)
    per (query, key) pair that the mask keeps."""
    B, H, D = 2, 3, 64
    pairs = sum(1 for i, j in itertools.product(range(N), range(N)) if not causal or j <= i)
    assert bench.prefill_ops(B, H, N, D, causal) == 4 * D * B * H * pairs


@pytest.mark.parametrize("kv_dtype,group", [(synth.INT8, 128), (synth.INT4_PACKED, 128), (synth.INT4_PACKED, 64)])
def test_decode_bytes_are_the_arrays_of_one_step(kv_dtype, group):
    """K and V codes and scales, the bf16 query and the bf16 output."""
    p = synth.DecodeProblem("small", 2, 8, 2, 300, 128, kv_dtype, seed=9, group=group)
    d = synth.make_decode(p)
    read = sum(d[n].nbytes for n in ("k", "v", "k_scales", "v_scales", "q"))
    written = p.B * p.Hq * p.D * 2
    assert bench.decode_bytes(p) == read + written


def _summary(tmp_path, lines, max_fallback=1965.0):
    c = bench.ClockSampler(None)
    c.path = str(tmp_path / "clocks.csv")
    with open(c.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    return c.summary(max_fallback)


def test_clock_summary_median_under_load_and_reasons(tmp_path):
    idle = "1965, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    busy = ["%d, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active" % mhz for mhz in (1800, 1850, 1900)]
    s = _summary(tmp_path, [idle] + busy)
    assert s["sm_mhz"] == 1850 and s["sm_max_mhz"] == 1965 and s["samples"] == 4
    assert s["reasons"] == ["sw_power_cap"]
    hot = "1500, 1965, 950.0, 0x48, Not Active, Active, Not Active, Active"
    s = _summary(tmp_path, busy + [hot])
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_clock_summary_without_samples(tmp_path):
    s = _summary(tmp_path, ["garbage"])
    assert s["samples"] == 0 and s["reasons"] == ["unsampled"] and s["sm_max_mhz"] == 1965.0
