"""GPU widening of packed INT4 codes to INT8 codes, against the oracle's
nibble decoder, byte for byte.

Packing: "ops-transformer INT8/INT4 量化推理", 5.2 (two signed 4-bit codes
per byte, element 2i in the low nibble); widening to INT8 before the integer
matmul: "FlashAttention 的 INT8/INT4 量化", 第二层. The expected bytes come
from the oracle's int4_unpack of each packed byte value.
"""
import numpy as np
import pytest
import torch

import block_quantized_precision_b200 as qa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def table(orc):
    """byte value -> its two INT8 codes (low nibble first) as uint8."""
    t = np.empty((256, 2), dtype=np.uint8)
    for b in range(256):
        lo, hi = orc.int4_unpack(b)
        t[b] = (lo & 0xFF, hi & 0xFF)
    return t


def _widen_check(packed_np, table):
    packed = torch.from_numpy(packed_np).cuda()
    out = qa.qattn_widen_int4(packed)
    torch.cuda.synchronize()
    assert out.shape == packed_np.shape[:-1] + (2 * packed_np.shape[-1],)
    assert np.array_equal(out.cpu().numpy().reshape(-1), table[packed_np.reshape(-1)].reshape(-1))


def test_every_byte_value(table):
    _widen_check(np.tile(np.arange(256, dtype=np.uint8), 37), table)


@pytest.mark.parametrize("n", [1, 15, 16, 17, 31, 33, 1000, 4096 + 7, (1 << 20) + 9])
def test_sizes_and_tails(table, n):
    """Byte counts with and without a tail beyond the last 16-byte vector,
    below and above one vector per thread of the grid."""
    rng = np.random.default_rng(n)
    _widen_check(rng.integers(0, 256, n, dtype=np.uint8), table)


def test_code_tensor_of_the_int8_causal_problem(table):
    """A packed [1, 32, 4096, 64] code tensor (Q of B1 H32 N4096 D128 in
    packed INT4): the size the INT4 prefill widens."""
    rng = np.random.default_rng(7)
    _widen_check(rng.integers(0, 256, (1, 32, 4096, 64), dtype=np.uint8), table)


def test_empty_and_rejected_calls():
    L = qa.lib()
    a = torch.zeros(64, dtype=torch.uint8, device="cuda")
    b = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert L.qattn_widen_int4(a.data_ptr(), 0, b.data_ptr(), None) == qa.QATTN_OK
    assert L.qattn_widen_int4(a.data_ptr() + 1, 16, b.data_ptr(), None) == qa.QATTN_ERR_ALIGNMENT
    # out overlapping the packed input
    assert L.qattn_widen_int4(b.data_ptr() + 32, 32, b.data_ptr(), None) == qa.QATTN_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert np.all(b.cpu().numpy() == 0)
