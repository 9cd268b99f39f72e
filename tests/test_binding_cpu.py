"""The Python binding refuses, before any launch, tensors the kernels could
not address as dense device buffers: tensors in host memory and strided
views. CPU only (nothing reaches a kernel)."""
import pytest
import torch

import block_quantized_precision_b200 as qa


@pytest.fixture(scope="module", autouse=True)
def built():
    from block_quantized_precision_b200 import build
    build.build()
    qa.lib()


def test_host_tensors_are_refused():
    x = torch.zeros((1, 2, 128, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qa.qattn_rotate_block_quant(x, qa.QATTN_BNSD, None, 128, qa.QATTN_INT8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qa.qattn_widen_int4(torch.zeros((4, 64), dtype=torch.uint8), out=torch.zeros((4, 128), dtype=torch.uint8))
    c = torch.zeros((1, 2, 128, 128), dtype=torch.uint8)
    s = torch.zeros((1, 2, 1), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        qa.qattn_prefill(c, s, c, s, c, s, qa.QATTN_INT8, qa.QATTN_BNSD, True, out=torch.zeros(c.shape, dtype=torch.bfloat16))


def test_strided_views_are_refused():
    # a transposed view has the right shape but not the dense layout the kernels address
    x = torch.zeros((1, 128, 2, 128), dtype=torch.bfloat16).transpose(1, 2)
    assert not x.is_contiguous()
    with pytest.raises(ValueError):
        qa._dptr(x)
    assert qa._dptr(None) is None
