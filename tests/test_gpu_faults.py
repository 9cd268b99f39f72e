"""Failure reporting on the GPU, without faulting it: a kernel whose barrier
is never completed gives up after its bounded wait, records
QATTN_ERR_TIMEOUT and returns; the context stays usable."""
import pytest
import torch

import block_quantized_precision_b200 as qa

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    assert qa.qattn_device_error() == qa.QATTN_OK          # clean start
    qa.qattn_selftest_wait_timeout(50)
    assert qa.qattn_device_error() == qa.QATTN_ERR_TIMEOUT
    assert qa.qattn_device_error() == qa.QATTN_OK           # cleared by the read
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0                      # context still usable


def test_invalid_arguments_raise():
    x = torch.zeros((1, 1, 256, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qa.QAttnError) as e:
        qa.qattn_rotate_block_quant(x, qa.QATTN_BNSD, None, 128, qa.QATTN_INT8)
    assert e.value.status == qa.QATTN_ERR_UNSUPPORTED
    q = torch.zeros((1, 1, 256, 128), dtype=torch.uint8, device="cuda")
    s = torch.zeros((1, 1, 2), dtype=torch.float32, device="cuda")
    with pytest.raises(qa.QAttnError):
        qa.qattn_prefill(q, s, q, s, q, s, qa.QATTN_INT8, qa.QATTN_BNSD, True, kv_block=128)


def test_short_workspace_is_rejected():
    q = torch.zeros((2, 32, 1, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((2, 8, 512, 128), dtype=torch.int8, device="cuda")
    s = torch.ones((2, 8, 2), dtype=torch.float32, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(qa.QAttnError) as e:
        qa.qattn_decode_kvq(q, k, k, s, s, qa.QATTN_INT8, workspace=ws)
    assert e.value.status == qa.QATTN_ERR_WORKSPACE
