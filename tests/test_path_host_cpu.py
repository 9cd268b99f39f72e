"""Host logic of qattn_attention_path_host that needs no GPU: the workspace
size of the head-group plan, and the argument checks that answer before any
CUDA call is made.

CPU only."""
import ctypes as C

import pytest

import block_quantized_precision_b200 as qa


@pytest.fixture(scope="module")
def L():
    from block_quantized_precision_b200 import build
    build.build()
    return qa.lib()


def _slot_min(heads, N, D):
    # x q/k/v (2 bytes), codes q/k/v (1 byte), out (2 bytes); scales are extra
    return heads * N * D * (3 * 2 + 3 + 2)


@pytest.mark.parametrize("B,H,N,D,layout,groups,heads", [
    (1, 32, 4096, 128, qa.QATTN_BNSD, 8, 4),      # 32 heads in 8 groups of 4
    (2, 5, 700, 128, qa.QATTN_BNSD, 3, 4),        # 10 heads in groups of ceil(10 / 3) = 4
    (2, 6, 300, 64, qa.QATTN_BSND, 1, 12),        # one group: both b's, all heads
    (2, 6, 300, 64, qa.QATTN_BSND, 5, 2),         # 3 head ranges of 2 per b
    (3, 4, 129, 128, qa.QATTN_BSND, 2, 8),        # whole b's: 2 per group
    (1, 32, 4096, 128, qa.QATTN_BNSD, 0, 4),      # default: 8 groups
])
def test_workspace_size_follows_the_group_plan(L, B, H, N, D, layout, groups, heads):
    got = qa.qattn_attention_path_host_workspace_size(B, H, N, D, layout, groups)
    lo = 2 * _slot_min(heads, N, D)
    # scales: float32 per (head, block) for Q (128) and K, V (256), and 256-byte alignment of 10 buffers
    hi = lo + 2 * (4 * heads * (-(-N // 128) + 2 * -(-N // 256)) + 10 * 256)
    assert lo <= got <= hi


def test_workspace_size_of_invalid_shapes_is_zero(L):
    assert qa.qattn_attention_path_host_workspace_size(0, 4, 128, 128, qa.QATTN_BNSD, 0) == 0
    assert qa.qattn_attention_path_host_workspace_size(1, 4, 128, 128, 7, 0) == 0


def test_fewer_groups_need_more_workspace(L):
    sizes = [qa.qattn_attention_path_host_workspace_size(1, 32, 1024, 128, qa.QATTN_BNSD, g) for g in (1, 2, 4, 8)]
    assert sizes == sorted(sizes, reverse=True)


def _call(L, **kw):
    buf = C.create_string_buffer(64)
    a = dict(q=buf, k=buf, v=buf, x_dtype=qa.QATTN_BF16, layout=qa.QATTN_BNSD, B=1, H=2, N=128, D=128, rot=None,
             code=qa.QATTN_INT8, causal=1, scale=0.0, out=buf, groups=0, ws=None, ws_bytes=0)
    a.update(kw)
    return L.qattn_attention_path_host(C.addressof(a["q"]) if a["q"] is not None else None,
                                       C.addressof(a["k"]), C.addressof(a["v"]), a["x_dtype"], a["layout"],
                                       a["B"], a["H"], a["N"], a["D"], a["rot"], a["code"], a["causal"],
                                       a["scale"], C.addressof(a["out"]), a["groups"], a["ws"], a["ws_bytes"], None)


def test_argument_checks_answer_before_any_cuda_call(L):
    assert _call(L, x_dtype=qa.QATTN_INT8) == qa.QATTN_ERR_INVALID_ARG
    assert _call(L, code=qa.QATTN_INT4_PACKED) == qa.QATTN_ERR_INVALID_ARG
    assert _call(L, layout=5) == qa.QATTN_ERR_INVALID_ARG
    assert _call(L, causal=2) == qa.QATTN_ERR_INVALID_ARG
    assert _call(L, groups=-1) == qa.QATTN_ERR_INVALID_ARG
    assert _call(L, D=96) == qa.QATTN_ERR_UNSUPPORTED
    assert _call(L, q=None) == qa.QATTN_ERR_INVALID_ARG
    assert _call(L, ws=None) == qa.QATTN_ERR_WORKSPACE
    assert _call(L, N=0) == qa.QATTN_OK                 # empty problem: nothing to do
