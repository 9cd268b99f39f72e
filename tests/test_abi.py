"""The C-ABI library builds, loads and exports every entry point declared in
include/qattn.h; argument validation answers without launching anything.

CPU only (no kernel is launched by these calls).
"""
import os
import re
import subprocess

import pytest

import block_quantized_precision_b200 as qa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qattn.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qattn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from block_quantized_precision_b200 import build
    build.build()
    return qa.lib()


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert set(declared) == set(qa.EXPORTED)
    out = subprocess.check_output(["nm", "-D", "--defined-only", qa.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (qattn_[a-z0-9_]+)", out))
    assert set(declared) <= exported
    for name in declared:
        assert hasattr(L, name)


def test_version_and_status_strings(L):
    assert qa.qattn_abi_version() == 1
    for code in range(7):
        assert qa.status_string(code) and qa.status_string(code) != "unknown status"
    assert qa.status_string(99) == "unknown status"


def test_rotate_block_quant_validation(L):
    f = L.qattn_rotate_block_quant
    bad = 0x1000
    # negative size, bad dtypes, bad layout
    assert f(bad, qa.QATTN_BF16, 0, -1, 1, 1, 128, None, 128, qa.QATTN_INT8, bad, bad, None) == qa.QATTN_ERR_INVALID_ARG
    assert f(bad, qa.QATTN_INT8, 0, 1, 1, 1, 128, None, 128, qa.QATTN_INT8, bad, bad, None) == qa.QATTN_ERR_INVALID_ARG
    assert f(bad, qa.QATTN_BF16, 0, 1, 1, 1, 128, None, 128, qa.QATTN_BF16, bad, bad, None) == qa.QATTN_ERR_INVALID_ARG
    assert f(bad, qa.QATTN_BF16, 7, 1, 1, 1, 128, None, 128, qa.QATTN_INT8, bad, bad, None) == qa.QATTN_ERR_INVALID_ARG
    # unsupported head size / block size
    assert f(bad, qa.QATTN_BF16, 0, 1, 1, 1, 96, None, 128, qa.QATTN_INT8, bad, bad, None) == qa.QATTN_ERR_UNSUPPORTED
    assert f(bad, qa.QATTN_BF16, 0, 1, 1, 1, 128, None, 100, qa.QATTN_INT8, bad, bad, None) == qa.QATTN_ERR_UNSUPPORTED
    # empty problem: nothing to do
    assert f(None, qa.QATTN_BF16, 0, 0, 4, 128, 128, None, 128, qa.QATTN_INT8, None, None, None) == qa.QATTN_OK
    # null pointers / misalignment
    assert f(None, qa.QATTN_BF16, 0, 1, 1, 8, 128, None, 128, qa.QATTN_INT8, bad, bad, None) == qa.QATTN_ERR_INVALID_ARG
    assert f(bad + 8, qa.QATTN_BF16, 0, 1, 1, 8, 128, None, 128, qa.QATTN_INT8, bad, bad, None) == qa.QATTN_ERR_ALIGNMENT


def test_prefill_validation(L):
    f = L.qattn_prefill
    p = 0x1000
    args = dict(B=1, H=1, Nq=256, Nkv=256, D=128, qb=128, kb=256, causal=0)

    def call(**kw):
        a = dict(args, **kw)
        return f(p, p, p, p, p, p, kw.get("code", qa.QATTN_INT8), kw.get("layout", 0), a["B"], a["H"], a["Nq"],
                 a["Nkv"], a["D"], a["qb"], a["kb"], a["causal"], 0.0, kw.get("out", p), None, None)
    assert call(code=qa.QATTN_BF16) == qa.QATTN_ERR_INVALID_ARG
    assert call(causal=2) == qa.QATTN_ERR_INVALID_ARG
    assert call(causal=1, Nkv=512) == qa.QATTN_ERR_UNSUPPORTED
    assert call(qb=64) == qa.QATTN_ERR_UNSUPPORTED
    assert call(kb=128) == qa.QATTN_ERR_UNSUPPORTED
    assert call(D=96) == qa.QATTN_ERR_UNSUPPORTED
    assert call(Nq=0) == qa.QATTN_OK
    assert call(Nkv=0) == qa.QATTN_ERR_UNSUPPORTED
    assert call(out=None) == qa.QATTN_ERR_INVALID_ARG
    assert call(out=p + 2) == qa.QATTN_ERR_ALIGNMENT
    assert call(B=-1) == qa.QATTN_ERR_INVALID_ARG


def test_decode_validation(L):
    f = L.qattn_decode_kvq
    p = 0x1000

    def call(kv=qa.QATTN_INT8, B=1, Hq=32, Hkv=8, Lk=256, D=128, kvb=256, grp=128, ws=p):
        return f(p, p, p, p, p, kv, B, Hq, Hkv, Lk, D, kvb, grp, 0.0, p, ws, 1 << 30, None)
    assert call(Hq=30) == qa.QATTN_ERR_INVALID_ARG
    assert call(kv=qa.QATTN_FP8_E4M3) == qa.QATTN_ERR_INVALID_ARG
    assert call(Hq=48, Hkv=3) == qa.QATTN_ERR_UNSUPPORTED     # 16 query heads per kv head
    assert call(kvb=128) == qa.QATTN_ERR_UNSUPPORTED
    assert call(kv=qa.QATTN_INT4_PACKED, grp=96) == qa.QATTN_ERR_INVALID_ARG
    assert call(kv=qa.QATTN_INT4_PACKED, grp=32) == qa.QATTN_ERR_UNSUPPORTED
    assert call(D=64) == qa.QATTN_ERR_UNSUPPORTED
    assert call(B=0) == qa.QATTN_OK
    assert call(ws=None) == qa.QATTN_ERR_INVALID_ARG
    assert call(ws=p + 4) == qa.QATTN_ERR_ALIGNMENT


def test_selftest_rejects_out_of_range_limits(L):
    assert L.qattn_selftest_wait_timeout(0, None) == qa.QATTN_ERR_INVALID_ARG
    assert L.qattn_selftest_wait_timeout(5000, None) == qa.QATTN_ERR_INVALID_ARG


def test_oracle_and_library_share_no_code():
    """The oracle is plain C compiled by gcc; the library is CUDA. Neither
    includes or imports the other."""
    ora = open(os.path.join(ROOT, "oracle", "qattn_oracle.c")).read()
    assert "qattn.h" not in ora and "csrc" not in ora
    for f in os.listdir(os.path.join(ROOT, "block_quantized_precision_b200", "csrc")):
        src = open(os.path.join(ROOT, "block_quantized_precision_b200", "csrc", f)).read()
        assert "oracle" not in src.lower().replace("oracle-only", "")
    pkg = open(os.path.join(ROOT, "block_quantized_precision_b200", "__init__.py")).read()
    assert "import oracle" not in pkg and "from oracle" not in pkg


def test_kv_append_validation(L):
    f = L.qattn_kv_append
    p = 0x1000

    def call(B=2, H=8, n=1, D=128, kv=qa.QATTN_INT8, Lk=10, Lmax=256, kvb=256, grp=128, x=p, c=p, s=p):
        return f(x, B, H, n, D, kv, Lk, Lmax, c, s, kvb, grp, None)
    assert call(Lk=256) == qa.QATTN_ERR_INVALID_ARG              # L + n > L_max
    assert call(Lk=-1) == qa.QATTN_ERR_INVALID_ARG
    assert call(kv=qa.QATTN_FP8_E4M3) == qa.QATTN_ERR_INVALID_ARG
    assert call(kvb=128) == qa.QATTN_ERR_UNSUPPORTED
    assert call(D=12) == qa.QATTN_ERR_UNSUPPORTED
    assert call(kv=qa.QATTN_INT4_PACKED, grp=96) == qa.QATTN_ERR_INVALID_ARG
    assert call(kv=qa.QATTN_INT4_PACKED, grp=32) == qa.QATTN_ERR_UNSUPPORTED
    assert call(kv=qa.QATTN_INT4_PACKED, D=64, grp=64) == qa.QATTN_ERR_UNSUPPORTED
    assert call(n=0) == qa.QATTN_OK
    assert call(c=None) == qa.QATTN_ERR_INVALID_ARG
    assert call(x=p + 2) == qa.QATTN_ERR_ALIGNMENT


def test_dequant_path_validation(L):
    bad = 0x1000
    d = L.qattn_dequant_bf16
    assert d(bad, bad, qa.QATTN_BF16, 0, 1, 1, 128, 128, 128, bad, None) == qa.QATTN_ERR_INVALID_ARG
    assert d(bad, bad, qa.QATTN_INT8, 3, 1, 1, 128, 128, 128, bad, None) == qa.QATTN_ERR_INVALID_ARG
    assert d(bad, bad, qa.QATTN_INT8, 0, 1, 1, 128, 120, 128, bad, None) == qa.QATTN_ERR_UNSUPPORTED
    assert d(bad + 8, bad, qa.QATTN_INT8, 0, 1, 1, 128, 128, 128, bad, None) == qa.QATTN_ERR_ALIGNMENT
    assert d(None, None, qa.QATTN_INT8, 0, 0, 1, 128, 128, 128, None, None) == qa.QATTN_OK
    a = L.qattn_attention_bf16
    assert a(bad, bad, bad, 0, 1, 1, 128, 128, 96, 0, 0.0, bad, None, None) == qa.QATTN_ERR_UNSUPPORTED
    assert a(bad, bad, bad, 0, 1, 1, 128, 200, 128, 1, 0.0, bad, None, None) == qa.QATTN_ERR_UNSUPPORTED
    assert a(bad, bad, bad, 0, 1, 1, 128, 128, 128, 2, 0.0, bad, None, None) == qa.QATTN_ERR_INVALID_ARG
    assert a(bad, bad, bad, 0, 1, 1, 128, 0, 128, 0, 0.0, bad, None, None) == qa.QATTN_ERR_UNSUPPORTED
    assert a(bad, bad + 8, bad, 0, 1, 1, 128, 128, 128, 0, 0.0, bad, None, None) == qa.QATTN_ERR_ALIGNMENT


def test_rotate_block_quant_qkv_validation(L):
    bad = 0x1000
    f = L.qattn_rotate_block_quant_qkv
    args = lambda **kw: [kw.get("q", bad), bad, bad, kw.get("x", qa.QATTN_BF16), 0, kw.get("B", 1), 1, 128, kw.get("D", 128),
                         None, kw.get("code", qa.QATTN_INT8), bad, bad, bad, bad, kw.get("vc", bad), bad, None]
    assert f(*args(B=-1)) == qa.QATTN_ERR_INVALID_ARG
    assert f(*args(x=qa.QATTN_INT8)) == qa.QATTN_ERR_INVALID_ARG
    assert f(*args(code=qa.QATTN_BF16)) == qa.QATTN_ERR_INVALID_ARG
    assert f(*args(D=96)) == qa.QATTN_ERR_UNSUPPORTED
    assert f(*args(q=bad + 8)) == qa.QATTN_ERR_ALIGNMENT
    assert f(*args(vc=None)) == qa.QATTN_ERR_INVALID_ARG          # V codes missing
    assert f(*args(B=0)) == qa.QATTN_OK                            # empty problem


def test_widen_int4_validation(L):
    bad = 0x1000
    w = L.qattn_widen_int4
    assert w(bad, -1, bad + 4096, None) == qa.QATTN_ERR_INVALID_ARG
    assert w(None, 0, None, None) == qa.QATTN_OK                      # nothing to widen
    assert w(None, 16, bad, None) == qa.QATTN_ERR_INVALID_ARG
    assert w(bad, 16, None, None) == qa.QATTN_ERR_INVALID_ARG
    assert w(bad + 8, 16, bad + 4096, None) == qa.QATTN_ERR_ALIGNMENT
    assert w(bad, 16, bad + 4104, None) == qa.QATTN_ERR_ALIGNMENT
    assert w(bad, 64, bad + 48, None) == qa.QATTN_ERR_INVALID_ARG    # out overlaps the input's tail
    assert w(bad + 64, 64, bad, None) == qa.QATTN_ERR_INVALID_ARG    # input inside the output
