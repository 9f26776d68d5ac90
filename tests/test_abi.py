"""The C-ABI library: it builds for sm_100a, loads, exports every symbol include/adx.h
declares, and rejects bad arguments on the host before touching a GPU."""

import ctypes
import os
import re

import pytest

from sparse_attention_token_indexer_b200 import _lib as L
from sparse_attention_token_indexer_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return L.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "adx.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(adx_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert set(names) == set(L.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_constants(lib):
    assert lib.adx_abi_version() == 1
    assert lib.adx_bank_width(8192, 64, L.ADX_BANK_WINDOW) == 8192
    assert lib.adx_bank_width(8192, 64, L.ADX_BANK_PAPER) == 8192 + 63
    assert lib.adx_bank_width(64, 64, L.ADX_BANK_WINDOW) == 0
    for code in range(7):
        assert L.status_string(code)


def _ops(**kw):
    o = L.Operands()
    o.q_dtype, o.k_dtype = L.ADX_BF16, L.ADX_BF16
    o.q, o.w, o.k = 256, 512, 1024          # never dereferenced: validation fails first
    o.T, o.H, o.d, o.S = 4, 64, 128, 16
    for k, v in kw.items():
        setattr(o, k, v)
    return o


def _prefill(lib, o, K=4):
    return lib.adx_index_prefill(ctypes.byref(o), K, ctypes.c_void_p(4096), None, None, 0,
                                 ctypes.c_void_p(8192), 1 << 20, None)


def test_host_validation(lib):
    assert _prefill(lib, _ops(q=None)) == L.ADX_EINVAL
    assert _prefill(lib, _ops(T=0)) == L.ADX_EINVAL
    assert _prefill(lib, _ops(H=5)) == L.ADX_EUNSUPPORTED
    assert _prefill(lib, _ops(d=96)) == L.ADX_EUNSUPPORTED
    assert _prefill(lib, _ops(q_pos0=13)) == L.ADX_EINVAL           # q_pos0 + T > S
    assert _prefill(lib, _ops(), K=0) == L.ADX_EINVAL
    assert _prefill(lib, _ops(q_dtype=L.ADX_E4M3)) == L.ADX_EINVAL   # e4m3 without scale
    assert _prefill(lib, _ops(q_dtype=L.ADX_E4M3, q_scale=64, d=64, k_dtype=L.ADX_E4M3,
                              k_scale=64)) == L.ADX_EUNSUPPORTED    # e4m3 needs d = 128
    assert lib.adx_index_prefill(ctypes.byref(_ops()), 4, ctypes.c_void_p(4096), None, None,
                                 0, ctypes.c_void_p(8192), 16, None) == L.ADX_EWORKSPACE
    # decode layout needs seq_len; bank modes are checked
    assert lib.adx_index_decode(ctypes.byref(_ops()), 4, ctypes.c_void_p(4096), None,
                                ctypes.c_void_p(8192), 1 << 20, None) == L.ADX_EINVAL
    assert lib.adx_group_bank(ctypes.byref(_ops()), 4, 8, 7, ctypes.c_void_p(4096),
                              ctypes.c_void_p(8192), 1 << 20, None) == L.ADX_EINVAL


def test_workspace_size(lib):
    o = _ops(T=1024, S=1024)
    n = lib.adx_workspace_size(L.ADX_OP_PREFILL, ctypes.byref(o), 64, 0, 0, 0)
    assert n >= 1024 * 1024 * 4 + L.ADX_STATUS_BYTES
    assert lib.adx_workspace_size(L.ADX_OP_PREFILL, ctypes.byref(_ops(H=3)), 64, 0, 0, 0) == 0
