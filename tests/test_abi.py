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
    # an external score matrix needs 16-byte rows: stride >= S rounded up to 128, a multiple
    # of 4, and an aligned base
    for ptr, ld in ((1 << 16, 64), (1 << 16, 129), (1 << 16 | 8, 128)):
        assert lib.adx_index_prefill(ctypes.byref(_ops()), 4, ctypes.c_void_p(4096), None,
                                     ctypes.c_void_p(ptr), ld, ctypes.c_void_p(8192), 1 << 20,
                                     None) == L.ADX_EINVAL
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


def _hisa(lib, o, n_blocks=64, K=2048, kbar=2048, kbar_scale=None, ws_bytes=1 << 40):
    return lib.adx_index_hisa(ctypes.byref(o), ctypes.c_void_p(kbar) if kbar else None,
                              ctypes.c_void_p(kbar_scale) if kbar_scale else None, n_blocks, K,
                              ctypes.c_void_p(4096), None, None, ctypes.c_void_p(8192), ws_bytes,
                              None)


def test_hisa_host_validation(lib):
    o = _ops(T=4, S=16)
    assert _hisa(lib, o, n_blocks=1) == L.ADX_EINVAL                 # fewer than two blocks
    assert _hisa(lib, o, n_blocks=256) == L.ADX_EINVAL               # slot bytes hold < 255
    assert _hisa(lib, o, n_blocks=4, K=4 * 128 + 1) == L.ADX_EINVAL  # K beyond the candidates
    assert _hisa(lib, o, kbar=0) == L.ADX_EINVAL
    assert _hisa(lib, _ops(H=16)) == L.ADX_EUNSUPPORTED               # 64 heads only
    assert _hisa(lib, o, ws_bytes=16) == L.ADX_EWORKSPACE
    assert lib.adx_hisa_workspace_size(ctypes.byref(o), 1, 64, 0) == 0
    assert lib.adx_hisa_workspace_size(ctypes.byref(o), 64, 2048, 0) > \
        lib.adx_hisa_workspace_size(ctypes.byref(o), 64, 2048, 1)     # blocks_out given
    assert lib.adx_hisa_block_keys(ctypes.byref(o), 0, None, None, None) == L.ADX_EINVAL
    assert lib.adx_hisa_block_keys(ctypes.byref(_ops(T=0)), 0, ctypes.c_void_p(64), None,
                                   None) == L.ADX_EINVAL


def _gi(**kw):
    g = L.GroupIndexer()
    g.cq, g.h, g.w_pool, g.w_q, g.w_g = 256, 512, 1024, 2048, 4096   # 16-byte aligned
    g.T, g.d_c, g.d_h, g.H_S, g.d, g.rope_dim = 256, 64, 128, 16, 128, 64
    g.rope_base, g.q_pos0 = 10000.0, 0
    for k, v in kw.items():
        setattr(g, k, v)
    return g


def test_group_indexer_host_validation(lib):
    size = lib.adx_group_indexer_workspace_size
    assert size(ctypes.byref(_gi()), 64) > 0
    for bad in (dict(d_c=60), dict(d_h=100), dict(H_S=65), dict(rope_dim=63),
                dict(rope_dim=130), dict(cq=258), dict(w_g=None), dict(rope_base=0.0),
                dict(T=32)):
        assert size(ctypes.byref(_gi(**bad)), 64) == 0, bad
    assert size(ctypes.byref(_gi()), 0) == 0
    g = _gi()
    assert lib.adx_group_indexer_queries(ctypes.byref(g), 64, ctypes.c_void_p(64),
                                         ctypes.c_void_p(128), ctypes.c_void_p(8192), 16,
                                         None) == L.ADX_EWORKSPACE
    assert lib.adx_group_indexer_queries(ctypes.byref(_gi(d_c=60)), 64, ctypes.c_void_p(64),
                                         ctypes.c_void_p(128), ctypes.c_void_p(8192), 1 << 40,
                                         None) == L.ADX_EINVAL


def test_group_helpers_host_validation(lib):
    # union sizes: empty shapes, and G * K beyond int32
    assert lib.adx_group_union_sizes(ctypes.c_void_p(64), 0, 8, 4, 16, ctypes.c_void_p(128),
                                     None) == L.ADX_EINVAL
    assert lib.adx_group_union_sizes(ctypes.c_void_p(64), 16, 1 << 20, 1 << 12, 16,
                                     ctypes.c_void_p(128), None) == L.ADX_EINVAL
    # group means: Hg beyond H, e4m3 without its scale
    assert lib.adx_group_query_mean(L.ADX_BF16, ctypes.c_void_p(256), None, ctypes.c_void_p(512),
                                    64, 16, 128, 8, 32, ctypes.c_void_p(1024),
                                    ctypes.c_void_p(2048), None) == L.ADX_EINVAL
    assert lib.adx_group_query_mean(L.ADX_E4M3, ctypes.c_void_p(256), None, ctypes.c_void_p(512),
                                    64, 16, 128, 8, 16, ctypes.c_void_p(1024),
                                    ctypes.c_void_p(2048), None) == L.ADX_EINVAL
    # MTP: the window length must split into whole groups
    full = _ops(T=32 * 16, S=4096)
    full.seq_len = 64
    grp = _ops(T=32 * 2, H=16, S=4096)
    grp.seq_len = 64
    assert lib.adx_mtp_workspace_size(ctypes.byref(full), ctypes.byref(grp), 16, 5, 512,
                                      64) == 0


def test_noalloc_reports_operand_errors_like_the_workspace_entry_point(lib):
    """adx_index_prefill_noalloc checks the operands before it touches the device, with the
    codes adx_index_prefill returns: an unsupported head count is ADX_EUNSUPPORTED, not a
    workspace error."""
    def noalloc(o, K=4):
        return lib.adx_index_prefill_noalloc(ctypes.byref(o), K, ctypes.c_void_p(4096), None,
                                             None, None)
    assert noalloc(_ops(H=5)) == L.ADX_EUNSUPPORTED
    assert noalloc(_ops(H=5)) == _prefill(lib, _ops(H=5))
    assert noalloc(_ops(d=96)) == L.ADX_EUNSUPPORTED
    assert noalloc(_ops(q=None)) == L.ADX_EINVAL
    assert noalloc(_ops(), K=0) == L.ADX_EINVAL
