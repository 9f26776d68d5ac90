"""ctypes binding of libadx.so (include/adx.h): structure layout, symbol signatures and the
library loader. Loading fails loudly when the library has not been built; there is no
fallback implementation."""

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libadx.so")

ADX_OK, ADX_EINVAL, ADX_EUNSUPPORTED, ADX_EWORKSPACE, ADX_ECUDA, ADX_EOVERFLOW, ADX_ETIMEOUT = range(7)
ADX_BF16, ADX_E4M3 = 0, 1
ADX_BANK_PAPER, ADX_BANK_WINDOW = 0, 1
(ADX_OP_PREFILL, ADX_OP_DECODE, ADX_OP_GROUP_BANK, ADX_OP_BANK_REFINE, ADX_OP_PREFILL_HOST,
 ADX_OP_BANK_REFINE_PACKED) = range(6)
ADX_HISA_BLOCK = 128
ADX_STATUS_BYTES = 256

# every extern "C" symbol include/adx.h declares
EXPORTS = ("adx_abi_version", "adx_bank_width", "adx_status_string", "adx_workspace_size",
           "adx_index_prefill", "adx_index_decode", "adx_group_bank", "adx_bank_refine",
           "adx_read_device_status", "adx_set_timing_events", "adx_launch_count",
           "adx_index_prefill_noalloc", "adx_mtp_workspace_size", "adx_index_mtp",
           "adx_group_union_sizes", "adx_group_query_mean", "adx_index_prefill_host",
           "adx_check_wait_timeout", "adx_group_indexer_workspace_size",
           "adx_group_indexer_queries", "adx_hisa_block_keys", "adx_hisa_workspace_size",
           "adx_index_hisa", "adx_bank_coverage", "adx_pack_bank_keys",
           "adx_bank_refine_packed")


class Operands(ctypes.Structure):
    _fields_ = [
        ("q_dtype", ctypes.c_int32),
        ("k_dtype", ctypes.c_int32),
        ("q", ctypes.c_void_p),
        ("q_scale", ctypes.c_void_p),
        ("w", ctypes.c_void_p),
        ("k", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("T", ctypes.c_int32),
        ("H", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("S", ctypes.c_int32),
        ("q_pos0", ctypes.c_int64),
        ("seq_len", ctypes.c_void_p),
    ]


class GroupIndexer(ctypes.Structure):
    _fields_ = [
        ("cq", ctypes.c_void_p),
        ("h", ctypes.c_void_p),
        ("w_pool", ctypes.c_void_p),
        ("w_q", ctypes.c_void_p),
        ("w_g", ctypes.c_void_p),
        ("T", ctypes.c_int32),
        ("d_c", ctypes.c_int32),
        ("d_h", ctypes.c_int32),
        ("H_S", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("rope_dim", ctypes.c_int32),
        ("rope_base", ctypes.c_float),
        ("q_pos0", ctypes.c_int64),
    ]


class AdxError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {code} ({status_string(code)})")


_lib = None


def _declare(lib):
    P, I32, I64, SZ, VP = (ctypes.POINTER(Operands), ctypes.c_int32, ctypes.c_int64,
                           ctypes.c_size_t, ctypes.c_void_p)
    sig = {
        "adx_abi_version": (I32, []),
        "adx_bank_width": (I32, [I32, I32, I32]),
        "adx_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "adx_workspace_size": (SZ, [I32, P, I32, I32, I32, I32]),
        "adx_index_prefill": (ctypes.c_int, [P, I32, VP, VP, VP, I64, VP, SZ, VP]),
        "adx_index_decode": (ctypes.c_int, [P, I32, VP, VP, VP, SZ, VP]),
        "adx_group_bank": (ctypes.c_int, [P, I32, I32, I32, VP, VP, SZ, VP]),
        "adx_bank_refine": (ctypes.c_int, [P, I32, I32, I32, VP, I32, VP, VP, VP, SZ, VP]),
        "adx_read_device_status": (ctypes.c_int, [VP, VP]),
        "adx_set_timing_events": (None, [ctypes.POINTER(VP), I32]),
        "adx_launch_count": (I64, []),
        "adx_index_prefill_noalloc": (ctypes.c_int, [P, I32, VP, VP, VP, VP]),
        "adx_mtp_workspace_size": (SZ, [P, P, I32, I32, I32, I32]),
        "adx_index_mtp": (ctypes.c_int, [P, P, I32, I32, I32, I32, VP, VP, VP, VP, SZ, VP]),
        "adx_group_union_sizes": (ctypes.c_int, [VP, I32, I32, I32, I32, VP, VP]),
        "adx_bank_coverage": (ctypes.c_int, [VP, I32, I32, VP, I32, I32, I32, VP, VP, VP]),
        "adx_pack_bank_keys": (ctypes.c_int, [P, I32, I32, VP, VP, VP, VP]),
        "adx_bank_refine_packed": (ctypes.c_int, [P, I32, I32, VP, VP, VP, I32, VP, VP, VP, SZ,
                                                  VP]),
        "adx_index_prefill_host": (ctypes.c_int, [P, I32, I32, VP, VP, VP, SZ, VP]),
        "adx_check_wait_timeout": (ctypes.c_int, [VP, ctypes.c_uint64, VP]),
        "adx_hisa_block_keys": (ctypes.c_int, [P, I32, VP, VP, VP]),
        "adx_hisa_workspace_size": (SZ, [P, I32, I32, I32]),
        "adx_index_hisa": (ctypes.c_int, [P, VP, VP, I32, I32, VP, VP, VP, VP, SZ, VP]),
        "adx_group_indexer_workspace_size": (SZ, [ctypes.POINTER(GroupIndexer), I32]),
        "adx_group_indexer_queries": (ctypes.c_int, [ctypes.POINTER(GroupIndexer), I32, VP, VP,
                                                     VP, SZ, VP]),
        "adx_group_query_mean": (ctypes.c_int, [I32, VP, VP, VP, I32, I32, I32, I32, I32, VP,
                                                VP, VP]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args


def lib():
    """The loaded library; raises if libadx.so is missing (build it with build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run "
                               "`python -m sparse_attention_token_indexer_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        _declare(handle)
        _lib = handle
    return _lib


def status_string(code):
    return lib().adx_status_string(int(code)).decode()


def check(fn, code):
    if code != ADX_OK:
        raise AdxError(fn, code)
