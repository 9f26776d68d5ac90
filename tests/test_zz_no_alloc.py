"""adx_index_prefill_noalloc: the flat prefill for callers that cannot allocate device memory
(engines that plan every buffer in their own arena, plugin hosts without an allocator). It
runs on a scratch array compiled into the library instead of a caller workspace.

Checked through the C ABI against adx_index_prefill (same operands, a caller workspace) on
two calls in a row (the second call sees the first call's leftovers in the shared scratch).
Both entry points run the same kernels on the same inputs, so their outputs must agree bit
for bit. This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

from sparse_attention_token_indexer_b200 import _lib as L
from sparse_attention_token_indexer_b200 import build, indexer, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    return L.lib()


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _noalloc(lib, p, K):
    ops = indexer.make_operands(p["q"], p["w"], p["k"], p["q_scale"], p["k_scale"], p["q_pos0"])
    idx = torch.full((ops.T, K), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((ops.T, K), 7.0, dtype=torch.float32, device="cuda")
    st = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    code = lib.adx_index_prefill_noalloc(ctypes.byref(ops), K, ctypes.c_void_p(idx.data_ptr()),
                                         ctypes.c_void_p(sc.data_ptr()),
                                         ctypes.c_void_p(st.data_ptr()), _stream())
    assert code == L.ADX_OK, L.status_string(code)
    torch.cuda.synchronize()
    assert int(st.item()) == L.ADX_OK
    return idx.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("case", ["tiny", "anchor_bf16", "anchor_e4m3"])
def test_noalloc_matches_workspace_entry_point(lib, case):
    if case == "tiny":
        p = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inputs.tiny_prefill().items()}
    else:
        dt = case.split("_")[1]
        p = inputs.anchor_prefill(700, H=64, d=128, K=128, seed=41, device="cuda", dtype=dt)
    K = p["K"]
    ref_idx, ref_sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K, p["q_scale"],
                                               p["k_scale"], with_scores=True)
    ref_idx, ref_sc = ref_idx.cpu().numpy(), ref_sc.cpu().numpy()
    for _ in range(2):
        idx, sc = _noalloc(lib, p, K)
        assert np.array_equal(idx, ref_idx)
        assert np.array_equal(sc.view(np.uint32), ref_sc.view(np.uint32))
        assert np.all((idx >= -1) & (idx < p["S"]))


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    p = inputs.anchor_prefill(4096, H=64, d=128, K=64, seed=42, device="cuda")
    ops = indexer.make_operands(p["q"], p["w"], p["k"])
    need = lib.adx_workspace_size(L.ADX_OP_PREFILL, ctypes.byref(ops), 64, 0, 0, 0)
    assert need > (32 << 20)
    idx = torch.empty(4096, 64, dtype=torch.int32, device="cuda")
    code = lib.adx_index_prefill_noalloc(ctypes.byref(ops), 64, ctypes.c_void_p(idx.data_ptr()),
                                         None, None, _stream())
    assert code == L.ADX_EWORKSPACE
