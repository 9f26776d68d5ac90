"""Failure detection without a GPU fault: a bounded device-side wait that runs out is recorded
in the workspace status word, read back on the host, and leaves the device usable."""

import ctypes

import pytest
import torch

from sparse_attention_token_indexer_b200 import _lib as L
from sparse_attention_token_indexer_b200 import build, indexer, inputs

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_is_reported_and_the_device_stays_usable():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    ws = indexer.Workspace("cuda")
    buf = ws.get(L.ADX_STATUS_BYTES)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.lib().adx_check_wait_timeout(ctypes.c_void_p(buf.data_ptr()), 5_000_000,
                                          stream) == L.ADX_OK
    assert indexer.read_device_status(ws) == L.ADX_ETIMEOUT
    assert indexer.read_device_status(ws) == L.ADX_OK            # reading clears it
    p = inputs.anchor_prefill(300, H=64, d=128, K=32, seed=29, device="cuda")
    idx, _, _ = indexer.index_prefill(p["q"], p["w"], p["k"], 32, ws=ws)
    torch.cuda.synchronize()
    assert indexer.read_device_status(ws) == L.ADX_OK
    assert int(idx[299].ge(0).sum()) == 32
    assert L.lib().adx_check_wait_timeout(ctypes.c_void_p(buf.data_ptr()), 0, stream) == L.ADX_EINVAL
