"""The library's calls captured in a CUDA graph and replayed give, bit for bit, what the same
calls give when launched directly: every kernel of a call (query preparation, scoring, the
cluster select of few long decode rows, the bulk-copy select of many long prefill rows, bank
building and refinement) is a plain stream operation with no host synchronisation, and a
replay reads its inputs as they are at replay time.

Checked through the Python binding (which passes the current stream to the C ABI, the capture
stream inside torch.cuda.graph).
"""

import pytest
import torch

from sparse_attention_token_indexer_b200 import build, indexer, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    yield
    assert indexer.read_device_status() == 0


def _capture(fn):
    """Runs fn once directly (which also sizes its workspace), then captures it."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = fn()
    return g, out


def _same(got, ref, what):
    for a, b in zip(got, ref):
        assert torch.equal(a, b), what


def test_decode_step_from_a_graph():
    # 8 rows of up to 40000 keys: the cluster select; a row of 1 key and one of 300 as well
    prob = inputs.decode_problem(Bs=8, S=40000, H=64, d=128, K=512, Hg=16, steps=2, seed=51,
                                 device="cuda")
    seq = torch.tensor([40000, 39000, 20000, 8000, 40000, 1, 300, 33000], dtype=torch.int32,
                       device="cuda")
    q, w = prob["q_steps"][0].clone(), prob["w_steps"][0].clone()
    ws = indexer.Workspace("cuda")

    def step():
        return indexer.index_decode(q, w, prob["k"], seq, 512, k_scale=prob["k_scale"],
                                    with_scores=True, ws=ws)

    ref = [t.clone() for t in step()]
    g, out = _capture(step)
    g.replay()
    torch.cuda.synchronize()
    _same(out, ref, "decode replay")
    # the next step's query in the same buffers: the replay reads it
    q.copy_(prob["q_steps"][1])
    w.copy_(prob["w_steps"][1])
    ref2 = [t.clone() for t in step()]
    assert not torch.equal(ref2[0], ref[0])
    g.replay()
    torch.cuda.synchronize()
    _same(out, ref2, "decode replay, next query")
    del g


def test_long_row_prefill_from_a_graph():
    # 160 rows of ~40000 keys: the sample-threshold select with its bulk-copy ring
    p = inputs.anchor_prefill(160, H=64, d=128, K=256, seed=52, device="cuda", S=40000)
    ws = indexer.Workspace("cuda")

    def step():
        idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], 256, q_pos0=p["q_pos0"],
                                           with_scores=True, ws=ws)
        return idx, sc

    ref = [t.clone() for t in step()]
    g, out = _capture(step)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    _same(out, ref, "long-row prefill replay")
    del g


def test_group_bank_and_refine_from_a_graph():
    G, B, K = 64, 1024, 128
    p = inputs.group_prefill(2048, H=64, d=128, K=K, G=G, B=B, Hg=16, seed=53, device="cuda")
    ws = indexer.Workspace("cuda")

    def step():
        bank = indexer.group_bank(p["qbar"], p["wbar"], p["k"], G, B, "window", ws=ws)
        idx, sc = indexer.bank_refine(p["q"], p["w"], p["k"], bank, G, B, "window", K,
                                      with_scores=True, ws=ws)
        return bank, idx, sc

    ref = [t.clone() for t in step()]
    g, out = _capture(step)
    g.replay()
    torch.cuda.synchronize()
    _same(out, ref, "group bank and refinement replay")
    del g
