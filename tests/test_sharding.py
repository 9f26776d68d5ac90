"""Row-sharded prefill of one sequence over several ranks (host logic, gloo on CPU, world size
2): the longest-first row partition, the key all-gather and the gather of every rank's Top-K
rows to rank 0 (and to all ranks). The per-rank indexer is stubbed by the fp64 oracle's flat
Top-K of the same rows (ADIndex §3, Eqs. (1)-(2)), so the sharded result must equal the
single-rank one row for row. The CUDA path behind the default per-rank call is the library's
adx_index_prefill; this file covers what happens around it."""

import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

from oracle import indexer as ox
from sparse_attention_token_indexer_b200 import sharding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _problem(T=300, S=340, H=2, d=8, seed=3):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(T, H, d, generator=g, dtype=torch.float64)
    w = torch.rand(T, H, generator=g, dtype=torch.float64)
    k = torch.randn(S, d, generator=g, dtype=torch.float64)
    return q, w, k, S - T


def _oracle_rows(q, w, k, K, p0):
    out = torch.full((q.shape[0], K), -1, dtype=torch.int32)
    for i in range(q.shape[0]):
        top = np.sort(ox.flat_topk_row(q[i].numpy(), w[i].numpy(), k.numpy(), p0 + i, K))
        out[i, :len(top)] = torch.as_tensor(top, dtype=torch.int32)
    return out


def test_partition_covers_every_row_once_and_balances_the_triangle():
    for T, q_pos0, world, unit in ((16384, 0, 8, 64), (4096, 258048, 4, 64), (1000, 7, 3, 37),
                                   (50, 0, 8, 64)):
        ranges, loads = sharding.partition_rows(T, q_pos0, world, unit)
        rows = sorted(r for rs in ranges for r0, r1 in rs for r in range(r0, r1))
        assert rows == list(range(T))
        assert loads == [sum(sharding.unit_cost(q_pos0, r0, r1) for r0, r1 in rs)
                         for rs in ranges]
        assert sum(loads) == sum(q_pos0 + t + 1 for t in range(T))
        # longest-processing-time bound: no rank exceeds the mean by more than one unit
        biggest = max(sharding.unit_cost(q_pos0, r0, min(T, r0 + unit)) for r0 in range(0, T, unit))
        assert max(loads) <= sum(loads) / world + biggest
    ranges, loads = sharding.partition_rows(16384, 0, 8, 64)
    assert max(loads) / min(loads) < 1.01


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        q, w, k, q_pos0 = _problem()
        K = 16
        # keys: each rank holds a contiguous slice of the sequence (uneven split)
        cut = [0, 150, k.shape[0]]
        k_full = sharding.all_gather_keys(k[cut[rank]:cut[rank + 1]].contiguous())
        calls = []

        def stub(qr, wr, kk, KK, p0):
            calls.append((p0, qr.shape[0]))
            return _oracle_rows(qr, wr, kk, KK, p0)

        got0 = sharding.sharded_prefill(q, w, k_full, K, q_pos0=q_pos0, unit=37, index_fn=stub)
        got_all = sharding.sharded_prefill(q, w, k_full, K, q_pos0=q_pos0, unit=37,
                                           index_fn=stub, to_all=True)
        out.put((rank, torch.equal(k_full, k), None if got0 is None else got0.numpy(),
                 got_all.numpy(), calls))
    finally:
        dist.destroy_process_group()


def test_sharded_prefill_equals_the_single_rank_result_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    qout = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, qout)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, keys_ok, got0, got_all, calls = qout.get(timeout=300)
        res[rank] = (keys_ok, got0, got_all, calls)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, w, k, q_pos0 = _problem()
    ref = _oracle_rows(q, w, k, 16, q_pos0).numpy()
    assert res[0][0] and res[1][0]                      # the gathered keys are the sequence's
    assert np.array_equal(res[0][1], ref)               # rank 0 holds every row
    assert res[1][1] is None                            # the other rank gets nothing
    assert np.array_equal(res[0][2], ref) and np.array_equal(res[1][2], ref)
    # each rank indexed its own units only (two calls per unit: gather, then all-gather)
    ranges, _ = sharding.partition_rows(q.shape[0], q_pos0, 2, 37)
    for rank in (0, 1):
        want = sorted((q_pos0 + r0, r1 - r0) for r0, r1 in ranges[rank])
        assert sorted(res[rank][3]) == sorted(want * 2)
