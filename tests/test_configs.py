"""The workload records under configs/ hold the constants the generators and the bench use."""

import inspect
import json
import os

import bench
from sparse_attention_token_indexer_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load(name):
    with open(os.path.join(ROOT, "configs", name + ".json")) as f:
        return json.load(f)


def _anchor_defaults():
    sig = inspect.signature(inputs.AnchorStructure.__init__).parameters
    return {k: sig[k].default for k in ("n_anchor", "copies", "beta", "sigma", "gamma", "rho",
                                        "eps", "block")}


def test_records_match_the_bench_and_generators():
    pairs = {"c2_flat_prefill": bench.FLAT, "c3_group_mode": bench.GROUP,
             "c4_decode": bench.DECODE, "c5_chunked_prefill": bench.CHUNKED,
             "hisa_prefill": bench.HISA, "group_indexer": bench.GROUP_INDEXER,
             "mtp_round": bench.MTP}
    for name, consts in pairs.items():
        rec = _load(name)
        for k, v in consts.items():
            assert rec[k] == v, (name, k)
        if "anchor" in rec:
            assert rec["anchor"] == _anchor_defaults(), name
    tiny = _load("c1_tiny_prefill")
    for k, p in inspect.signature(inputs.tiny_prefill).parameters.items():
        if k != "device":
            assert tiny[k] == p.default, k
