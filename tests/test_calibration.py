"""Layer-wise reuse calibration (ADIndex §4.1): the speedup S(G, P; L) against the oracle's
plan counts and the paper's Table 5 panel c, the configuration choice of Eq. (5) against a
brute-force search, the capacity criteria, and (GPU) the union sizes of Eq. (4) against the
oracle on the indexer's own Top-K output."""

import os

import numpy as np
import pytest
import torch

from oracle import cost_model
from oracle import indexer as ox
from sparse_attention_token_indexer_b200 import calibration as cal

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "table5_speedups.txt")
K1 = 1024


def test_speedup_equals_the_oracle_plan_counts():
    for L in (16 * K1, 32 * K1, 64 * K1, 128 * K1):
        for G in cal.GROUP_SIZES:
            for P in cal.BUDGETS:
                assert cal.speedup(G, P, L) == pytest.approx(cost_model.speedups(L, G, P)[2],
                                                            rel=1e-12)


def test_speedup_reproduces_table5_panel_c():
    cols = (16 * K1, 32 * K1, 64 * K1, 128 * K1)
    n = 0
    for line in open(GOLDEN):
        f = line.split()
        if not f or f[0] != "c":
            continue
        G, P = int(f[1]), int(f[2]) * K1
        for L, v in zip(cols, map(float, f[3:])):
            assert abs(cal.speedup(G, P, L) - v) <= 0.0101, (G, P, L)
            n += 1
    assert n == 36


def test_select_config_is_the_constrained_argmax():
    rng = np.random.default_rng(5)
    for _ in range(30):
        caps = {G: float(rng.integers(1000, 20000)) for G in cal.GROUP_SIZES}
        feasible = [(cal.speedup(G, P, 128 * K1), G, P) for G in cal.GROUP_SIZES
                    for P in cal.BUDGETS if caps[G] <= P]
        want = max(feasible)[1:] if feasible else None
        assert cal.select_config(caps) == want
    assert cal.select_config({4: 20000.0, 8: 30000.0, 16: 40000.0}) is None


def test_capacity_criteria():
    u = np.arange(1, 101)
    assert cal.capacity(u, "max") == 100
    assert cal.capacity(u, "mean") == pytest.approx(50.5)
    assert cal.capacity(u, "p90") == pytest.approx(np.percentile(u, 90))
    with pytest.raises(ValueError):
        cal.capacity(u, "median")


@pytest.mark.gpu
@pytest.mark.parametrize("G", cal.GROUP_SIZES)
def test_union_sizes_on_the_indexer_output(G):
    from sparse_attention_token_indexer_b200 import build, indexer, inputs
    build.build()
    T, K = 3000, 256
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=25, device="cuda")
    idx, _, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K)
    got = cal.union_sizes(idx, G, T).cpu().tolist()
    assert got == ox.group_union_sizes(idx.cpu().numpy(), G)
    choice, caps = cal.calibrate_layer(idx, T)
    ref_caps = {g: float(max(ox.group_union_sizes(idx.cpu().numpy(), g)))
                for g in cal.GROUP_SIZES}
    assert caps == ref_caps
    feasible = [(cost_model.speedups(128 * K1, g, P)[2], g, P) for g in cal.GROUP_SIZES
                for P in cal.BUDGETS if ref_caps[g] <= P]
    assert choice == (max(feasible)[1:] if feasible else None)


def test_coverage_by_position_hand_values():
    hits = [4, 2, 2, 3]
    count = [4, 2, 4, 4]
    per_pos, mean = cal.coverage_by_position(hits, count, 2)
    assert per_pos.tolist() == [0.75, 0.875]
    assert mean == pytest.approx(0.8125)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["window", "paper"])
def test_bank_coverage_equals_the_oracle(mode):
    """ADIndex Figure 1(c) / Appendix B.4 coverage on the library's own outputs: the flat
    Top-K rows and the group banks of a group-mode problem. Integer work: equal to the
    oracle's counts on the same rows, element for element."""
    from sparse_attention_token_indexer_b200 import build, indexer, inputs
    build.build()
    T, G, B, K, Hg = 64 * 20 + 9, 64, 512, 256, 16
    p = inputs.group_prefill(T, H=64, d=128, K=K, G=G, B=B, Hg=Hg, seed=29, device="cuda")
    flat, _, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K)
    bank = indexer.group_bank(p["qbar"], p["wbar"], p["k"], G, B, mode)
    hits, count = cal.bank_coverage(flat, bank, G, T)
    ref_h, ref_c = ox.bank_coverage(flat.cpu().numpy(), bank.cpu().numpy(), G)
    assert hits.cpu().numpy().tolist() == ref_h.tolist()
    assert count.cpu().numpy().tolist() == ref_c.tolist()
    # groups whose bank holds the anchor's whole visible prefix cover every member fully: the
    # PAPER groups that fall back (a + 1 <= B, their bank path keeps every key) and the WINDOW
    # groups whose scan is no longer than the bank
    full = [g for g, pl in enumerate(ox.plan_groups(T, 0, G, B, mode))
            if len(pl.rows) == G and (pl.kind == "flat" or pl.scan_n <= pl.bank_k)]
    h, c = hits.cpu().numpy().reshape(-1, G), count.cpu().numpy().reshape(-1, G)
    assert full and all(np.array_equal(h[g], c[g]) for g in full)
    assert (h < c).any()
