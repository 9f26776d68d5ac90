"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Sources: "ADIndex: Layer-Adaptive Sparse Attention Indexing via Group-Level Distillation"
(arXiv 2611.12956v1) - §3 Eqs. (1)-(2), §1 (exact recovery when the bank holds the Top-K),
§4.3 Eqs. (13)-(14) and the fallback rules, Appendix A and Table 5 (score counts) - plus
library routines (torch's bf16 / float8 conversions, numpy's stable argsort) and brute force.
"""

import itertools
import os

import numpy as np
import pytest
import torch

from oracle import cost_model, fp_formats
from oracle import indexer as ox

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------------------
# operand decoding
# ---------------------------------------------------------------------------------------

def test_bf16_decode_matches_torch_on_every_code():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = fp_formats.bf16_bits_to_f64(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = fp_formats.e4m3_to_f64(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9  # largest finite, smallest subnormal


def test_dequantize_applies_per_row_scale():
    codes = np.array([[0x38, 0xB8], [0x40, 0x00]], dtype=np.uint8)  # 1, -1 ; 2, 0
    got = fp_formats.dequantize(codes, np.array([0.5, 3.0], dtype=np.float32), "e4m3")
    assert np.array_equal(got, [[0.5, -0.5], [6.0, 0.0]])


# ---------------------------------------------------------------------------------------
# Eq. (1): hand-computed values and closed forms
# ---------------------------------------------------------------------------------------

Q2 = np.array([[1.0, 2.0], [-1.0, 1.0]])          # H = 2 heads, d = 2
K3 = np.array([[3.0, -1.0], [0.0, 1.0], [-2.0, -2.0]])


def test_score_hand_values():
    # head 0 dots: 1, 2, -6 -> ReLU 1, 2, 0 ; head 1 dots: -4, 1, 0 -> ReLU 0, 1, 0
    # I = 0.5 * [1, 2, 0] + 2 * [0, 1, 0]
    assert np.array_equal(ox.score_keys(Q2, [0.5, 2.0], K3), [0.5, 3.0, 0.0])


def test_score_negative_gate_keeps_relu_per_head():
    # ReLU before the gate: a negative gate can make a score negative
    assert np.array_equal(ox.score_keys(Q2, [-1.0, 1.0], K3), [-1.0, -1.0, 0.0])


def test_score_all_negative_logits_is_zero():
    k = -np.abs(np.random.default_rng(0).normal(size=(5, 2)))
    q = np.abs(np.random.default_rng(1).normal(size=(3, 2)))
    assert np.array_equal(ox.score_keys(q, [1.0, 2.0, 3.0], k), np.zeros(5))


def test_score_single_head_unit_gate_is_dot_product():
    rng = np.random.default_rng(2)
    q = rng.normal(size=(1, 16))
    k = rng.normal(size=(40, 16))
    k[np.dot(k, q[0]) < 0] *= -1                     # make every dot product positive
    assert np.allclose(ox.score_keys(q, [1.0], k), np.dot(k, q[0]), rtol=1e-14, atol=0)


def test_score_positive_scales_factor_out():
    rng = np.random.default_rng(3)
    q, w, k = rng.normal(size=(4, 8)), rng.normal(size=4), rng.normal(size=(10, 8))
    got = ox.score_keys(q * 0.25, w, k * 8.0)
    assert np.allclose(got, 2.0 * ox.score_keys(q, w, k), rtol=1e-13, atol=1e-13)


def test_indexer_scores_causal_mask():
    rng = np.random.default_rng(4)
    T, H, d = 6, 2, 4
    q, w, k = rng.normal(size=(T, H, d)), rng.random((T, H)), rng.normal(size=(T, d))
    I = ox.indexer_scores(q, w, k, np.arange(T))
    for t in range(T):
        assert np.all(np.isfinite(I[t, : t + 1])) and np.all(I[t, t + 1:] == -np.inf)
        # brute force: per head, per key, written out
        for s in range(t + 1):
            ref = sum(w[t, j] * max(0.0, sum(q[t, j, x] * k[s, x] for x in range(d)))
                      for j in range(H))
            assert abs(I[t, s] - ref) <= 1e-12 * max(1.0, abs(ref))


# ---------------------------------------------------------------------------------------
# Eq. (2): Top-K
# ---------------------------------------------------------------------------------------

def test_topk_brute_force_small():
    rng = np.random.default_rng(5)
    for n in range(1, 10):
        for K in range(1, 5):
            sc = rng.normal(size=n)
            got = set(ox.topk(sc, K).tolist())
            best = None
            for sub in itertools.combinations(range(n), min(K, n)):
                rest = [s for s in range(n) if s not in sub]
                if not rest or min(sc[list(sub)]) >= max(sc[rest]):
                    best = set(sub)
            assert got == best


def test_topk_matches_stable_argsort_with_ties():
    sc = np.array([3.0, 1.0, 3.0, 2.0, 3.0, 1.0, 2.0])
    for K in range(1, 8):
        ref = np.argsort(-sc, kind="stable")[:K]
        assert np.array_equal(ox.topk(sc, K), ref)


def test_flat_topk_causal_counts():
    rng = np.random.default_rng(6)
    T, H, d, K = 12, 2, 4, 4
    q, w, k = rng.normal(size=(T, H, d)), rng.random((T, H)), rng.normal(size=(T, d))
    res = ox.flat_topk(q, w, k, np.arange(T), K)
    for t, idx in res.items():
        assert len(idx) == min(K, t + 1) == len(set(idx.tolist()))
        assert idx.max() <= t
        if t + 1 <= K:
            assert sorted(idx.tolist()) == list(range(t + 1))


def test_topk_permutation_equivariance_and_monotonicity():
    rng = np.random.default_rng(7)
    H, d, S, K = 3, 8, 40, 6
    q, w, k = rng.normal(size=(H, d)), rng.random(H), rng.normal(size=(S, d))
    base = set(ox.flat_topk_row(q, w, k, S - 1, K).tolist())
    perm = rng.permutation(S)
    permuted = set(ox.flat_topk_row(q, w, k[perm], S - 1, K).tolist())
    assert {int(perm[i]) for i in permuted} == base
    sc = ox.score_keys(q, w, k)
    chosen = sorted(base)[0]
    unchosen = [s for s in range(S) if s not in base][0]
    k2 = k.copy()
    k2[chosen] *= 1.5 if sc[chosen] > 0 else 1.0       # raise a selected score
    k2[unchosen] *= 0.5 if sc[unchosen] > 0 else 1.0   # lower an unselected one
    assert set(ox.flat_topk_row(q, w, k2, S - 1, K).tolist()) == base


# ---------------------------------------------------------------------------------------
# Eqs. (13)-(14): bank and refinement
# ---------------------------------------------------------------------------------------

def _prob(T=48, H=3, Hg=2, d=8, G=8, seed=8):
    rng = np.random.default_rng(seed)
    q, w, k = rng.normal(size=(T, H, d)), rng.random((T, H)), rng.normal(size=(T, d))
    qbar, wbar = rng.normal(size=(T // G, Hg, d)), rng.random((T // G, Hg))
    return q, w, k, qbar, wbar


def test_refine_exact_recovery_when_bank_holds_topk():
    q, w, k, *_ = _prob()
    rng = np.random.default_rng(9)
    K = 5
    for i in range(10, 48):
        full = ox.flat_topk_row(q[i], w[i], k, i, K)
        extra = rng.choice(i, size=3, replace=False)
        bank = np.union1d(full, extra)
        got = ox.refine_row(q[i], w[i], k, bank, i + 1, i, K)
        assert set(got.tolist()) == set(full.tolist())


@pytest.mark.parametrize("mode", ["paper", "window"])
def test_large_bank_equals_flat(mode):
    q, w, k, qbar, wbar = _prob()
    T, K, G = 48, 5, 8
    flat = ox.flat_topk(q, w, k, np.arange(T), K)
    got, _ = ox.group_topk(q, w, k, qbar, wbar, 0, G, B=T + G, K=K, mode=mode)
    for t in range(T):
        assert set(got[t].tolist()) == set(flat[t].tolist())


def test_window_group_of_one_is_flat():
    q, w, k, _, _ = _prob()
    T, K = 48, 5
    rng = np.random.default_rng(10)
    qbar, wbar = rng.normal(size=(T, 2, 8)), rng.random((T, 2))
    flat = ox.flat_topk(q, w, k, np.arange(T), K)
    got, _ = ox.group_topk(q, w, k, qbar, wbar, 0, 1, B=T + 1, K=K, mode="window")
    assert all(set(got[t].tolist()) == set(flat[t].tolist()) for t in range(T))


def test_candidates_stay_causal_and_in_bank():
    q, w, k, qbar, wbar = _prob()
    T, K, G, B = 48, 4, 8, 12
    for mode in ("paper", "window"):
        got, banks = ox.group_topk(q, w, k, qbar, wbar, 0, G, B, K, mode)
        plans = ox.plan_groups(T, 0, G, B, mode)
        for gi, plan in enumerate(plans):
            for t in plan.rows:
                idx = got[t]
                assert len(idx) == len(set(idx.tolist())) and idx.max() <= t
                if plan.kind == "bank":
                    allowed = set(banks[gi].tolist()) | set(range(plan.post_lo, t + 1))
                    assert set(idx.tolist()) <= allowed
                    assert len(banks[gi]) == min(plan.bank_k, plan.scan_n)
                    assert banks[gi].max(initial=-1) < plan.scan_n


def test_window_group_cost_closed_form():
    """WINDOW reading (the group-mode workloads; ADIndex §4.3, Eqs. (13)-(14)): a bank group
    whose anchor a has at least B - G keys before it scores a scan of the a keys s < a, then
    member i = a + r (r = 0 .. G-1) scores the B - G bank keys plus its r + 1 window keys
    a .. a + r: a + G (B - G) + G (G + 1) / 2 in all. With fewer than B - G keys before the
    anchor the bank holds all a of them instead."""
    for G, B, a in ((16, 64, 1000), (64, 8192, 65536 - 64), (8, 40, 32), (8, 40, 20)):
        plans = ox.plan_groups(G, a, G, B, "window")
        assert len(plans) == 1 and plans[0].kind == "bank"
        bank = min(B - G, a)
        assert cost_model.plan_cost(plans, a) == a + G * bank + G * (G + 1) // 2, (G, B, a)


def _window_hand_case():
    """One WINDOW group (G = 4, B = 8, anchor a = 10) with hand-set keys. The group query
    reads dimension 0, the members' queries dimension 1.
      group scores: s < a score s + 1, so the scan's best B - G = 4 keys are 9, 8, 7, 6 and
                    the fifth (rank B - G + 1) is 5; the anchor's own key scores 100, above
                    every scanned key.
      member scores: key 5 scores 50 and the anchor's key 60, every other key at most 1.3."""
    G, B, a, K = 4, 8, 10, 3
    S = a + G
    k = np.zeros((S, 4))
    k[:a, 0] = np.arange(1, a + 1)
    k[a, 0] = 100.0
    k[:, 1] = 0.1 * np.arange(S)
    k[5, 1], k[a, 1] = 50.0, 60.0
    qbar, wbar = np.array([[[1.0, 0, 0, 0]]]), np.array([[1.0]])
    q = np.tile(np.array([[0, 1.0, 0, 0], [0, 0.5, 0, 0]]), (G, 1, 1))   # [G, 2, 4]
    w = np.ones((G, 2))
    return q, w, k, qbar, wbar, G, B, a, K


def test_window_bank_holds_the_anchor_through_the_window_not_the_scan():
    """The WINDOW scan covers s < a only: the anchor's key, although the group query's best,
    is not a scanned bank entry; every member still sees it through the window a .. i."""
    q, w, k, qbar, wbar, G, B, a, K = _window_hand_case()
    plans = ox.plan_groups(G, a, G, B, "window")
    bank = ox.token_bank(qbar[0], wbar[0], k, plans[0])
    assert a not in bank.tolist()
    got, _ = ox.group_topk(q, w, k, qbar, wbar, a, G, B, K, "window")
    for r in range(G):
        assert a in got[r].tolist(), r


def test_window_bank_keeps_exactly_B_minus_G_scan_keys():
    """The WINDOW bank keeps the scan's best B - G keys and not one more: the key of rank
    B - G + 1 (position 5) stays out of the bank and out of every member's result, although
    it would be every member's second-best key."""
    q, w, k, qbar, wbar, G, B, a, K = _window_hand_case()
    plans = ox.plan_groups(G, a, G, B, "window")
    bank = ox.token_bank(qbar[0], wbar[0], k, plans[0])
    assert sorted(bank.tolist()) == [6, 7, 8, 9]
    got, banks = ox.group_topk(q, w, k, qbar, wbar, a, G, B, K, "window")
    assert sorted(banks[0].tolist()) == [6, 7, 8, 9]
    for r in range(G):
        assert 5 not in got[r].tolist(), r
    # the same query against the flat indexer does take key 5: the bank is what drops it
    flat = ox.flat_topk_row(q[G - 1], w[G - 1], k, a + G - 1, K)
    assert 5 in flat.tolist()


def test_paper_fallback_rule():
    plans = ox.plan_groups(T=40, q_pos0=0, G=8, B=16, mode="paper")
    # anchors 0, 8, 16, 24, 32: reuse needs a + 1 > 16; the last group is complete
    assert [p.kind for p in plans] == ["flat", "flat", "bank", "bank", "bank"]
    # at the boundary: a bank only when the anchor's visible prefix a + 1 exceeds B (ADIndex
    # §4.3, Shared Token Bank Construction; Appendix A: a prefix that does not exceed the
    # budget falls back), so the anchor 16 with a + 1 = B = 17 takes the plain indexer
    plans = ox.plan_groups(T=40, q_pos0=0, G=8, B=17, mode="paper")
    assert [p.kind for p in plans] == ["flat", "flat", "flat", "bank", "bank"]
    plans = ox.plan_groups(T=36, q_pos0=0, G=8, B=16, mode="paper")
    assert plans[-1].kind == "flat" and len(plans[-1].rows) == 4   # incomplete group
    # MTP: the whole window falls back when its first query sees <= B keys
    assert all(p.kind == "flat" for p in ox.plan_groups(16, 15, 4, 16, "paper", "window"))
    assert all(p.kind == "bank" for p in ox.plan_groups(16, 16, 4, 16, "paper", "window"))


def test_decode_bank_reuse_matches_definitions():
    rng = np.random.default_rng(11)
    Bs, H, Hg, d, S, K, B = 3, 3, 2, 8, 60, 5, 10
    caches = rng.normal(size=(Bs, S, d))
    q, w = rng.normal(size=(Bs, H, d)), rng.random((Bs, H))
    qbar, wbar = rng.normal(size=(Bs, Hg, d)), rng.random((Bs, Hg))
    n0 = np.array([50, 40, 55])
    banks = ox.decode_bank(qbar, wbar, caches, n0, B)
    flat = ox.decode_topk(q, w, caches, n0 + 4, K)
    # a bank as large as the prefix makes reuse exact
    big = ox.decode_bank(qbar, wbar, caches, n0, S)
    got = ox.decode_refine(q, w, caches, n0 + 4, big, n0 - 1, K)
    assert all(set(got[b].tolist()) == set(flat[b].tolist()) for b in range(Bs))
    got = ox.decode_refine(q, w, caches, n0 + 4, banks, n0 - 1, K)
    for b in range(Bs):
        allowed = set(banks[b].tolist()) | set(range(n0[b], n0[b] + 4))
        assert set(got[b].tolist()) <= allowed and len(got[b]) == K
    # Eq. (13) scans s <= t, the anchor's own key included: a key at the anchor that the group
    # query scores far above the rest is in the bank
    c2 = caches.copy()
    for b in range(Bs):
        c2[b, n0[b] - 1] = 1000.0 * qbar[b, 0]
    banks2 = ox.decode_bank(qbar, wbar, c2, n0, B)
    assert all(int(n0[b]) - 1 in set(banks2[b].tolist()) for b in range(Bs))


# ---------------------------------------------------------------------------------------
# Appendix A: the procedure's score counts reproduce Table 5
# ---------------------------------------------------------------------------------------

def _table5():
    rows = []
    with open(os.path.join(GOLDEN, "table5_speedups.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                p, G, P, *vals = line.split()
                rows.append((p, int(G), int(P) * 1024, [float(v) for v in vals]))
    return rows


def test_cost_closed_forms_of_appendix_a():
    """ADIndex Appendix A, exact: a verification round's baseline count m N + m (m - 1) / 2
    (Eq. (16), query r of the round sees N + r keys); an active round's count
    sum over its m / G groups b of N + bG + GP + G (G - 1) / 2 (Eq. (20)); the prefill baseline
    sum_t (t + 1) = L (L + 1) / 2 (the discrete sum Eq. (15) integrates); and the joint
    workload's rounds at N_j = L + (j - 1) a, so sum_j N_j = R L + a R (R - 1) / 2 (Eqs. (28),
    (29)), which fixes the joint speedup given the prefill counts."""
    m = 16
    for N in (5000, 16384, 70001):
        assert cost_model.base_cost(m, N - 1) == m * N + m * (m - 1) // 2
        for G in (4, 8, 16):
            for P in (1024, 4096):
                assert cost_model.mtp_round_cost(N, G, P, m) == sum(
                    N + b * G + G * P + G * (G - 1) // 2 for b in range(m // G))
    for L in (4096, 20000):
        assert cost_model.base_cost(L, 0) == L * (L + 1) // 2
    L, R, a = 65536, 32, 8
    S = R * L + a * R * (R - 1) // 2
    for G in (4, 8, 16):
        for P in (4096, 16384):
            nb = m // G
            jb = L * (L + 1) // 2 + m * S + R * m * (m - 1) // 2
            jr = cost_model.prefill_cost(L, G, P) + nb * S + R * (
                G * nb * (nb - 1) // 2 + nb * (G * P + G * (G - 1) // 2))
            assert cost_model.speedups(L, G, P, R, m, a)[2] == pytest.approx(jb / jr, rel=1e-12)


def test_group_cost_matches_eq17():
    # one bank group with anchor visible prefix N: N + G P + G (G - 1) / 2
    G, P, a = 16, 4096, 10000
    plan = ox.plan_groups(G, a, G, P, "paper")
    assert len(plan) == 1 and plan[0].kind == "bank"
    assert cost_model.plan_cost(plan, a) == (a + 1) + G * P + G * (G - 1) // 2


def test_table5_reproduced_by_the_group_plan():
    rows = _table5()
    assert len(rows) == 27
    ctx = [16 * 1024, 32 * 1024, 64 * 1024, 128 * 1024]
    cache = {}
    for panel, G, P, vals in rows:
        for L, ref in zip(ctx, vals):
            key = (L, G, P)
            if key not in cache:
                cache[key] = cost_model.speedups(L, G, P)
            got = cache[key]["abc".index(panel)]
            if panel == "b":
                # Eqs. (20)-(21) are discrete: same 2-decimal value
                assert round(got, 2) == pytest.approx(ref, abs=1e-9), (panel, G, P, L, got)
            else:
                # (a) and (c) use the integral of Eq. (19); the discrete count differs from it
                # by less than one unit in the last printed digit
                assert abs(got - ref) <= 0.0101, (panel, G, P, L, got)


# ---------------------------------------------------------------------------------------
# MTP target verification (ADIndex §4.3 and Appendix A.2)
# ---------------------------------------------------------------------------------------

def _relu_scores(qh, wh, keys):
    """Eq. (1) written out with einsum, independent of the oracle's score_keys."""
    return (np.maximum(np.einsum("hd,nd->hn", qh, keys), 0.0) * wh[:, None]).sum(axis=0)


def test_mtp_window_fallback_is_flat_even_past_the_budget():
    """N <= P sends the whole window to the plain indexer, also for groups whose anchors
    already see more than P keys (the per-group prefill rule would bank those)."""
    rng = np.random.default_rng(40)
    m, G, P, K, H, d = 16, 4, 40, 8, 3, 8
    N = P - 2
    n = N + m - 1
    k = rng.standard_normal((n, d))
    q = rng.standard_normal((m, H, d))
    w = rng.random((m, H))
    qbar, wbar = -q[::G], w[::G]        # banks that prefer the keys the rows like least
    out = ox.mtp_topk(q, w, [k], qbar, wbar, [n], m, G, P, K)
    for j in range(m):
        p = n - m + j
        s = _relu_scores(q[j], w[j], k[:p + 1])
        ref = sorted(range(p + 1), key=lambda x: (-s[x], x))[:K]
        assert set(out[j]) == set(ref)
    per_group, _ = ox.group_topk(q, w, k, qbar, wbar, n - m, G, P, K, "paper", fallback="group")
    assert any(set(per_group[j]) != set(out[j]) for j in range(m))


def test_mtp_banked_window_matches_the_equations():
    """N > P: group g of sequence b has its anchor at seq_len[b] - m + g*G, a bank of the P
    best keys (group query, s <= anchor) and candidates bank U {anchor+1 .. own position}."""
    rng = np.random.default_rng(41)
    m, G, P, K, H, Hg, d = 16, 8, 20, 6, 4, 2, 8
    seq_len = [60, 91]
    caches = [rng.standard_normal((n, d)) for n in seq_len]
    q = rng.standard_normal((2 * m, H, d))
    w = rng.random((2 * m, H))
    qbar = rng.standard_normal((2 * m // G, Hg, d))
    wbar = rng.random((2 * m // G, Hg))
    out = ox.mtp_topk(q, w, caches, qbar, wbar, seq_len, m, G, P, K)
    for b, n in enumerate(seq_len):
        k = caches[b]
        for g in range(m // G):
            a = n - m + g * G
            sb = _relu_scores(qbar[b * (m // G) + g], wbar[b * (m // G) + g], k[:a + 1])
            bank = sorted(range(a + 1), key=lambda x: (-sb[x], x))[:P]
            for j in range(g * G, g * G + G):
                p = n - m + j
                cand = sorted(set(bank) | set(range(a + 1, p + 1)))
                s = _relu_scores(q[b * m + j], w[b * m + j], k[cand])
                ref = [cand[i] for i in sorted(range(len(cand)), key=lambda x: (-s[x], cand[x]))[:K]]
                assert set(out[b * m + j]) == set(ref), (b, j)


# ---------------------------------------------------------------------------------------
# Calibration statistic (ADIndex §4.1, Eq. (4))
# ---------------------------------------------------------------------------------------

def test_union_sizes_hand_cases():
    same = [[5, 3, 1]] * 4
    disjoint = [[4 * i, 4 * i + 1, 4 * i + 2] for i in range(4)]
    padded = [[7, -1, -1], [7, 8, -1], [9, 8, 7], [-1, -1, -1]]
    assert ox.group_union_sizes(same, 4) == [3]
    assert ox.group_union_sizes(disjoint, 4) == [12]
    assert ox.group_union_sizes(disjoint, 2) == [6, 6]
    assert ox.group_union_sizes(padded, 2) == [2, 3]
    assert ox.group_union_sizes(padded + [[1, 2, 3]], 2) == [2, 3]   # incomplete group dropped


def test_union_sizes_bounds_and_monotonicity():
    rng = np.random.default_rng(42)
    K, T = 6, 32
    rows = [rng.choice(40, size=K, replace=False) for _ in range(T)]
    for G in (2, 4, 8):
        u = ox.group_union_sizes(rows, G)
        assert len(u) == T // G
        assert all(K <= x <= min(G * K, 40) for x in u)
    # a group of 2G contains two groups of G: its union is at least either of theirs
    u4, u8 = ox.group_union_sizes(rows, 4), ox.group_union_sizes(rows, 8)
    for g, x in enumerate(u8):
        assert x >= max(u4[2 * g], u4[2 * g + 1])


def test_bank_coverage_hand_cases():
    """A bank holding a query's whole Top-K covers it fully, a disjoint bank not at all,
    a bank with half of it one half; padding counts on neither side."""
    topk = [[3, 5, 7, 9], [3, 5, -1, -1], [1, 2, 4, 6], [0, 8, 10, 12]]
    banks = [[3, 5, 7, 9, 11, -1], [4, 6, 8, 10, 12, -1]]
    hits, count = ox.bank_coverage(topk, banks, 2)
    assert hits.tolist() == [4, 2, 2, 3]
    assert count.tolist() == [4, 2, 4, 4]
    # an incomplete trailing group has no bank and no coverage
    hits, count = ox.bank_coverage(topk[:3], banks[:1], 2)
    assert len(hits) == len(count) == 2


def test_bank_coverage_one_is_exact_recovery():
    """ADIndex §1: refinement over the bank recovers a query's full Top-K exactly when the bank
    holds all of it. On random problems, rows whose coverage (against the group's candidates:
    bank plus post-anchor positions) is 1 refine to the flat Top-K, and rows whose flat
    Top-K holds a key the candidates lack do not."""
    rng = np.random.default_rng(21)
    T, H, Hg, d, G, B, K = 96, 3, 2, 8, 8, 24, 6
    seen_full = seen_part = 0
    for trial in range(4):
        q, w, k = rng.normal(size=(T, H, d)), rng.random((T, H)), rng.normal(size=(T, d))
        qbar, wbar = rng.normal(size=(T // G, Hg, d)), rng.random((T // G, Hg))
        for mode in ("paper", "window"):
            plans = ox.plan_groups(T, 0, G, B, mode)
            flat = ox.flat_topk(q, w, k, np.arange(T), K)
            got, banks = ox.group_topk(q, w, k, qbar, wbar, 0, G, B, K, mode)
            rows, brows = [], []
            for gi, plan in enumerate(plans):
                if plan.kind != "bank":
                    continue
                cand = np.union1d(banks[gi], np.arange(plan.post_lo, plan.rows[-1] + 1))
                brows.append(cand)
                rows.extend(flat[t] for t in plan.rows)
            hits, count = ox.bank_coverage(rows, brows, G)
            members = [t for p in plans if p.kind == "bank" for t in p.rows]
            for j, t in enumerate(members):
                same = set(got[t].tolist()) == set(flat[t].tolist())
                if hits[j] == count[j]:
                    assert same, (mode, t)
                    seen_full += 1
                else:
                    assert not same, (mode, t)
                    seen_part += 1
    assert seen_full > 20 and seen_part > 20


def test_mean_pool_group_hand_values():
    q = np.zeros((5, 3, 2))
    w = np.zeros((5, 3))
    for i in range(5):
        q[i, :, 0] = i          # head-independent ramp
        q[i, 1, 1] = 10 * i
        w[i] = [1, 2, 3 + i]
    qbar, wbar = ox.mean_pool_group(q, w, 2, 2)
    assert qbar.shape == (2, 2, 2) and wbar.shape == (2, 2)   # trailing row 4 dropped
    assert qbar[:, 0, 0].tolist() == [0.5, 2.5]
    assert qbar[:, 1, 1].tolist() == [5.0, 25.0]
    assert wbar.tolist() == [[1, 2], [1, 2]]
    # G = 1 is the identity on the kept heads
    qb1, wb1 = ox.mean_pool_group(q, w, 1, 3)
    assert np.array_equal(qb1, q) and np.array_equal(wb1, w)


# ---------------------------------------------------------------------------------------
# Group indexer queries (ADIndex §4.2, Eqs. (6)-(7))
# ---------------------------------------------------------------------------------------

def test_rope_identity_norms_inverse_and_a_hand_value():
    rng = np.random.default_rng(43)
    x = rng.standard_normal(16)
    assert np.allclose(ox.rope(x, 0, 8), x)
    y = ox.rope(x, 37, 8)
    assert np.allclose(y[8:], x[8:])                       # beyond rope_dim: unchanged
    for i in range(4):                                     # each pair keeps its length
        assert np.isclose(np.hypot(y[2 * i], y[2 * i + 1]), np.hypot(x[2 * i], x[2 * i + 1]))
    assert np.allclose(ox.rope(y, -37, 8), x)             # rotating back recovers x
    e = np.zeros(4)
    e[0] = 1.0
    assert np.allclose(ox.rope(e, 1, 4)[:2], [np.cos(1.0), np.sin(1.0)])   # pair 0: angle = pos
    assert np.allclose(ox.rope(e[[1, 0, 2, 3]], 1, 4)[:2], [-np.sin(1.0), np.cos(1.0)])
    # pair i turns by pos * base^(-2i / rope_dim): pair 1 of a 4-dim rotary part at position 1
    # turns by 10000^(-1/2) = 0.01
    assert np.allclose(ox.rope(e[[2, 3, 0, 1]], 1, 4)[2:], [np.cos(0.01), np.sin(0.01)])


def test_group_indexer_pools_projects_and_gates():
    rng = np.random.default_rng(44)
    T, G, dc, dh, HS, d = 9, 4, 3, 5, 2, 4
    cq, h = rng.standard_normal((T, dc)), rng.standard_normal((T, dh))
    eye, zero = np.eye(dc), np.zeros((dc, dc))
    wq = np.zeros((HS * d, dc))
    wq[0:3, :] = np.eye(3)                                 # head 0, dims 0..2 <- c-bar
    for k, sel in enumerate(([eye, zero, zero], [zero, eye, zero], [zero, zero, eye])):
        qbar, wbar = ox.group_indexer_queries(cq, h, np.hstack(sel), wq, np.zeros((HS, dh)),
                                              G, HS, d, rope_dim=0)
        assert qbar.shape == (2, HS, d) and wbar.shape == (2, HS)   # trailing row dropped
        for g in range(2):
            members = cq[g * G:(g + 1) * G]
            want = (members.max(0), members.min(0), members.mean(0))[k]
            assert np.allclose(qbar[g, 0, :3], want)
        assert np.allclose(wbar, 0.5)                      # sigmoid(0)
    wg = np.zeros((HS, dh))
    wg[1, 2] = 1.0
    _, wbar = ox.group_indexer_queries(cq, h, np.hstack([eye, zero, zero]), wq, wg, G, HS, d,
                                       rope_dim=0)
    assert np.allclose(wbar[:, 1], 1 / (1 + np.exp(-np.array([h[0:4, 2].mean(), h[4:8, 2].mean()]))))
    # RoPE at each group's anchor position
    qb, _ = ox.group_indexer_queries(cq, h, np.hstack([eye, zero, zero]), wq, wg, G, HS, d,
                                     q_pos0=10, rope_dim=4)
    qn, _ = ox.group_indexer_queries(cq, h, np.hstack([eye, zero, zero]), wq, wg, G, HS, d,
                                     q_pos0=10, rope_dim=0)
    assert np.allclose(qb[1, 0], ox.rope(qn[1, 0], 14, 4))


# ---------------------------------------------------------------------------------------
# HISA (block filter + token refinement)
# ---------------------------------------------------------------------------------------

def test_hisa_block_keys_are_block_means():
    k = np.arange(10, dtype=np.float64)[:, None] * np.array([[1.0, -2.0]])   # ramp rows
    kbar = ox.hisa_block_keys(k, block=4)
    # block b holds rows 4b..4b+3 (mean 4b + 1.5); the partial block holds rows 8, 9 (8.5)
    assert np.allclose(kbar[:, 0], [1.5, 5.5, 8.5]) and np.allclose(kbar[:, 1], [-3, -11, -17])


def test_hisa_scores_pooled_keys_not_pooled_scores():
    """Block 1 holds +v and -v (pooled key 0: block score 0, although the mean of its token
    scores is 1.5); block 2 holds 0.5 v twice (block score 0.5). With one free slot the filter
    must take block 2."""
    k = np.zeros((12, 2))
    k[2], k[3] = [3.0, 0], [-3.0, 0]
    k[4], k[5] = [0.5, 0], [0.5, 0]
    q, w = np.array([[1.0, 0.0]]), np.array([1.0])
    kbar = ox.hisa_block_keys(k, block=2)
    assert list(ox.hisa_blocks_row(q, w, kbar, 11, n_blocks=3, block=2)) == [0, 2, 5]
    # the refined candidates are the tokens of those blocks up to the query's position
    assert list(ox.hisa_candidates([0, 2, 5], 10, 12, block=2)) == [0, 1, 4, 5, 10]


def test_hisa_forces_first_and_own_block():
    """Blocks 0 and the query's own block score lowest yet are kept and count toward the
    budget; the other slots go to the best-scoring blocks."""
    d, block = 3, 2
    scores = [-5.0, 4.0, 1.0, 3.0, 2.0, -6.0]       # desired block score of each block
    k = np.zeros((12, d))
    for b, s in enumerate(scores):
        k[2 * b:2 * b + 2, 0] = s
    q, w = np.array([[1.0, 0.0, 0.0]]), np.array([1.0])
    kbar = ox.hisa_block_keys(k, block)
    assert list(ox.hisa_blocks_row(q, w, kbar, 10, n_blocks=4, block=block)) == [0, 1, 3, 5]
    # query in block 0: only one forced block; all visible when they fit
    assert list(ox.hisa_blocks_row(q, w, kbar, 1, n_blocks=4, block=block)) == [0]
    assert list(ox.hisa_blocks_row(q, w, kbar, 7, n_blocks=4, block=block)) == [0, 1, 2, 3]


def test_hisa_equals_flat_indexer_when_every_block_fits():
    rng = np.random.default_rng(45)
    T, S, H, d = 24, 24, 3, 5
    q, w, k = rng.standard_normal((T, H, d)), rng.random((T, H)), rng.standard_normal((S, d))
    pos = np.arange(T)
    got = ox.hisa_topk(q, w, k, pos, K=5, n_blocks=6, block=4)
    want = ox.flat_topk(q, w, k, pos, K=5)
    for t in range(T):
        assert set(got[t]) == set(want[t])


def test_hisa_matches_brute_force_subsets():
    """Top-m of distinct scores is the m-subset with the largest sum: brute force over all
    block subsets (forced blocks included) and then over all K-subsets of the candidates."""
    rng = np.random.default_rng(46)
    H, d, block, n_blocks, K = 2, 3, 3, 4, 4
    S = 7 * block
    k = rng.standard_normal((S, d))
    for trial in range(6):
        q, w = rng.standard_normal((H, d)), rng.random(H)
        p = int(rng.integers(5 * block, S))
        cur, nb = p // block, p // block + 1
        kbar = np.stack([k[b * block:(b + 1) * block].mean(0) for b in range(nb)])
        bs = [sum(w[j] * max(0.0, q[j] @ kbar[b]) for j in range(H)) for b in range(nb)]
        others = [b for b in range(nb) if b not in (0, cur)]
        best = max(itertools.combinations(others, n_blocks - 2), key=lambda c: sum(bs[b] for b in c))
        blocks = sorted(set(best) | {0, cur})
        assert list(ox.hisa_blocks_row(q, w, ox.hisa_block_keys(k, block), p, n_blocks,
                                       block)) == blocks
        cand = [s for b in blocks for s in range(b * block, (b + 1) * block) if s <= p]
        ts = {s: sum(w[j] * max(0.0, q[j] @ k[s]) for j in range(H)) for s in cand}
        top = max(itertools.combinations(cand, K), key=lambda c: sum(ts[s] for s in c))
        got = ox.hisa_topk(q[None], w[None], k, [p], K, n_blocks, block)[0]
        assert set(got) == set(top)


def test_hisa_short_prefix_keeps_every_token():
    rng = np.random.default_rng(47)
    q, w, k = rng.standard_normal((1, 2, 3)), rng.random((1, 2)), rng.standard_normal((40, 3))
    assert list(ox.hisa_topk(q, w, k, [9], K=10, n_blocks=2, block=4)[0]) == list(range(10))
