"""Mistakes planted in the oracle are caught by its pins.

Each case below is a copy of one oracle function carrying one plausible mistake (a dropped
term, a wrong sign or bias, an index off by one, a reversed order, a missing scale). The test
puts the copy in place of the function for its own duration, runs the pins named beside it
(tests of this directory that compare the oracle with facts from outside it: the pages'
worked values and Table 5, closed forms, brute force, library routines) and requires at
least one of them to fail. A pin set that let a case through would mean the pins cannot
tell that mistake from the pages' arithmetic.

The mistakes are made on the CPU, in the oracle only; nothing here touches a GPU.
"""

import numpy as np
import pytest

from oracle import cost_model, fp_formats
from oracle import indexer as ox

import test_calibration as tc
import test_oracle_pins as tp


# ---------------------------------------------------------------------------------------
# planted mistakes (each differs from the oracle function it replaces in one place)
# ---------------------------------------------------------------------------------------

def score_no_relu(q_t, w_t, keys):  # Eq. (1) without the ReLU
    keys = np.asarray(keys, np.float64)
    if keys.shape[0] == 0:
        return np.zeros(0)
    return np.asarray(w_t, np.float64) @ (np.asarray(q_t, np.float64) @ keys.T)


def score_relu_after_gate(q_t, w_t, keys):  # the ReLU taken of the gated sum
    keys = np.asarray(keys, np.float64)
    if keys.shape[0] == 0:
        return np.zeros(0)
    return np.maximum(np.asarray(w_t, np.float64) @ (np.asarray(q_t, np.float64) @ keys.T), 0.0)


def score_no_gate(q_t, w_t, keys):  # the heads summed without their gates
    keys = np.asarray(keys, np.float64)
    if keys.shape[0] == 0:
        return np.zeros(0)
    return np.maximum(np.asarray(q_t, np.float64) @ keys.T, 0.0).sum(axis=0)


def score_scaled(q_t, w_t, keys):  # an attention-style 1/sqrt(d) the equation does not have
    keys = np.asarray(keys, np.float64)
    if keys.shape[0] == 0:
        return np.zeros(0)
    logits = np.asarray(q_t, np.float64) @ keys.T / np.sqrt(keys.shape[1])
    return np.asarray(w_t, np.float64) @ np.maximum(logits, 0.0)


def scores_strictly_causal(q, w, k, pos):  # the query's own position hidden
    T, S = q.shape[0], k.shape[0]
    out = np.full((T, S), -np.inf)
    for t in range(T):
        n = min(int(pos[t]), S)
        out[t, :n] = ox.score_keys(q[t], w[t], k[:n])
    return out


def flat_row_strictly_causal(q_t, w_t, k, p, K):
    n = min(int(p), k.shape[0])
    return ox.topk(ox.score_keys(q_t, w_t, k[:n]), K)


def topk_ties_descending(scores, K, positions=None):  # ties to the highest position
    scores = np.asarray(scores, np.float64)
    positions = np.arange(scores.shape[0]) if positions is None else np.asarray(positions, np.int64)
    order = np.lexsort((-positions, -scores))
    return positions[order[: min(int(K), scores.shape[0])]]


def topk_lowest(scores, K, positions=None):  # the K lowest scores
    scores = np.asarray(scores, np.float64)
    positions = np.arange(scores.shape[0]) if positions is None else np.asarray(positions, np.int64)
    order = np.lexsort((positions, scores))
    return positions[order[: min(int(K), scores.shape[0])]]


def topk_one_short(scores, K, positions=None):  # K - 1 kept
    scores = np.asarray(scores, np.float64)
    positions = np.arange(scores.shape[0]) if positions is None else np.asarray(positions, np.int64)
    order = np.lexsort((positions, -scores))
    return positions[order[: max(0, min(int(K), scores.shape[0]) - 1)]]


def _plan_with(window_scan=None, window_bank=None, paper_scan=None, paper_post=None,
               paper_short=None):
    """plan_groups with one of its terms replaced."""
    def plan(T, q_pos0, G, B, mode, fallback="group"):
        plans = []
        whole_window_flat = fallback == "window" and (q_pos0 + 1) <= B
        for g0 in range(0, T, G):
            rows = tuple(range(g0, min(g0 + G, T)))
            a = q_pos0 + g0
            incomplete = len(rows) < G
            if mode == "paper":
                fb = (paper_short or (lambda a, B: (a + 1) <= B))(a, B)
                short = fb if fallback == "group" else whole_window_flat
                if incomplete or short:
                    plans.append(ox.GroupPlan("flat", rows, a))
                else:
                    plans.append(ox.GroupPlan(
                        "bank", rows, a, scan_n=(paper_scan or (lambda a: a + 1))(a), bank_k=B,
                        post_lo=(paper_post or (lambda a: a + 1))(a)))
            else:
                if incomplete or whole_window_flat:
                    plans.append(ox.GroupPlan("flat", rows, a))
                else:
                    plans.append(ox.GroupPlan(
                        "bank", rows, a, scan_n=(window_scan or (lambda a: a))(a),
                        bank_k=(window_bank or (lambda B, G: B - G))(B, G), post_lo=a))
        return plans
    return plan


def refine_bank_only(q_i, w_i, k, bank, post_lo, p_i, K):  # post-anchor positions dropped
    cand = np.asarray(bank, np.int64)
    cand = np.unique(cand[cand <= p_i])
    return ox.topk(ox.score_keys(q_i, w_i, k[cand]), K, positions=cand)


def refine_without_self(q_i, w_i, k, bank, post_lo, p_i, K):  # the query's own position lost
    cand = np.union1d(np.asarray(bank, np.int64), np.arange(post_lo, int(p_i) + 1))
    cand = cand[cand < p_i]
    return ox.topk(ox.score_keys(q_i, w_i, k[cand]), K, positions=cand)


def bank_one_short(qbar_g, wbar_g, k, plan):  # Top-(B - 1) kept in the bank
    n = min(plan.scan_n, k.shape[0])
    return ox.topk(ox.score_keys(qbar_g, wbar_g, k[:n]), plan.bank_k - 1)


def e4m3_bias_8(codes):  # exponent bias 8 instead of 7
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = sign * np.where(e == 0, (m / 8.0) * np.exp2(1.0 - 8.0),
                          (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 8.0))
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)


def e4m3_no_subnormals(codes):  # exponent field 0 read as a normal number
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = sign * (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)


def bf16_low_half(bits):  # the code placed in the low half of the binary32
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32)
    return b.view(np.float32).astype(np.float64)


def dequantize_divides(codes, scale, dtype):  # the per-row scale divided instead of multiplied
    if dtype == "bf16":
        return fp_formats.bf16_bits_to_f64(codes)
    v = fp_formats.e4m3_to_f64(codes)
    s = np.asarray(scale, dtype=np.float32).astype(np.float64)
    return v / s.reshape(s.shape + (1,) * (v.ndim - s.ndim))


def mean_pool_sums(q, w, G, Hg):  # member sums, not means
    q, w = np.asarray(q, np.float64), np.asarray(w, np.float64)
    ng = q.shape[0] // G
    qbar = np.stack([q[g * G:(g + 1) * G, :Hg].sum(0) for g in range(ng)])
    wbar = np.stack([w[g * G:(g + 1) * G, :Hg].sum(0) for g in range(ng)])
    return qbar, wbar


def mean_pool_shifted(q, w, G, Hg):  # groups one row late
    q, w = np.asarray(q, np.float64), np.asarray(w, np.float64)
    ng = q.shape[0] // G
    qbar = np.stack([q[min(g * G + 1, q.shape[0] - G):][:G, :Hg].mean(0) for g in range(ng)])
    wbar = np.stack([w[min(g * G + 1, w.shape[0] - G):][:G, :Hg].mean(0) for g in range(ng)])
    return qbar, wbar


def union_counts_padding(topk_rows, G):  # -1 padding counted as an index
    rows = [set(int(x) for x in np.asarray(r).ravel()) for r in topk_rows]
    return [len(set().union(*rows[g0:g0 + G])) for g0 in range(0, len(rows) - G + 1, G)]


def union_one_row_short(topk_rows, G):  # the union of G - 1 members
    rows = [set(int(x) for x in np.asarray(r).ravel() if int(x) >= 0) for r in topk_rows]
    return [len(set().union(*rows[g0:g0 + G - 1])) for g0 in range(0, len(rows) - G + 1, G)]


_bank_coverage = ox.bank_coverage


def coverage_counts_K(topk_rows, bank_rows, G):  # |T_i| taken as the row width
    hits, count = _bank_coverage(topk_rows, bank_rows, G)
    return hits, np.full_like(count, np.asarray(topk_rows[0]).size)


def rope_reversed(x, pos, rope_dim=64, base=10000.0):  # rotated the other way
    y = np.array(x, dtype=np.float64)
    for i in range(rope_dim // 2):
        a = -pos * base ** (-2.0 * i / rope_dim)
        c, s = np.cos(a), np.sin(a)
        x0, x1 = y[2 * i], y[2 * i + 1]
        y[2 * i], y[2 * i + 1] = x0 * c - x1 * s, x0 * s + x1 * c
    return y


def rope_frequency_off(x, pos, rope_dim=64, base=10000.0):  # frequencies over d/2, not rope_dim/2
    y = np.array(x, dtype=np.float64)
    for i in range(rope_dim // 2):
        a = pos * base ** (-1.0 * i / rope_dim)
        c, s = np.cos(a), np.sin(a)
        x0, x1 = y[2 * i], y[2 * i + 1]
        y[2 * i], y[2 * i + 1] = x0 * c - x1 * s, x0 * s + x1 * c
    return y


def block_keys_max(k, block=ox.HISA_BLOCK):  # max pooling instead of mean
    k = np.asarray(k, np.float64)
    nb = -(-k.shape[0] // block)
    return np.stack([k[b * block:(b + 1) * block].max(axis=0) for b in range(nb)])


def hisa_blocks_not_forced(q_t, w_t, kbar, p, n_blocks, block=ox.HISA_BLOCK):  # no forced blocks
    cur = int(p) // block
    nvis = min(cur + 1, kbar.shape[0])
    if nvis <= n_blocks:
        return np.arange(nvis)
    rest = np.arange(nvis)
    return np.sort(ox.topk(ox.score_keys(q_t, w_t, kbar[rest]), n_blocks, rest))


def hisa_candidates_past_query(blocks, p, S, block=ox.HISA_BLOCK):  # the own block not masked
    parts = [np.arange(b * block, min((b + 1) * block, S)) for b in blocks]
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def plan_cost_no_post(plans, q_pos0):  # the post-anchor keys not counted
    total = 0
    for p in plans:
        pos = [q_pos0 + r for r in p.rows]
        if p.kind == "flat":
            total += sum(x + 1 for x in pos)
        else:
            total += p.scan_n + sum(min(p.bank_k, p.scan_n) for _ in pos)
    return total


def group_indexer_no_min(cq, h, w_pool, w_q, w_g, G, H_S, d, q_pos0=0, rope_dim=64,
                         base=10000.0):  # the min pooling term replaced by a second max
    cq, h = np.asarray(cq, np.float64), np.asarray(h, np.float64)
    ng = cq.shape[0] // G
    qbar, wbar = np.zeros((ng, H_S, d)), np.zeros((ng, H_S))
    for g in range(ng):
        c = cq[g * G:(g + 1) * G]
        cbar = np.asarray(w_pool, np.float64) @ np.concatenate([c.max(0), c.max(0), c.mean(0)])
        qpre = (np.asarray(w_q, np.float64) @ cbar).reshape(H_S, d)
        for j in range(H_S):
            qbar[g, j] = ox.rope(qpre[j], q_pos0 + g * G, rope_dim, base)
        z = np.asarray(w_g, np.float64) @ h[g * G:(g + 1) * G].mean(0)
        wbar[g] = 1.0 / (1.0 + np.exp(-z))
    return qbar, wbar


def group_indexer_rope_at_zero(cq, h, w_pool, w_q, w_g, G, H_S, d, q_pos0=0, rope_dim=64,
                               base=10000.0):  # RoPE at position 0 instead of the anchor
    return ox_group_indexer_queries(cq, h, w_pool, w_q, w_g, G, H_S, d, q_pos0, rope_dim, base,
                                    anchor_pos=lambda g: 0)


def ox_group_indexer_queries(cq, h, w_pool, w_q, w_g, G, H_S, d, q_pos0, rope_dim, base,
                             anchor_pos):
    cq, h = np.asarray(cq, np.float64), np.asarray(h, np.float64)
    ng = cq.shape[0] // G
    qbar, wbar = np.zeros((ng, H_S, d)), np.zeros((ng, H_S))
    for g in range(ng):
        c = cq[g * G:(g + 1) * G]
        cbar = np.asarray(w_pool, np.float64) @ np.concatenate([c.max(0), c.min(0), c.mean(0)])
        qpre = (np.asarray(w_q, np.float64) @ cbar).reshape(H_S, d)
        for j in range(H_S):
            qbar[g, j] = ox.rope(qpre[j], anchor_pos(g), rope_dim, base)
        z = np.asarray(w_g, np.float64) @ h[g * G:(g + 1) * G].mean(0)
        wbar[g] = 1.0 / (1.0 + np.exp(-z))
    return qbar, wbar


def decode_refine_from_anchor(q, w, caches, seq_len, banks, anchors, K):  # post-anchor keys from a
    return {b: ox.refine_row(q[b], w[b], caches[b], banks[b], int(anchors[b]),
                             int(seq_len[b]) - 1, K) for b in range(q.shape[0])}


def decode_bank_without_anchor(qbar, wbar, caches, seq_len, B):  # the anchor's own key not scanned
    return {b: ox.token_bank(qbar[b], wbar[b], caches[b],
                             ox.GroupPlan("bank", (b,), int(seq_len[b]) - 1,
                                          scan_n=int(seq_len[b]) - 1, bank_k=B))
            for b in range(qbar.shape[0])}


_group_topk = ox.group_topk


def mtp_one_late(q, w, caches, qbar, wbar, seq_len, m, G, P, K):  # window placed one position late
    out = {}
    gps = m // G
    for b in range(len(caches)):
        res, _ = _group_topk(q[b * m:(b + 1) * m], w[b * m:(b + 1) * m], caches[b],
                             qbar[b * gps:(b + 1) * gps], wbar[b * gps:(b + 1) * gps],
                             int(seq_len[b]) - m + 1, G, P, K, "paper", fallback="window")
        for j, v in res.items():
            out[b * m + j] = v
    return out


def group_topk_first_query(q, w, k, qbar, wbar, q_pos0, G, B, K, mode, rows=None,
                           fallback="group"):  # every group's bank from group 0's query
    out, banks = {}, {}
    for gi, plan in enumerate(ox.plan_groups(q.shape[0], q_pos0, G, B, mode, fallback)):
        todo = [t for t in plan.rows if rows is None or t in set(int(r) for r in rows)]
        if not todo:
            continue
        if plan.kind == "flat":
            for t in todo:
                out[t] = ox.flat_topk_row(q[t], w[t], k, q_pos0 + t, K)
            continue
        bank = ox.token_bank(qbar[0], wbar[0], k, plan)
        banks[gi] = bank
        for t in todo:
            out[t] = ox.refine_row(q[t], w[t], k, bank, plan.post_lo, q_pos0 + t, K)
    return out, banks


_hisa_topk_row = ox.hisa_topk_row


def hisa_short_prefix_strict(q_t, w_t, k, kbar, p, K, n_blocks, block=ox.HISA_BLOCK):
    S = k.shape[0]  # a prefix of exactly K tokens sent through the block filter
    if int(p) + 1 < K:
        return np.arange(min(int(p) + 1, S))
    cand = ox.hisa_candidates(ox.hisa_blocks_row(q_t, w_t, kbar, p, n_blocks, block), p, S, block)
    return ox.topk(ox.score_keys(q_t, w_t, k[cand]), K, cand)


def decode_topk_one_early(q, w, caches, seq_len, K):  # the row placed at seq_len - 2
    return {b: ox.flat_topk_row(q[b], w[b], caches[b], int(seq_len[b]) - 2, K)
            for b in range(q.shape[0])}


def base_cost_no_self(T, q_pos0):  # the plain indexer's own-position score not counted
    return sum(q_pos0 + t for t in range(T))


def mtp_round_cost_late(N, G, P, m=16, mode="paper"):  # the window's first query sees N + 1 keys
    return cost_model.plan_cost(ox.plan_groups(m, N, G, P, mode, fallback="window"), N)


_base_cost, _prefill_cost, _mtp_round_cost = (cost_model.base_cost, cost_model.prefill_cost,
                                              cost_model.mtp_round_cost)


def speedups_rounds_from_one(L, G, P, R=32, m=16, a=8):  # round j's prefix L + j a, not L + (j-1) a
    pre_b, pre_r = _base_cost(L, 0), _prefill_cost(L, G, P)
    jb, jr = pre_b, pre_r
    for j in range(1, R + 1):
        n = L + j * a
        jb += _base_cost(m, n - 1)
        jr += _mtp_round_cost(n, G, P, m)
    return pre_b / pre_r, _base_cost(m, L - 1) / _mtp_round_cost(L, G, P, m), jb / jr


# (module, attribute, planted mistake, pins that must catch it)
CASES = [
    ("score: no ReLU", ox, "score_keys", score_no_relu,
     [tp.test_score_hand_values, tp.test_score_all_negative_logits_is_zero]),
    ("score: ReLU of the gated sum", ox, "score_keys", score_relu_after_gate,
     [tp.test_score_negative_gate_keeps_relu_per_head]),
    ("score: gates dropped", ox, "score_keys", score_no_gate,
     [tp.test_score_hand_values, tp.test_score_positive_scales_factor_out]),
    ("score: 1/sqrt(d) added", ox, "score_keys", score_scaled,
     [tp.test_score_hand_values, tp.test_score_single_head_unit_gate_is_dot_product]),
    ("scores: own position hidden", ox, "indexer_scores", scores_strictly_causal,
     [tp.test_indexer_scores_causal_mask]),
    ("flat Top-K: own position hidden", ox, "flat_topk_row", flat_row_strictly_causal,
     [tp.test_flat_topk_causal_counts]),
    ("Top-K: ties to the highest position", ox, "topk", topk_ties_descending,
     [tp.test_topk_matches_stable_argsort_with_ties]),
    ("Top-K: lowest scores", ox, "topk", topk_lowest,
     [tp.test_topk_brute_force_small]),
    ("Top-K: one short", ox, "topk", topk_one_short,
     [tp.test_topk_brute_force_small, tp.test_flat_topk_causal_counts]),
    ("window bank: scan includes the anchor", ox, "plan_groups", _plan_with(window_scan=lambda a: a + 1),
     [tp.test_window_group_cost_closed_form, tp.test_window_bank_holds_the_anchor_through_the_window_not_the_scan]),
    ("window bank: B scan keys", ox, "plan_groups", _plan_with(window_bank=lambda B, G: B),
     [tp.test_window_group_cost_closed_form, tp.test_window_bank_keeps_exactly_B_minus_G_scan_keys]),
    ("paper bank: anchor not scanned", ox, "plan_groups", _plan_with(paper_scan=lambda a: a),
     [tp.test_group_cost_matches_eq17, tp.test_table5_reproduced_by_the_group_plan]),
    ("paper fallback: strict inequality", ox, "plan_groups",
     _plan_with(paper_short=lambda a, B: (a + 1) < B), [tp.test_paper_fallback_rule]),
    ("refinement: post-anchor keys dropped", ox, "refine_row", refine_bank_only,
     [tp.test_refine_exact_recovery_when_bank_holds_topk, tp.test_decode_bank_reuse_matches_definitions]),
    ("refinement: own position dropped", ox, "refine_row", refine_without_self,
     [tp.test_refine_exact_recovery_when_bank_holds_topk, tp.test_candidates_stay_causal_and_in_bank]),
    ("bank: Top-(B-1)", ox, "token_bank", bank_one_short,
     [tp.test_decode_bank_reuse_matches_definitions, tp.test_window_bank_keeps_exactly_B_minus_G_scan_keys]),
    ("e4m3: bias 8", fp_formats, "e4m3_to_f64", e4m3_bias_8,
     [tp.test_e4m3_decode_matches_torch_on_every_code]),
    ("e4m3: no subnormals", fp_formats, "e4m3_to_f64", e4m3_no_subnormals,
     [tp.test_e4m3_decode_matches_torch_on_every_code]),
    ("bf16: low half", fp_formats, "bf16_bits_to_f64", bf16_low_half,
     [tp.test_bf16_decode_matches_torch_on_every_code]),
    ("dequantise: scale divided", fp_formats, "dequantize", dequantize_divides,
     [tp.test_dequantize_applies_per_row_scale]),
    ("group query: sums, not means", ox, "mean_pool_group", mean_pool_sums,
     [tp.test_mean_pool_group_hand_values]),
    ("group query: groups one row late", ox, "mean_pool_group", mean_pool_shifted,
     [tp.test_mean_pool_group_hand_values]),
    ("union sizes: padding counted", ox, "group_union_sizes", union_counts_padding,
     [tp.test_union_sizes_hand_cases]),
    ("union sizes: G - 1 members", ox, "group_union_sizes", union_one_row_short,
     [tp.test_union_sizes_hand_cases, tp.test_union_sizes_bounds_and_monotonicity]),
    ("coverage: divided by the row width", ox, "bank_coverage", coverage_counts_K,
     [tp.test_bank_coverage_hand_cases]),
    ("RoPE: reversed rotation", ox, "rope", rope_reversed,
     [tp.test_rope_identity_norms_inverse_and_a_hand_value]),
    ("RoPE: frequencies off", ox, "rope", rope_frequency_off,
     [tp.test_rope_identity_norms_inverse_and_a_hand_value]),
    ("group indexer: min pooling lost", ox, "group_indexer_queries", group_indexer_no_min,
     [tp.test_group_indexer_pools_projects_and_gates]),
    ("group indexer: RoPE at 0", ox, "group_indexer_queries", group_indexer_rope_at_zero,
     [tp.test_group_indexer_pools_projects_and_gates]),
    ("HISA: max-pooled block keys", ox, "hisa_block_keys", block_keys_max,
     [tp.test_hisa_block_keys_are_block_means]),
    ("HISA: first and own block not forced", ox, "hisa_blocks_row", hisa_blocks_not_forced,
     [tp.test_hisa_forces_first_and_own_block]),
    ("HISA: own block past the query", ox, "hisa_candidates", hisa_candidates_past_query,
     [tp.test_hisa_short_prefix_keeps_every_token, tp.test_hisa_matches_brute_force_subsets]),
    ("decode refinement: post-anchor keys from the anchor", ox, "decode_refine",
     decode_refine_from_anchor, [tp.test_decode_bank_reuse_matches_definitions]),
    ("decode bank: anchor not scanned", ox, "decode_bank", decode_bank_without_anchor,
     [tp.test_decode_bank_reuse_matches_definitions]),
    ("MTP: window one position late", ox, "mtp_topk", mtp_one_late,
     [tp.test_mtp_window_fallback_is_flat_even_past_the_budget, tp.test_mtp_banked_window_matches_the_equations]),
    ("group mode: group 0's query for every bank", ox, "group_topk", group_topk_first_query,
     [tp.test_candidates_stay_causal_and_in_bank, tp.test_mtp_banked_window_matches_the_equations]),
    ("HISA: a prefix of K tokens filtered", ox, "hisa_topk_row", hisa_short_prefix_strict,
     [tp.test_hisa_short_prefix_keeps_every_token, tp.test_hisa_matches_brute_force_subsets]),
    ("decode: row one position early", ox, "decode_topk", decode_topk_one_early,
     [tp.test_decode_bank_reuse_matches_definitions]),
    ("cost: own position not counted", cost_model, "base_cost", base_cost_no_self,
     [tp.test_cost_closed_forms_of_appendix_a, tp.test_table5_reproduced_by_the_group_plan, tc.test_speedup_reproduces_table5_panel_c]),
    ("cost: MTP window one key late", cost_model, "mtp_round_cost", mtp_round_cost_late,
     [tp.test_cost_closed_forms_of_appendix_a, tp.test_table5_reproduced_by_the_group_plan, tc.test_speedup_reproduces_table5_panel_c]),
    ("cost: MTP rounds from L + a", cost_model, "speedups", speedups_rounds_from_one,
     [tp.test_cost_closed_forms_of_appendix_a, tp.test_table5_reproduced_by_the_group_plan, tc.test_speedup_reproduces_table5_panel_c]),
    ("cost: post-anchor keys not counted", cost_model, "plan_cost", plan_cost_no_post,
     [tp.test_table5_reproduced_by_the_group_plan, tc.test_speedup_reproduces_table5_panel_c]),
]


def _fails(pin):
    try:
        pin()
    except (AssertionError, ValueError, IndexError, TypeError):
        return True
    return False


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_planted_mistake_is_caught(case, monkeypatch):
    _, module, attr, mutant, pins = case
    assert callable(getattr(module, attr))
    monkeypatch.setattr(module, attr, mutant)
    if module is ox and attr == "plan_groups":  # the cost model holds its own reference
        monkeypatch.setattr(cost_model, "plan_groups", mutant)
    assert any(_fails(pin) for pin in pins), "no pin caught the planted mistake"


def test_pins_pass_on_the_oracle_as_it_stands():
    """The same pins with nothing planted (the control for every case above)."""
    pins = {p for case in CASES for p in case[4]}
    failing = [p.__name__ for p in pins if _fails(p)]
    assert failing == []
