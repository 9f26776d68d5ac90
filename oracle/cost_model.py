"""Score-evaluation counts of the group procedure (oracle; test infrastructure only).

ADIndex (arXiv 2611.12956v1), Appendix A counts one unit per (query, key) score, for the
plain indexer and for the group indexer alike. The counts here are taken from the same
``plan_groups`` objects that ``oracle.indexer.group_topk`` executes, so reproducing the
paper's Table 5 pins which pairs the procedure scores: the scan range, the bank size and
the post-anchor positions of every member.
"""

from .indexer import plan_groups


def plan_cost(plans, q_pos0):
    """Total score evaluations of an executed plan.

    flat group:  each member i scores its whole prefix, pos_i + 1 keys (Eq. (15)/(16) terms)
    bank group:  one scan of scan_n keys, then member i scores
                 min(bank_k, scan_n) bank entries + (pos_i - post_lo + 1) post-anchor keys
                 (Eq. (17) and the per-group terms of Eq. (20)).
    """
    total = 0
    for p in plans:
        pos = [q_pos0 + r for r in p.rows]
        if p.kind == "flat":
            total += sum(x + 1 for x in pos)
        else:
            total += p.scan_n
            total += sum(min(p.bank_k, p.scan_n) + max(0, x - p.post_lo + 1) for x in pos)
    return total


def base_cost(T, q_pos0):
    """Plain indexer over T queries at positions q_pos0 .. q_pos0+T-1 (Eqs. (15)-(16))."""
    return sum(q_pos0 + t + 1 for t in range(T))


def prefill_cost(L, G, P, mode="paper"):
    """Reuse cost of prefilling L tokens with group size G and bank budget P."""
    return plan_cost(plan_groups(L, 0, G, P, mode, fallback="group"), 0)


def mtp_round_cost(N, G, P, m=16, mode="paper"):
    """Reuse cost of one verification window of m queries whose first query sees N keys
    (window-level fallback; Appendix A.2, Eqs. (20)-(21))."""
    return plan_cost(plan_groups(m, N - 1, G, P, mode, fallback="window"), N - 1)


def speedups(L, G, P, R=32, m=16, a=8):
    """Table 5's three speedups at prefill length L (Appendix A.3-A.4, Eqs. (23)-(24), (28)).

    (a) prefill: base / reuse over the L prefill queries;
    (b) one MTP round whose first query sees L keys;
    (c) prefill plus R rounds of m queries, round j's first query seeing L + (j-1) a keys.
    """
    pre_b, pre_r = base_cost(L, 0), prefill_cost(L, G, P)
    mtp_b = base_cost(m, L - 1)
    mtp_r = mtp_round_cost(L, G, P, m)
    jb, jr = pre_b, pre_r
    for j in range(1, R + 1):
        n = L + (j - 1) * a
        jb += base_cost(m, n - 1)
        jr += mtp_round_cost(n, G, P, m)
    return pre_b / pre_r, mtp_b / mtp_r, jb / jr
