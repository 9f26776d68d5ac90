"""fp64 oracle of the indexer hot path (test infrastructure only; see the package header).

Everything here follows "ADIndex: Layer-Adaptive Sparse Attention Indexing via Group-Level
Distillation" (arXiv 2611.12956v1), cited as "ADIndex" with section and equation. All
arrays are float64 real values (operand codes are decoded by ``oracle.fp_formats`` first);
positions are absolute token positions (0-based).

Readings taken where the page is garbled or silent (each one is also listed in the design
notes of the repository):
  * Eq. (1): the gate w multiplies ReLU(q.k) per head and the heads are summed; no 1/sqrt(d)
    or other scale appears, so none is applied. w may have any sign.
  * Causal visibility includes the query's own position: key s is visible to a query at
    position p iff s <= p.
  * Top-K ties are broken by ascending position; rows with fewer than K visible keys return
    all of them. Results are sets; order carries no meaning.
  * Group mode has two readings of the bank (Eq. 13) and the candidate set (Eq. 14):
      "paper"  - anchor a = the group's first query; scan s <= a; bank = Top-B; query i adds
                 the post-anchor positions a+1..i. Groups with a + 1 <= B and incomplete
                 trailing groups use the plain indexer (§4.3 "Shared Token Bank
                 Construction" and "Application to Prefill and MTP").
      "window" - scan s < a; bank = Top-(B-G) of the scan plus the group's own window
                 a..a+G-1 (total B); query i's candidates are the bank entries <= i.
                 Incomplete trailing groups use the plain indexer.
  * HISA (the HISA paper's abstract; ADIndex Appendix C.5 for its settings): a block is
    scored with Eq. (1) applied to its mean-pooled key (pooling keys, not token scores); the
    query's own block is visible (its tokens up to the query's position); a trailing partial
    block pools the keys it holds; the forced blocks take budget slots first and the other
    slots follow the block scores with ties broken by ascending block number.
"""

from dataclasses import dataclass

import numpy as np


# ---------------------------------------------------------------------------------------
# Eq. (1) and Eq. (2)
# ---------------------------------------------------------------------------------------

def score_keys(q_t, w_t, keys):
    """ADIndex §3, Eq. (1) for one query against an explicit list of key vectors.

    q_t [H, d], w_t [H], keys [n, d]  ->  I [n] with I[s] = sum_j w_t[j] * max(0, q_t[j] . keys[s]).
    """
    q_t = np.asarray(q_t, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    if keys.shape[0] == 0:
        return np.zeros(0)
    logits = q_t @ keys.T                     # [H, n], one dot product per (head, key)
    return np.asarray(w_t, dtype=np.float64) @ np.maximum(logits, 0.0)


def indexer_scores(q, w, k, pos):
    """Eq. (1) over the causal prefix of every query: I [T, S], -inf where s > pos[t].

    q [T, H, d], w [T, H], k [S, d], pos [T] (absolute position of each query row).
    """
    T, S = q.shape[0], k.shape[0]
    out = np.full((T, S), -np.inf)
    for t in range(T):
        n = min(int(pos[t]) + 1, S)
        out[t, :n] = score_keys(q[t], w[t], k[:n])
    return out


def topk(scores, K, positions=None):
    """ADIndex §3, Eq. (2): the min(K, n) highest-scoring candidates.

    ``scores`` [n] are candidate scores, ``positions`` [n] their key positions (defaults to
    0..n-1). Order: score descending, then position ascending. Returns positions, in that
    order.
    """
    scores = np.asarray(scores, dtype=np.float64)
    if positions is None:
        positions = np.arange(scores.shape[0])
    positions = np.asarray(positions, dtype=np.int64)
    if not np.all(np.isfinite(scores)):
        raise ValueError("oracle requires finite scores")
    order = np.lexsort((positions, -scores))
    return positions[order[: min(int(K), scores.shape[0])]]


def flat_topk_row(q_t, w_t, k, p, K):
    """Plain DSA indexer for one query at position p: Top-K over keys s <= p (Eqs. 1-2)."""
    n = min(int(p) + 1, k.shape[0])
    return topk(score_keys(q_t, w_t, k[:n]), K)


def flat_topk(q, w, k, pos, K, rows=None):
    """Plain DSA indexer: {row: Top-K positions} for the requested rows (all by default)."""
    rows = range(q.shape[0]) if rows is None else rows
    return {int(t): flat_topk_row(q[t], w[t], k, pos[t], K) for t in rows}


# ---------------------------------------------------------------------------------------
# Group plan: which keys each stage of the group procedure scores (§4.3, Appendix A.2)
# ---------------------------------------------------------------------------------------

@dataclass(frozen=True)
class GroupPlan:
    """One query group of the procedure.

    kind      "bank" (shared bank + refinement) or "flat" (plain indexer for every member)
    rows      query rows of the members (consecutive)
    anchor    position of the first member
    scan_n    keys scanned by the group query: positions 0..scan_n-1
    bank_k    size of the scan Top-K kept in the bank
    post_lo   first position added to every member i's candidates (post_lo..pos_i)
    """
    kind: str
    rows: tuple
    anchor: int
    scan_n: int = 0
    bank_k: int = 0
    post_lo: int = 0


def plan_groups(T, q_pos0, G, B, mode, fallback="group"):
    """Split T query rows (row t at position q_pos0 + t) into consecutive groups of G.

    mode      "paper" or "window" (see the module header)
    fallback  "group":  prefill rule - a group falls back when its anchor's visible prefix
                        a + 1 does not exceed the budget B, or when it is incomplete
                        (ADIndex §4.3, "Application to Prefill and MTP").
              "window": MTP rule - the whole window falls back when the first query's
                        visible prefix q_pos0 + 1 does not exceed B (§4.3 and Appendix A.2,
                        "Bank Sharing During MTP Target Verification").
    """
    if mode not in ("paper", "window"):
        raise ValueError(mode)
    plans = []
    whole_window_flat = fallback == "window" and (q_pos0 + 1) <= B
    for g0 in range(0, T, G):
        rows = tuple(range(g0, min(g0 + G, T)))
        a = q_pos0 + g0
        incomplete = len(rows) < G
        if mode == "paper":
            short = (a + 1) <= B if fallback == "group" else whole_window_flat
            if incomplete or short:
                plans.append(GroupPlan("flat", rows, a))
            else:
                plans.append(GroupPlan("bank", rows, a, scan_n=a + 1, bank_k=B, post_lo=a + 1))
        else:
            if incomplete or whole_window_flat:
                plans.append(GroupPlan("flat", rows, a))
            else:
                plans.append(GroupPlan("bank", rows, a, scan_n=a, bank_k=B - G, post_lo=a))
    return plans


def token_bank(qbar_g, wbar_g, k, plan):
    """ADIndex §4.3, Eq. (13): the shared bank of one group.

    Scores the scanned prefix once with the group query (Eq. (8) has the same form as
    Eq. (1)) and keeps its Top-``bank_k`` positions.
    """
    n = min(plan.scan_n, k.shape[0])
    return topk(score_keys(qbar_g, wbar_g, k[:n]), plan.bank_k)


def refine_row(q_i, w_i, k, bank, post_lo, p_i, K):
    """ADIndex §4.3, Eq. (14): Top-K of the original indexer over C_i = bank U {post_lo..p_i}."""
    cand = np.union1d(np.asarray(bank, dtype=np.int64), np.arange(post_lo, int(p_i) + 1))
    cand = cand[cand <= p_i]
    return topk(score_keys(q_i, w_i, k[cand]), K, positions=cand)


def group_topk(q, w, k, qbar, wbar, q_pos0, G, B, K, mode, rows=None, fallback="group"):
    """Prefill in group mode: {row: Top-K positions}; group g uses qbar[g], wbar[g].

    Banks are only built for groups that own a requested row.
    """
    want = None if rows is None else set(int(r) for r in rows)
    out, banks = {}, {}
    for gi, plan in enumerate(plan_groups(q.shape[0], q_pos0, G, B, mode, fallback)):
        todo = [t for t in plan.rows if want is None or t in want]
        if not todo:
            continue
        if plan.kind == "flat":
            for t in todo:
                out[t] = flat_topk_row(q[t], w[t], k, q_pos0 + t, K)
            continue
        bank = token_bank(qbar[gi], wbar[gi], k, plan)
        banks[gi] = bank
        for t in todo:
            out[t] = refine_row(q[t], w[t], k, bank, plan.post_lo, q_pos0 + t, K)
    return out, banks


# ---------------------------------------------------------------------------------------
# Decode (one query per sequence, each sequence with its own key cache)
# ---------------------------------------------------------------------------------------

def decode_topk(q, w, caches, seq_len, K):
    """Plain indexer at decode: row b sits at position seq_len[b]-1 of its own cache."""
    return {b: flat_topk_row(q[b], w[b], caches[b], int(seq_len[b]) - 1, K)
            for b in range(q.shape[0])}


def decode_bank(qbar, wbar, caches, seq_len, B):
    """Bank refresh at decode: Eq. (13) with the anchor at the refreshing query's position
    a = seq_len[b]-1, i.e. Top-B of the group query's scores over s <= a."""
    return {b: token_bank(qbar[b], wbar[b], caches[b],
                          GroupPlan("bank", (b,), int(seq_len[b]) - 1,
                                    scan_n=int(seq_len[b]), bank_k=B))
            for b in range(qbar.shape[0])}


def decode_refine(q, w, caches, seq_len, banks, anchors, K):
    """Decode step reusing a bank: Eq. (14) with C = bank U {a+1 .. seq_len[b]-1}."""
    return {b: refine_row(q[b], w[b], caches[b], banks[b], int(anchors[b]) + 1,
                          int(seq_len[b]) - 1, K)
            for b in range(q.shape[0])}


# ---------------------------------------------------------------------------------------
# MTP target verification (one window of m queries per sequence)
# ---------------------------------------------------------------------------------------

def mtp_topk(q, w, caches, qbar, wbar, seq_len, m, G, P, K):
    """ADIndex §4.3 ("Application to Prefill and MTP") and Appendix A.2 ("Bank Sharing During
    MTP Target Verification"): each sequence b verifies a window of m queries, rows
    b*m .. b*m+m-1 of q, w. Its cache holds seq_len[b] keys, the window's own included, so
    window query j sits at position seq_len[b] - m + j and the first one sees
    N_b = seq_len[b] - m + 1 keys. The window is split into m/G groups of G queries (group
    queries qbar[b*m/G + g], wbar[...]), each with its own bank of P keys built over the
    history visible to its anchor, the group's first query. When N_b <= P the whole window
    uses the plain indexer instead (window-level fallback). Returns {row: Top-K positions}.
    """
    out = {}
    gps = m // G
    for b in range(len(caches)):
        q_pos0 = int(seq_len[b]) - m
        res, _ = group_topk(q[b * m:(b + 1) * m], w[b * m:(b + 1) * m], caches[b],
                            qbar[b * gps:(b + 1) * gps], wbar[b * gps:(b + 1) * gps], q_pos0,
                            G, P, K, "paper", fallback="window")
        for j, v in res.items():
            out[b * m + j] = v
    return out


# ---------------------------------------------------------------------------------------
# Layer-wise reuse calibration (ADIndex §4.1)
# ---------------------------------------------------------------------------------------

def group_union_sizes(topk_rows, G):
    """ADIndex §4.1, Eq. (4): for every group of G consecutive query rows (rows g*G ..
    g*G+G-1, complete groups only), the size of the union of their Top-K index sets; -1
    padding is not an index. U^max of the page is the maximum of these sizes."""
    rows = [set(int(x) for x in np.asarray(r).ravel() if int(x) >= 0) for r in topk_rows]
    return [len(set().union(*rows[g0:g0 + G])) for g0 in range(0, len(rows) - G + 1, G)]


def bank_coverage(topk_rows, bank_rows, G):
    """Shared-bank coverage (ADIndex §1, Figure 1(c), and Appendix B.4): the fraction of a
    query's original Top-K selections (the flat indexer's, Eq. (2)) that its group's shared
    bank includes. Query row i belongs to group i // G (complete groups only); a bank row
    lists the group's candidate positions - the bank of Eq. (13) and the post-anchor or
    window positions every member scans under Eq. (14) - and -1 is padding, as in a Top-K
    row. Reading: the post-anchor positions are counted as included, so coverage 1 is
    exactly the condition under which refinement recovers the full Top-K.

    Returns (hits, count) per row of the complete groups: hits[i] = |T_i n bank_g|,
    count[i] = |T_i|; coverage_i = hits[i] / count[i]."""
    hits, count = [], []
    ng = len(topk_rows) // G
    for i in range(ng * G):
        sel = set(int(x) for x in np.asarray(topk_rows[i]).ravel() if int(x) >= 0)
        bank = set(int(x) for x in np.asarray(bank_rows[i // G]).ravel() if int(x) >= 0)
        hits.append(len(sel & bank))
        count.append(len(sel))
    return np.asarray(hits, np.int64), np.asarray(count, np.int64)


# ---------------------------------------------------------------------------------------
# Training-free group queries
# ---------------------------------------------------------------------------------------

def mean_pool_group(q, w, G, Hg):
    """The proxy group query of the PIVOT baseline the paper compares with (ADIndex,
    Appendix B, "PIVOT"): per group of G consecutive rows, the member mean of each indexing
    head and of its gate, for the first Hg heads. q [T, H, d], w [T, H] (float64) ->
    qbar [T // G, Hg, d], wbar [T // G, Hg]; an incomplete trailing group gets none."""
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    ng = q.shape[0] // G
    qbar = np.zeros((ng, Hg, q.shape[2]))
    wbar = np.zeros((ng, Hg))
    for g in range(ng):
        for i in range(g * G, g * G + G):
            qbar[g] += q[i, :Hg]
            wbar[g] += w[i, :Hg]
        qbar[g] /= G
        wbar[g] /= G
    return qbar, wbar


def rope(x, pos, rope_dim=64, base=10000.0):
    """Rotary position embedding at position pos of one head vector x [d]: the pairs
    (x[2i], x[2i+1]), i < rope_dim/2, are rotated by the angle pos * base^(-2i/rope_dim); the
    other dimensions are left as they are (reading: the paper names RoPE at the group anchor
    without its layout; this is the interleaved-pair form over the first rope_dim dims)."""
    y = np.array(x, dtype=np.float64)
    if rope_dim > y.shape[0] or rope_dim % 2:
        raise ValueError("rope_dim must be even and at most the head dimension")
    for i in range(rope_dim // 2):
        a = pos * base ** (-2.0 * i / rope_dim)
        c, s = np.cos(a), np.sin(a)
        x0, x1 = y[2 * i], y[2 * i + 1]
        y[2 * i], y[2 * i + 1] = x0 * c - x1 * s, x0 * s + x1 * c
    return y


def group_indexer_queries(cq, h, w_pool, w_q, w_g, G, H_S, d, q_pos0=0, rope_dim=64,
                          base=10000.0):
    """ADIndex §4.2, Eqs. (6)-(7): the group indexer's query and gates for each complete group
    of G consecutive rows (anchor t = q_pos0 + g*G):
      c-bar = W_pool [max_i c_i ; min_i c_i ; mean_i c_i]   (element-wise over the members)
      h-bar = mean_i h_i
      q-bar_j = RoPE_t([W_Q c-bar]_j),   w-bar_j = sigmoid([W_G h-bar]_j).
    cq [T, d_c], h [T, d_h], w_pool [d_c, 3 d_c], w_q [H_S*d, d_c], w_g [H_S, d_h] ->
    qbar [T // G, H_S, d], wbar [T // G, H_S]."""
    cq, h = np.asarray(cq, np.float64), np.asarray(h, np.float64)
    ng = cq.shape[0] // G
    qbar, wbar = np.zeros((ng, H_S, d)), np.zeros((ng, H_S))
    for g in range(ng):
        c = cq[g * G:(g + 1) * G]
        cbar = np.asarray(w_pool, np.float64) @ np.concatenate([c.max(0), c.min(0), c.mean(0)])
        qpre = (np.asarray(w_q, np.float64) @ cbar).reshape(H_S, d)
        for j in range(H_S):
            qbar[g, j] = rope(qpre[j], q_pos0 + g * G, rope_dim, base)
        z = np.asarray(w_g, np.float64) @ h[g * G:(g + 1) * G].mean(0)
        wbar[g] = 1.0 / (1.0 + np.exp(-z))
    return qbar, wbar


# ---------------------------------------------------------------------------------------
# HISA: block filter, then token refinement (the HISA paper's two-stage indexer, with the
# reproduction settings of ADIndex Appendix C.5)
# ---------------------------------------------------------------------------------------

HISA_BLOCK = 128


def hisa_block_keys(k, block=HISA_BLOCK):
    """Mean-pooled block keys: kbar[b] = mean of k[b*block : (b+1)*block]; a trailing partial
    block is the mean of the keys it holds (HISA abstract: pooled block representations;
    ADIndex Appendix C.5: mean pooling of indexing keys over 128-token blocks)."""
    k = np.asarray(k, np.float64)
    nb = -(-k.shape[0] // block)
    return np.stack([k[b * block:(b + 1) * block].mean(axis=0) for b in range(nb)]) \
        if nb else np.zeros((0, k.shape[1]))


def hisa_blocks_row(q_t, w_t, kbar, p, n_blocks, block=HISA_BLOCK):
    """Candidate blocks of a query at position p (ADIndex Appendix C.5, HISA paragraph):
    blocks 0 .. p // block are visible; when at most n_blocks are, all of them; otherwise the
    first block and the query's own block, plus the n_blocks - (number forced) highest-scoring
    other visible blocks, a block scored like a key with its pooled key (Eq. (1) with kbar_b).
    Returns the block numbers, ascending."""
    cur = int(p) // block
    nvis = min(cur + 1, kbar.shape[0])
    if nvis <= n_blocks:
        return np.arange(nvis)
    forced = sorted({0, cur})
    rest = np.array([b for b in range(nvis) if b not in forced], dtype=np.int64)
    chosen = topk(score_keys(q_t, w_t, kbar[rest]), n_blocks - len(forced), rest)
    return np.sort(np.concatenate([np.array(forced, np.int64), chosen]))


def hisa_candidates(blocks, p, S, block=HISA_BLOCK):
    """Tokens of the chosen blocks visible to a query at position p (causal masking)."""
    lim = min(int(p) + 1, S)
    parts = [np.arange(b * block, min((b + 1) * block, lim)) for b in blocks]
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def hisa_topk_row(q_t, w_t, k, kbar, p, K, n_blocks, block=HISA_BLOCK):
    """One query: candidate blocks, then Top-K of their visible tokens rescored with all heads
    (Eq. (1)); a query with at most K visible tokens keeps all of them."""
    S = k.shape[0]
    if int(p) + 1 <= K:
        return np.arange(min(int(p) + 1, S))
    cand = hisa_candidates(hisa_blocks_row(q_t, w_t, kbar, p, n_blocks, block), p, S, block)
    return topk(score_keys(q_t, w_t, k[cand]), K, cand)


def hisa_topk(q, w, k, pos, K, n_blocks=64, block=HISA_BLOCK, rows=None):
    """HISA indexer: {row: Top-K positions} for the requested rows (all by default)."""
    k = np.asarray(k, np.float64)
    kbar = hisa_block_keys(k, block)
    rows = range(q.shape[0]) if rows is None else rows
    return {int(t): hisa_topk_row(q[t], w[t], k, kbar, pos[t], K, n_blocks, block)
            for t in rows}
