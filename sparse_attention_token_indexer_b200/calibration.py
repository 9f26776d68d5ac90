"""Layer-wise reuse calibration (ADIndex, arXiv 2611.12956v1, §4.1).

For one layer, the original indexer's Top-K sets of calibration queries give the bank
capacity a group size needs (Eq. (4): the union of the Top-K sets of G consecutive queries),
and the reuse configuration is the (G, P) with the largest scoring speedup whose budget P
holds that capacity (Eq. (5)). The speedup S(G, P; L) is the paper's joint one (Appendix A,
Table 5 panel c): prefill of L tokens plus R = 32 MTP verification rounds of m = 16 queries,
round j's first query seeing L + (j-1)*8 keys, every score evaluation counted once whatever
the number of heads. The union sizes are computed on the GPU (adx_group_union_sizes); the
statistics and the choice are host arithmetic on a handful of numbers.
"""

import ctypes

import numpy as np
import torch

from . import _lib as L

GROUP_SIZES = (4, 8, 16)
BUDGETS = (4096, 8192, 16384)
CRITERIA = ("max", "p90", "mean")


def union_sizes(topk_idx, G, S, stream=None):
    """Union sizes [T // G] int32 (device) of the Top-K rows topk_idx [T, K] (device int32)."""
    if topk_idx.dtype != torch.int32 or not topk_idx.is_cuda or not topk_idx.is_contiguous():
        raise ValueError("topk_idx must be a contiguous CUDA int32 tensor")
    T, K = topk_idx.shape
    out = torch.empty(T // G, dtype=torch.int32, device=topk_idx.device)
    s = stream if stream is not None else torch.cuda.current_stream(topk_idx.device)
    L.check("adx_group_union_sizes", L.lib().adx_group_union_sizes(
        ctypes.c_void_p(topk_idx.data_ptr()), T, K, G, S, ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(s.cuda_stream)))
    return out


def bank_coverage(topk_idx, bank_idx, G, S, stream=None):
    """Shared-bank coverage (ADIndex §1, Figure 1(c); Appendix B.4) of the flat Top-K rows
    topk_idx [T, K] by the group bank rows bank_idx [T // G, W] (device int32, as written by
    adx_index_prefill and adx_group_bank): (hits, count) [T // G * G] int32 device tensors,
    coverage of row i = hits[i] / count[i]."""
    for t in (topk_idx, bank_idx):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("topk_idx and bank_idx must be contiguous CUDA int32 tensors")
    T, K = topk_idx.shape
    n = T // G * G
    hits = torch.empty(n, dtype=torch.int32, device=topk_idx.device)
    count = torch.empty(n, dtype=torch.int32, device=topk_idx.device)
    s = stream if stream is not None else torch.cuda.current_stream(topk_idx.device)
    L.check("adx_bank_coverage", L.lib().adx_bank_coverage(
        ctypes.c_void_p(topk_idx.data_ptr()), T, K, ctypes.c_void_p(bank_idx.data_ptr()),
        bank_idx.shape[1], G, S, ctypes.c_void_p(hits.data_ptr()),
        ctypes.c_void_p(count.data_ptr()), ctypes.c_void_p(s.cuda_stream)))
    return hits, count


def coverage_by_position(hits, count, G):
    """Mean coverage at each member position r = 0 .. G-1 of a group, over the groups (the
    per-position view of Appendix B.4, Figure 4), and its mean over the positions (the
    layer summary)."""
    h = np.asarray(hits, dtype=np.float64).reshape(-1, G)
    c = np.asarray(count, dtype=np.float64).reshape(-1, G)
    per_pos = (h / np.maximum(c, 1.0)).mean(axis=0)
    return per_pos, float(per_pos.mean())


def capacity(unions, criterion="max"):
    """Bank capacity a layer needs from its union sizes: the maximum (the paper's default),
    the 90th percentile or the mean (the relaxed criteria)."""
    u = np.asarray(unions, dtype=np.float64)
    if u.size == 0:
        raise ValueError("no complete group")
    if criterion == "max":
        return float(u.max())
    if criterion == "p90":
        return float(np.percentile(u, 90))
    if criterion == "mean":
        return float(u.mean())
    raise ValueError(criterion)


def _prefill_counts(Lq, G, P):
    """(plain, reuse) score evaluations of prefilling Lq tokens: complete groups whose anchor
    a sees more than P keys scan a + 1 keys once and refine G members over P bank entries plus
    0..G-1 post-anchor keys; every other query scores its whole prefix."""
    plain = Lq * (Lq + 1) // 2
    a = np.arange(0, Lq - G + 1, G, dtype=np.int64)     # anchors of complete groups
    banked = a[a + 1 > P]
    reuse_banked = int((banked + 1 + G * P + G * (G - 1) // 2).sum())
    return plain, plain - _sum_prefix_rows(banked, G) + reuse_banked


def _sum_prefix_rows(anchors, G):
    """Sum over the members of the given groups of their prefix lengths pos + 1."""
    return int((G * (anchors + 1) + G * (G - 1) // 2).sum())


def _round_counts(N, G, P, m):
    """(plain, reuse) score evaluations of one verification window of m queries whose first
    query sees N keys; the whole window falls back when N <= P."""
    plain = m * N + m * (m - 1) // 2
    if N <= P:
        return plain, plain
    a = N - 1 + np.arange(0, m, G, dtype=np.int64)
    return plain, int((a + 1 + G * P + G * (G - 1) // 2).sum())


def speedup(G, P, Lq, R=32, m=16, accepted=8):
    """S(G, P; L): plain over reuse scoring counts of prefill of Lq tokens plus R rounds."""
    plain, reuse = _prefill_counts(Lq, G, P)
    for j in range(R):
        pb, pr = _round_counts(Lq + j * accepted, G, P, m)
        plain, reuse = plain + pb, reuse + pr
    return plain / reuse


def select_config(cap_by_G, Lq=131072, group_sizes=GROUP_SIZES, budgets=BUDGETS):
    """Eq. (5): the (G, P) maximising S(G, P; Lq) among those with capacity(G) <= P, or None
    when no budget holds the capacity of any group size (the layer keeps the plain indexer)."""
    best, best_s = None, 0.0
    for G in group_sizes:
        if G not in cap_by_G:
            continue
        for P in budgets:
            if cap_by_G[G] <= P:
                s = speedup(G, P, Lq)
                if s > best_s:
                    best, best_s = (G, P), s
    return best


def calibrate_layer(topk_idx, S, criterion="max", Lq=131072):
    """One layer's configuration from its calibration Top-K rows (device int32 [T, K])."""
    caps = {G: capacity(union_sizes(topk_idx, G, S).cpu().numpy(), criterion)
            for G in GROUP_SIZES if topk_idx.shape[0] >= G}
    return select_config(caps, Lq), caps
