"""Comparison helpers shared by the GPU parity tests (CUDA path vs the fp64 oracle).

Tolerances: a GPU score must satisfy |I_gpu - I_ref| <= rtol * max(|I_ref|, F) with
rtol = 2e-2 for bf16 operands and 6e-2 for e4m3 operands, where
F = sum_j |w_j| * ||q_j|| * ||k_s|| / sqrt(d) is the typical magnitude of a score with
those operands (it keeps near-zero scores from making a relative error meaningless).
A GPU Top-K set must hold exactly min(K, n) distinct visible candidates and may differ
from the oracle's only at keys whose oracle score lies within that tolerance of the
oracle's K-th score.
"""

import numpy as np
import torch

from oracle import fp_formats

RTOL = {"bf16": 2e-2, "e4m3": 6e-2}


def f64(t, scale=None):
    """Exact float64 values of a bf16 tensor or of e4m3 codes times per-row scales."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return fp_formats.bf16_bits_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    if t.dtype == torch.uint8:
        return fp_formats.dequantize(t.numpy(), scale.detach().cpu().numpy(), "e4m3")
    return t.double().numpy()


def score_floor(q_t, w_t, keys):
    """F for one query against keys [n, d]."""
    d = q_t.shape[-1]
    qn = np.linalg.norm(q_t, axis=-1)                     # [H]
    kn = np.linalg.norm(keys, axis=-1)                    # [n]
    return (np.abs(w_t) * qn).sum() * kn / np.sqrt(d)


def check_scores(got, ref, floor, rtol, what=""):
    got = np.asarray(got, dtype=np.float64)
    bad = np.abs(got - ref) > rtol * np.maximum(np.abs(ref), floor)
    assert not bad.any(), (f"{what}: {bad.sum()} scores out of tolerance; first at "
                           f"{np.argwhere(bad)[:3].tolist()}: got {got[bad][:3]} ref {ref[bad][:3]}")


def check_topk(got_idx, cand_pos, cand_scores, cand_floor, K, rtol, got_scores=None, what=""):
    """One row. cand_pos / cand_scores / cand_floor: every visible candidate of the row with
    its oracle score and score floor. got_idx: the GPU row (-1 padded)."""
    got_idx = np.asarray(got_idx)
    n = len(cand_pos)
    m = min(K, n)
    valid = got_idx[got_idx >= 0]
    assert len(valid) == m, f"{what}: {len(valid)} indices, expected {m}"
    assert np.all(got_idx[m:] == -1), f"{what}: padding is not -1"
    assert len(set(valid.tolist())) == m, f"{what}: duplicate indices"
    where = {int(p): i for i, p in enumerate(cand_pos)}
    missing = [int(p) for p in valid if int(p) not in where]
    assert not missing, f"{what}: indices outside the candidate set: {missing[:5]}"
    if n > K:
        order = np.lexsort((np.asarray(cand_pos), -np.asarray(cand_scores)))
        ref_set = set(int(cand_pos[i]) for i in order[:K])
        theta = cand_scores[order[K - 1]]
        for p in set(valid.tolist()) ^ ref_set:
            i = where[p]
            tol = rtol * max(abs(cand_scores[i]), cand_floor[i])
            assert abs(cand_scores[i] - theta) <= tol, (
                f"{what}: key {p} (oracle score {cand_scores[i]:.6g}) differs from the oracle "
                f"set but is not within {tol:.3g} of the K-th score {theta:.6g}")
    if got_scores is not None:
        gs = np.asarray(got_scores, dtype=np.float64)[: m]
        idx = [where[int(p)] for p in valid]
        check_scores(gs, np.asarray(cand_scores)[idx], np.asarray(cand_floor)[idx], rtol,
                     what + " topk_score")
