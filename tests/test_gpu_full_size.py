"""Full-size parity on sampled rows, for the workloads whose rows are longer than 32768 keys:
the group-mode bank scan over 65536 tokens (ADIndex §4.3, Eq. (13): 1024 scan rows of up to
65472 keys, B = 8192) and one 4096-query chunk at the end of a 262144-token chunked prefill
(§3, Eqs. (1)-(2); group mode, §4.3, Eqs. (13)-(14)), in bf16 and e4m3, plus a launch of 160
rows of about 40000 keys whose K-th scores tie exactly. These are the configurations the
benchmark times; the oracle scores the sampled rows one by one.

Scan lengths and bank sizes come from the oracle's own group plan (oracle.indexer.plan_groups),
not from a restatement here.
"""

import numpy as np
import pytest
import torch

from oracle import indexer as ox
from sparse_attention_token_indexer_b200 import build, indexer, inputs

from parity import RTOL, check_scores, check_topk, f64, score_floor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    yield
    assert indexer.read_device_status() == 0


def _rows_f64(q, q_scale, rows):
    """Exact float64 values of the given rows of q (and their scales)."""
    r = torch.as_tensor(rows, device=q.device)
    return f64(q[r], None if q_scale is None else q_scale[r])


def _check_flat_rows(p, idx, sc, rows, k64, what):
    q64 = _rows_f64(p["q"], p["q_scale"], rows)
    w64 = p["w"][torch.as_tensor(rows, device=p["w"].device)].double().cpu().numpy()
    for j, t in enumerate(rows):
        n = p["q_pos0"] + t + 1
        keys = k64[:n]
        check_topk(idx[t], np.arange(n), ox.score_keys(q64[j], w64[j], keys),
                   score_floor(q64[j], w64[j], keys), p["K"], RTOL[p["dtype"]],
                   None if sc is None else sc[t], f"{what} row {t}")


def _chunk_rows(T, n=6, seed=0):
    rng = np.random.default_rng(seed)
    return sorted({0, 1, T // 2, T - 2, T - 1} | set(rng.choice(T, size=n, replace=False).tolist()))


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_chunk_at_the_end_of_a_262144_token_prefill(dtype):
    """The last 4096-query chunk of the 256K chunked prefill: every row sees 258049 to 262144
    keys, S = 262144 and the score workspace holds more than 2^32 bytes."""
    S, T, K = 262144, 4096, 2048
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=4, device="cuda", dtype=dtype, S=S)
    assert p["q_pos0"] == S - T
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K, p["q_scale"], p["k_scale"],
                                       q_pos0=p["q_pos0"], with_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    k64 = f64(p["k"], p["k_scale"])
    _check_flat_rows(p, idx, sc, _chunk_rows(T, seed=1), k64, f"c5 {dtype}")


def _group_inputs(T, S, q_pos0, G, Hg, dtype, seed):
    p = inputs.anchor_prefill(T, H=64, d=128, K=2048, seed=seed, device="cuda", S=S,
                              q_pos0=q_pos0)
    qbar, wbar = inputs.mean_pool_group_queries(p["q"].float(), p["w"], G, Hg)
    qbs = None
    if dtype == "e4m3":
        p.update(inputs.as_operands(p["q"].float(), p["k"].float(), "e4m3"))
        qbar, qbs = inputs.quantize_e4m3_rows(qbar)
        p["dtype"] = "e4m3"
    else:
        qbar = qbar.to(torch.bfloat16).contiguous()
    return p, qbar, qbs, wbar


def _check_groups(p, qbar, qbs, wbar, bank, idx, sc, mode, G, B, groups, k64, what,
                  rows_per_group=3):
    """Sampled groups of a group-mode call: the scanned bank part against Eq. (13) with the
    oracle's group scores, the post-anchor part exactly, and sampled members' refinement
    against Eq. (14) over the kernel's own bank (stage isolation)."""
    q_pos0, T, K = p["q_pos0"], p["T"], p["K"]
    plans = ox.plan_groups(T, q_pos0, G, B, mode)
    rtol = RTOL[p["dtype"]]
    qb64 = _rows_f64(qbar, qbs, groups)
    wb64 = wbar[torch.as_tensor(groups, device=wbar.device)].double().cpu().numpy()
    for j, g in enumerate(groups):
        plan = plans[g]
        assert plan.kind == "bank"
        keys = k64[:plan.scan_n]
        part = bank[g, :plan.bank_k]
        check_topk(part, np.arange(plan.scan_n), ox.score_keys(qb64[j], wb64[j], keys),
                   score_floor(qb64[j], wb64[j], keys), plan.bank_k, rtol,
                   what=f"{what} bank {g}")
        post = bank[g, plan.bank_k:]
        assert post.tolist() == list(range(plan.post_lo, plan.post_lo + len(post)))
        scan_part = part[part >= 0]
        members = [plan.rows[0], plan.rows[len(plan.rows) // 2], plan.rows[-1]][:rows_per_group]
        q64 = _rows_f64(p["q"], p["q_scale"], members)
        w64 = p["w"][torch.as_tensor(members, device=p["w"].device)].double().cpu().numpy()
        for m, r in enumerate(members):
            i = q_pos0 + r
            cand = np.union1d(scan_part, np.arange(plan.post_lo, i + 1))
            cand = cand[cand <= i]
            check_topk(idx[r], cand, ox.score_keys(q64[m], w64[m], k64[cand]),
                       score_floor(q64[m], w64[m], k64[cand]), K, rtol, sc[r],
                       f"{what} refine row {r}")


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_group_mode_scan_over_65536_tokens(dtype):
    """The group-mode workload at full size (T = 65536, G = 64, B = 8192, H_g = 16, WINDOW):
    1024 bank rows of 0 to 65472 scanned keys, sampled groups on both sides of 32768."""
    T, G, B, Hg = 65536, 64, 8192, 16
    p, qbar, qbs, wbar = _group_inputs(T, T, 0, G, Hg, dtype, seed=2)
    bank = indexer.group_bank(qbar, wbar, p["k"], G, B, "window", qbar_scale=qbs,
                              k_scale=p["k_scale"])
    idx, sc = indexer.bank_refine(p["q"], p["w"], p["k"], bank, G, B, "window", p["K"],
                                  q_scale=p["q_scale"], k_scale=p["k_scale"], with_scores=True)
    bank, idx, sc = bank.cpu().numpy(), idx.cpu().numpy(), sc.cpu().numpy()
    k64 = f64(p["k"], p["k_scale"])
    groups = [128, 129, 511, 512, 513, 700, 1023]      # scans of 8192 .. 65472 keys
    _check_groups(p, qbar, qbs, wbar, bank, idx, sc, "window", G, B, groups, k64,
                  f"c3 {dtype}", rows_per_group=2 if dtype == "e4m3" else 3)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_group_mode_on_the_last_chunk_of_262144_tokens(dtype):
    """Group mode (WINDOW, G = 64, B = 8192) on the last 4096-query chunk of the 256K prefill:
    64 bank rows scanning 258048 to 262080 keys."""
    S, T, G, B, Hg = 262144, 4096, 64, 8192, 16
    p, qbar, qbs, wbar = _group_inputs(T, S, S - T, G, Hg, dtype, seed=5)
    bank = indexer.group_bank(qbar, wbar, p["k"], G, B, "window", qbar_scale=qbs,
                              k_scale=p["k_scale"], q_pos0=p["q_pos0"])
    idx, sc = indexer.bank_refine(p["q"], p["w"], p["k"], bank, G, B, "window", p["K"],
                                  q_scale=p["q_scale"], k_scale=p["k_scale"],
                                  q_pos0=p["q_pos0"], with_scores=True)
    bank, idx, sc = bank.cpu().numpy(), idx.cpu().numpy(), sc.cpu().numpy()
    k64 = f64(p["k"], p["k_scale"])
    _check_groups(p, qbar, qbs, wbar, bank, idx, sc, "window", G, B, [0, 31, 63], k64,
                  f"c5 group {dtype}", rows_per_group=2)


@pytest.mark.parametrize("big,skew", [(0.6, 1.0), (0.03, 1.0), (0.03, 4.0)])
def test_many_long_rows_with_exact_ties(big, skew):
    """160 rows of 39841 to 40000 keys in one launch (more rows than SMs, every row longer than
    32768): keys are copies of 24 vectors a factor 2 apart, so each row's scores take 24 exact
    values and tens to thousands of keys tie at the K-th. The set must be the oracle's exactly
    (the lowest positions among the tied keys), in ascending positions. One copy holds a
    fraction `big` of the positions: 60 % (more keys at the threshold than the long-row select
    gathers: its radix passes take over) or 3 % (the gathered keys decide). With skew 4 the
    keys of every 16th tile of 128 positions (the tiles a long row's threshold is estimated
    from) are scaled by 4, so the estimate is far too high and the select lowers it."""
    S, T, K, nd, bigc = 40000, 160, 2048, 24, 3
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=18, device="cuda", S=S)
    rng = np.random.default_rng(9)
    which = np.where(rng.random(S) < big, bigc, rng.integers(0, nd, S))
    scales = torch.tensor([2.0 ** (nd - 13 - i) for i in range(nd)])
    v = p["k"][0].float().cpu()
    distinct = (scales[:, None] * v[None, :]).to(torch.bfloat16)
    k = distinct[torch.as_tensor(which)].contiguous()
    pos = np.arange(S)
    boost = ((pos // 128) % 16 == 0) & (skew != 1.0)
    k[torch.as_tensor(boost)] = (k[torch.as_tensor(boost)].float() * skew).to(torch.bfloat16)
    k = k.cuda()
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], k, K, q_pos0=p["q_pos0"],
                                       with_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    q64, w64, d64 = f64(p["q"]), p["w"].double().cpu().numpy(), f64(distinct)
    mult = np.where(boost, skew, 1.0)
    thresholds = set()
    for t in range(T):
        vals = ox.score_keys(q64[t], w64[t], d64)
        n = p["q_pos0"] + t + 1
        row = vals[which[:n]] * mult[:n]    # ReLU(c x) = c ReLU(x) for c > 0: exact
        order = np.lexsort((np.arange(n), -row))
        assert set(idx[t].tolist()) == set(order[:K].tolist()), f"row {t}"
        assert np.all(np.diff(idx[t]) > 0), f"row {t}: positions not ascending"
        keys = d64[which[idx[t]]] * mult[idx[t]][:, None]
        check_scores(sc[t], row[idx[t]], score_floor(q64[t], w64[t], keys), RTOL["bf16"],
                     f"row {t} scores")
        thresholds.add(int(np.sum(row == row[order[K - 1]])))
    assert max(thresholds) > 100       # rows whose K-th score is shared by many keys


def test_many_long_rows_with_negative_scores():
    """Negative gates over positive logits make every score negative: the long-row select's
    threshold then lies among negative scores (the float compare against a negative threshold
    value, keys below the sign bit). 160 rows of about 40000 keys, bf16, against the oracle
    with the parity tolerance."""
    S, T, K = 40000, 160, 2048
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=17, device="cuda", S=S)
    k = p["k"].float()
    k[:, 0] += 3.0                                        # every key shares a large component
    q = p["q"].float()
    q[..., 0] = q[..., 0].abs() + 3.0                     # which every query head reads
    p["k"], p["q"] = k.to(torch.bfloat16).contiguous(), q.to(torch.bfloat16).contiguous()
    p["w"] = (-p["w"] - 1e-3).contiguous()                # every gate negative
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K, q_pos0=p["q_pos0"],
                                       with_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    k64 = f64(p["k"])
    rows = [0, 1, 57, 100, 158, 159]
    q64 = _rows_f64(p["q"], None, rows)
    w64 = p["w"][torch.as_tensor(rows, device="cuda")].double().cpu().numpy()
    for j, t in enumerate(rows):
        n = p["q_pos0"] + t + 1
        cs = ox.score_keys(q64[j], w64[j], k64[:n])
        assert np.sort(cs)[-K] < 0, f"row {t}: the K-th score should be negative"
        check_topk(idx[t], np.arange(n), cs, score_floor(q64[j], w64[j], k64[:n]), K,
                   RTOL["bf16"], sc[t], f"negative row {t}")


def test_prefill_from_position_0_past_32768_rows():
    """One call of 36864 queries from position 0: the longest rows exceed what the register
    selects hold, so every row of the launch, from 1 key up, takes the sample-threshold select
    (rows shorter than K return all their keys, rows just past K, rows whose sample holds a
    handful of keys, rows ending a partial step of its copy ring)."""
    T, K = 36864, 256
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=61, device="cuda")
    assert p["q_pos0"] == 0
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K, with_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    k64 = f64(p["k"], p["k_scale"])
    rows = [0, 1, 2, K - 2, K - 1, K, K + 1, 2047, 2048, 4095, 4096, 4097, 8191, 8193, 20000,
            32767, 32768, T - 1]
    _check_flat_rows(p, idx, sc, rows, k64, "from 0")
