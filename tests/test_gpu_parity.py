"""Parity of the CUDA path (through the C ABI) with the fp64 oracle on the same seeded inputs.

Scores must agree within rtol * max(|I|, F) (2e-2 bf16, 6e-2 e4m3; see tests/parity.py);
Top-K sets must agree except at keys within that tolerance of the oracle's K-th score.
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


def _to_cuda(p):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in p.items()}


def _flat_reference(q64, w64, k64, pos, rows):
    """Per requested row: visible positions, oracle scores, score floors."""
    out = {}
    for t in rows:
        n = min(int(pos[t]) + 1, k64.shape[0])
        keys = k64[:n]
        out[t] = (np.arange(n), ox.score_keys(q64[t], w64[t], keys),
                  score_floor(q64[t], w64[t], keys))
    return out


def _check_flat(p, idx, sc, rows, what):
    q64, k64 = f64(p["q"], p["q_scale"]), f64(p["k"], p["k_scale"])
    w64 = p["w"].double().cpu().numpy()
    pos = p["q_pos0"] + np.arange(p["T"])
    ref = _flat_reference(q64, w64, k64, pos, rows)
    idx, sc = idx.cpu().numpy(), None if sc is None else sc.cpu().numpy()
    for t in rows:
        cpos, cs, cf = ref[t]
        check_topk(idx[t], cpos, cs, cf, p["K"], RTOL[p["dtype"]],
                   None if sc is None else sc[t], f"{what} row {t}")
    return ref


def _rows_sample(T, K, n=40, seed=0):
    rng = np.random.default_rng(seed)
    fixed = {0, 1, 2, T - 1, T - 2, min(K - 1, T - 1), min(K, T - 1), min(K + 1, T - 1)}
    return sorted(fixed | set(rng.choice(T, size=min(n, T), replace=False).tolist()))


# ---------------------------------------------------------------------------------------
# flat prefill
# ---------------------------------------------------------------------------------------

def test_tiny_prefill_every_score_and_row():
    p = _to_cuda(inputs.tiny_prefill(seed=0))
    idx, sc, full = indexer.index_prefill(p["q"], p["w"], p["k"], p["K"], with_scores=True,
                                          all_scores=True)
    torch.cuda.synchronize()
    q64, k64, w64 = f64(p["q"]), f64(p["k"]), p["w"].double().cpu().numpy()
    T = p["T"]
    ref = ox.indexer_scores(q64, w64, k64, np.arange(T))
    got = full.cpu().numpy()[:, :T]
    vis = np.isfinite(ref)
    # invisible keys are -inf up to the end of the row's own 128-key tile (entries past the
    # last tile of a row block are not written)
    for t in range(T):
        end = min(T, (t // 128 + 1) * 128)
        assert np.all(np.isneginf(got[t, t + 1:end])), f"row {t}: invisible keys must be -inf"
    floor = np.stack([score_floor(q64[t], w64[t], k64) for t in range(T)])
    check_scores(got[vis], ref[vis], floor[vis], RTOL["bf16"], "tiny scores")
    _check_flat(p, idx, sc, range(T), "tiny")


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_anchor_prefill_all_rows(dtype):
    p = _to_cuda(inputs.anchor_prefill(1000, H=64, d=128, K=256, seed=11, dtype=dtype))
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], p["K"], p["q_scale"],
                                       p["k_scale"], with_scores=True)
    _check_flat(p, idx, sc, range(p["T"]), f"anchor {dtype}")


@pytest.mark.parametrize("H,d", [(16, 128), (4, 128), (64, 64)])
def test_other_head_counts(H, d):
    p = _to_cuda(inputs.anchor_prefill(600, H=H, d=d, K=100, seed=12))
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], p["K"], with_scores=True)
    _check_flat(p, idx, sc, range(p["T"]), f"H={H} d={d}")


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_chunked_prefill_with_offset(dtype):
    p = _to_cuda(inputs.anchor_prefill(700, H=64, d=128, K=512, seed=13, S=3000, dtype=dtype))
    assert p["q_pos0"] == 2300
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], p["K"], q_scale=p["q_scale"],
                                       k_scale=p["k_scale"], q_pos0=p["q_pos0"],
                                       with_scores=True)
    _check_flat(p, idx, sc, _rows_sample(700, 512), "chunk")


def test_short_rows_return_every_visible_key():
    p = _to_cuda(inputs.anchor_prefill(130, H=64, d=128, K=200, seed=14))
    idx, _, _ = indexer.index_prefill(p["q"], p["w"], p["k"], p["K"])
    idx = idx.cpu().numpy()
    for t in range(130):
        assert sorted(idx[t][idx[t] >= 0].tolist()) == list(range(t + 1))
        assert np.all(idx[t][t + 1:] == -1)
    p1 = _to_cuda(inputs.anchor_prefill(1, H=64, d=128, K=8, seed=15))
    idx, _, _ = indexer.index_prefill(p1["q"], p1["w"], p1["k"], 8)
    assert idx.cpu().tolist() == [[0] + [-1] * 7]


def test_negative_gates():
    p = _to_cuda(inputs.anchor_prefill(300, H=64, d=128, K=64, seed=16))
    p["w"] = p["w"] - 0.5 / 64          # mixed signs
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], p["K"], with_scores=True)
    _check_flat(p, idx, sc, range(300), "signed gates")


def test_rows_where_most_scores_are_exactly_zero():
    """A ReLU sum is exactly 0 for a key no head responds to. Here 85 % of the keys are -e_0
    and every query head has a positive first component, so most of each row scores exactly
    0: the row minimum holds most keys (counted apart from the histogram atomics), and in
    many rows the K-th score is 0 itself."""
    T, K = 3000, 256
    p = _to_cuda(inputs.anchor_prefill(T, H=64, d=128, K=K, seed=19))
    q = p["q"].float()
    q[..., 0] = q[..., 0].abs() + 3.0
    p["q"] = q.to(torch.bfloat16).contiguous()
    rng = np.random.default_rng(11)
    dead = torch.as_tensor(rng.random(T) < 0.85, device="cuda")
    k = p["k"].clone()
    k[dead] = 0
    k[dead, 0] = -1.0
    p["k"] = k
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K, with_scores=True)
    ref = _check_flat(p, idx, sc, _rows_sample(T, K, n=60, seed=6), "zeros")
    zero_rows = [t for t, (_, cs, _) in ref.items() if len(cs) > K and np.sort(cs)[-K] == 0]
    assert len(zero_rows) >= 5, "the K-th score is 0 in too few sampled rows"


@pytest.mark.parametrize("S,K", [(1200, 100), (1200, 700), (250, 37), (1280, 1279)])
def test_exact_ties_short_rows(S, K):
    """Rows of at most 1280 keys take the one-warp-per-row select. Keys are copies of 24
    vectors a factor 2 apart (exact scores in a fixed order, many equal at the K-th); its set
    must be the oracle's exactly, in ascending positions, with exact scores."""
    T, nd, big = 64, 24, 5
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=19, device="cuda", S=S)
    rng = np.random.default_rng(11)
    which = np.where(rng.random(S) < 0.5, big, rng.integers(0, nd, S))
    scales = torch.tensor([2.0 ** (nd - 13 - i) for i in range(nd)])
    v = p["k"][0].float().cpu()
    distinct = (scales[:, None] * v[None, :]).to(torch.bfloat16)
    k = distinct[torch.as_tensor(which)].contiguous().cuda()
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], k, K, q_pos0=p["q_pos0"],
                                       with_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    q64, w64, d64 = f64(p["q"]), p["w"].double().cpu().numpy(), f64(distinct)
    for t in range(T):
        vals = ox.score_keys(q64[t], w64[t], d64)
        n = p["q_pos0"] + t + 1
        row = vals[which[:n]]
        order = np.lexsort((np.arange(n), -row))
        m = min(K, n)
        assert set(idx[t][:m].tolist()) == set(order[:m].tolist()), f"row {t}"
        assert np.all(idx[t][m:] == -1) and np.all(np.diff(idx[t][:m]) > 0)
        keys = d64[which[idx[t][:m]]]
        check_scores(sc[t][:m], row[idx[t][:m]], score_floor(q64[t], w64[t], keys),
                     RTOL["bf16"], f"row {t} scores")


def test_exact_ties_take_the_lowest_positions():
    """Every key is one of 24 copies of one vector scaled by powers of two (exact in bf16 and
    in every product), so each query's scores take 24 exact values in a fixed order, a factor
    2 apart (or are all zero). One copy holds 60 % of the positions.
    Across rows the K-th score is shared by tens to thousands of keys: the select resolves
    the threshold by counting, by digits over the gathered keys of the threshold bin, or by
    more passes over the whole row. Its set must equal the oracle's exactly: every key above
    the K-th score and the lowest positions among the keys equal to it."""
    T, K, nd, big = 16384, 2048, 24, 3
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=18, device="cuda")
    rng = np.random.default_rng(9)
    which = np.where(rng.random(T) < 0.6, big, rng.integers(0, nd, T))
    scales = torch.tensor([2.0 ** (nd - 13 - i) for i in range(nd)])
    v = p["k"][0].float().cpu()
    distinct = (scales[:, None] * v[None, :]).to(torch.bfloat16)     # [nd, d], decreasing
    k = distinct[torch.as_tensor(which)].contiguous().cuda()
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], k, K, with_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    q64, w64, d64 = f64(p["q"]), p["w"].double().cpu().numpy(), f64(distinct)
    # rows 3042 .. 3322 leave 1878 .. 2045 keys in the threshold bin (gathered digits)
    rows = sorted(set(_rows_sample(T, K, n=80, seed=5)) | set(range(3042, 3330, 40)) |
                  {2100, 2500, 3500, 4000, 8000, 12000, 16383})
    for t in rows:
        vals = ox.score_keys(q64[t], w64[t], d64)
        sv = np.sort(vals)
        assert np.all(sv == 0) or np.allclose(sv[1:] / sv[:-1], 2.0), t
        n = t + 1
        row = vals[which[:n]]
        order = np.lexsort((np.arange(n), -row))
        m = min(K, n)
        assert set(idx[t][:m].tolist()) == set(order[:m].tolist()), f"row {t}"
        assert np.all(idx[t][m:] == -1)
        assert np.all(np.diff(idx[t][:m]) > 0), f"row {t}: positions not ascending"


# ---------------------------------------------------------------------------------------
# group bank + refinement
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["window", "paper"])
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_group_bank_and_refine(mode, dtype):
    T, G, B, K, Hg = 1536 + 37, 64, 512, 128, 16
    p = _to_cuda(inputs.group_prefill(T, H=64, d=128, K=K, G=G, B=B, Hg=Hg, seed=21,
                                      dtype=dtype))
    rtol = RTOL[dtype]
    bank = indexer.group_bank(p["qbar"], p["wbar"], p["k"], G, B, mode, p["qbar_scale"],
                              p["k_scale"])
    idx, sc = indexer.bank_refine(p["q"], p["w"], p["k"], bank, G, B, mode, K, p["q_scale"],
                                  p["k_scale"], with_scores=True)
    torch.cuda.synchronize()
    q64, k64 = f64(p["q"], p["q_scale"]), f64(p["k"], p["k_scale"])
    w64 = p["w"].double().cpu().numpy()
    qb64, wb64 = f64(p["qbar"], p["qbar_scale"]), p["wbar"].double().cpu().numpy()
    bank = bank.cpu().numpy()
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    plans = ox.plan_groups(T, 0, G, B, mode)
    assert bank.shape[1] == indexer.bank_width(B, G, mode)
    n_complete = T // G
    for g in range(n_complete):
        a = g * G
        plan = plans[g]
        if plan.kind == "flat":
            # a PAPER group whose anchor sees at most B keys: the bank path still runs and its
            # bank must hold the anchor's whole prefix (then refinement is the plain indexer)
            bank_k = B
            assert sorted(x for x in bank[g, :bank_k].tolist() if x >= 0) == list(range(a + 1))
            lo = a + 1
        else:
            bank_k, lo = plan.bank_k, plan.post_lo
            # stage 1: the bank's scan part against Eq. (13) with the oracle's group scores
            keys = k64[:plan.scan_n]
            bs = ox.score_keys(qb64[g], wb64[g], keys)
            bf = score_floor(qb64[g], wb64[g], keys)
            check_topk(bank[g, :bank_k], np.arange(plan.scan_n), bs, bf, bank_k, rtol,
                       what=f"bank {g}")
        post = bank[g, bank_k:]
        assert post.tolist() == list(range(lo, lo + len(post)))
        # stage 2: refinement over the GPU's own bank (stage isolation)
        scan_part = bank[g, :bank_k]
        scan_part = scan_part[scan_part >= 0]
        for i in range(a, a + G, 7 if g % 3 else 1):
            cand = np.union1d(scan_part, np.arange(lo, i + 1))
            cand = cand[cand <= i]
            cs = ox.score_keys(q64[i], w64[i], k64[cand])
            cf = score_floor(q64[i], w64[i], k64[cand])
            check_topk(idx[i], cand, cs, cf, K, rtol, sc[i], f"refine row {i}")
    # the incomplete trailing group uses the plain indexer
    pos = np.arange(T)
    tail = list(range(n_complete * G, T))
    ref = _flat_reference(q64, w64, k64, pos, tail)
    for t in tail:
        cpos, cs, cf = ref[t]
        check_topk(idx[t], cpos, cs, cf, K, rtol, sc[t], f"tail row {t}")
    # paper fallback groups (a + 1 <= B) give the plain indexer's result exactly
    if mode == "paper":
        flat_idx, _, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K, p["q_scale"],
                                               p["k_scale"])
        flat_idx = flat_idx.cpu().numpy()
        for plan in plans:
            if plan.kind == "flat":
                for t in plan.rows:
                    assert set(idx[t].tolist()) == set(flat_idx[t].tolist()), t


# ---------------------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("k_dtype", ["e4m3", "bf16"])
def test_decode_flat(k_dtype):
    prob = inputs.decode_problem(Bs=4, S=5000, H=64, d=128, K=256, Hg=16, steps=1, seed=31,
                                 k_dtype=k_dtype, device="cuda")
    seq_len = torch.tensor([5000, 4097, 129, 1], dtype=torch.int32, device="cuda")
    q, w = prob["q_steps"][0], prob["w_steps"][0]
    idx, sc = indexer.index_decode(q, w, prob["k"], seq_len, 256, k_scale=prob["k_scale"],
                                   with_scores=True)
    torch.cuda.synchronize()
    q64, w64 = f64(q), w.double().cpu().numpy()
    k64 = f64(prob["k"].reshape(-1, 128), None if prob["k_scale"] is None
              else prob["k_scale"].reshape(-1)).reshape(4, -1, 128)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    for b, n in enumerate(seq_len.tolist()):
        keys = k64[b, :n]
        check_topk(idx[b], np.arange(n), ox.score_keys(q64[b], w64[b], keys),
                   score_floor(q64[b], w64[b], keys), 256, RTOL[k_dtype], sc[b], f"decode {b}")


@pytest.mark.parametrize("S", [12000, 40000])
def test_decode_long_rows_with_ties(S):
    """Few long rows: each row is selected by one cluster of CTAs (3 and 8 CTAs for these
    lengths), the row cut into one slice per CTA. Keys tied at the threshold lie in every
    slice; the lowest positions among them must be the ones taken."""
    Bs, K = 3, 512
    prob = inputs.decode_problem(Bs=Bs, S=S, H=64, d=128, K=K, Hg=16, steps=1, seed=33,
                                 device="cuda")
    k, ks = prob["k"], prob["k_scale"]
    q, w = prob["q_steps"][0], prob["w_steps"][0]
    seq_len = torch.tensor([S, S * 4 // 7 + 3, 2], dtype=torch.int32, device="cuda")
    # sequence 0: 300 keys far above the rest and 1500 exact copies of one key below them
    q64, w64 = f64(q), w.double().cpu().numpy()
    base = ox.score_keys(q64[0], w64[0], f64(k[0, :S], ks[0, :S]))
    top = int(np.argmax(base))
    rng = np.random.default_rng(7)
    pos = rng.choice(S, size=1800, replace=False)
    p_hi, p_tie = np.sort(pos[:300]), np.sort(pos[300:])
    row, scale = k[0, top].clone(), float(ks[0, top])
    for ps, mult in ((p_hi, 8.0), (p_tie, 4.0)):
        sel = torch.as_tensor(ps, device="cuda")
        k[0, sel] = row
        ks[0, sel] = scale * mult
    idx, sc = indexer.index_decode(q, w, k, seq_len, K, k_scale=ks, with_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    expect = set(p_hi.tolist()) | set(p_tie[: K - len(p_hi)].tolist())
    assert set(idx[0].tolist()) == expect
    for b, n in enumerate(seq_len.tolist()):
        keys = f64(k[b, :n], ks[b, :n])
        check_topk(idx[b], np.arange(n), ox.score_keys(q64[b], w64[b], keys),
                   score_floor(q64[b], w64[b], keys), K, RTOL["e4m3"], sc[b], f"dlong {b}")


def test_decode_bank_reuse():
    Bs, S, K, B, G = 4, 6000, 256, 1024, 16
    prob = inputs.decode_problem(Bs=Bs, S=S, H=64, d=128, K=K, Hg=16, steps=G, seed=32,
                                 device="cuda")
    k, ks = prob["k"], prob["k_scale"]
    seq0 = inputs.decode_seq_len(prob, 0)
    qbar, wbar = prob["q_steps"][0][:, :16].contiguous(), prob["w_steps"][0][:, :16].contiguous()
    bank = indexer.group_bank(qbar, wbar, k, G, B, "paper", k_scale=ks, seq_len=seq0)
    k64 = f64(k.reshape(-1, 128), ks.reshape(-1)).reshape(Bs, -1, 128)
    qb64, wb64 = f64(qbar), wbar.double().cpu().numpy()
    bank_np = bank.cpu().numpy()
    assert bank_np.shape == (Bs, B + G - 1)
    for b in range(Bs):
        keys = k64[b, :S]
        check_topk(bank_np[b, :B], np.arange(S), ox.score_keys(qb64[b], wb64[b], keys),
                   score_floor(qb64[b], wb64[b], keys), B, RTOL["e4m3"], what=f"dbank {b}")
        assert bank_np[b, B:].tolist() == list(range(S, S + G - 1))
    for step in (0, 1, 5, G - 1):
        seq = inputs.decode_seq_len(prob, step)
        q, w = prob["q_steps"][step], prob["w_steps"][step]
        idx, sc = indexer.bank_refine(q, w, k, bank, G, B, "paper", K, k_scale=ks,
                                      seq_len=seq, with_scores=True)
        idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
        q64, w64 = f64(q), w.double().cpu().numpy()
        pos = S + step - 1
        for b in range(Bs):
            cand = np.union1d(bank_np[b, :B], np.arange(S, pos + 1))
            cand = cand[(cand >= 0) & (cand <= pos)]
            keys = k64[b, cand]
            check_topk(idx[b], cand, ox.score_keys(q64[b], w64[b], keys),
                       score_floor(q64[b], w64[b], keys), K, RTOL["e4m3"], sc[b],
                       f"dref step {step} seq {b}")


@pytest.mark.parametrize("k_dtype,B", [("e4m3", 1024), ("bf16", 1024), ("e4m3", 8192)])
def test_decode_refine_over_a_packed_bank_equals_the_gather_path(k_dtype, B):
    """The bank's key rows packed once at the refresh and streamed by every refinement give the
    same result as gathering them from the cache each step, bit for bit (same keys, same
    kernels): both Top-K rows and scores, at the refresh step and at later steps whose
    post-anchor keys the refinement copies into the packed bank; e4m3 and bf16 caches, and a
    bank larger than the history (empty slots, -1 in the bank row)."""
    Bs, S, K, G = 4, 6000, 256, 16
    prob = inputs.decode_problem(Bs=Bs, S=S, H=64, d=128, K=K, Hg=16, steps=G, seed=35,
                                 device="cuda", k_dtype=k_dtype)
    k, ks = prob["k"], prob["k_scale"]
    seq0 = inputs.decode_seq_len(prob, 0)
    qbar = prob["q_steps"][0][:, :16].contiguous()
    wbar = prob["w_steps"][0][:, :16].contiguous()
    bank = indexer.group_bank(qbar, wbar, k, G, B, "paper", k_scale=ks, seq_len=seq0)
    keys, kss = indexer.pack_bank_keys(prob["q_steps"][0], prob["w_steps"][0], k, bank, G,
                                       B, k_scale=ks, seq_len=seq0)
    for step in (0, 1, 5, G - 1):
        seq = inputs.decode_seq_len(prob, step)
        q, w = prob["q_steps"][step], prob["w_steps"][step]
        ref = indexer.bank_refine(q, w, k, bank, G, B, "paper", K, k_scale=ks, seq_len=seq,
                                  with_scores=True)
        got = indexer.bank_refine_packed(q, w, k, bank, keys, kss, G, B, K, k_scale=ks,
                                         seq_len=seq, with_scores=True)
        assert torch.equal(got[0], ref[0]), (k_dtype, step)
        assert torch.equal(got[1], ref[1]), (k_dtype, step)


# ---------------------------------------------------------------------------------------
# MTP target verification
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("G", [4, 8, 16])
@pytest.mark.parametrize("k_dtype", ["e4m3", "bf16"])
def test_mtp_windows(G, k_dtype):
    """Four windows of m = 16 queries: one falls back (its first query sees P - 5 keys), one
    is just past the budget, one mid-size, one at the end of the cache."""
    Bs, S0, m, P, K, Hg = 4, 4096, 16, 512, 128, 16
    prob = inputs.decode_problem(Bs=Bs, S=S0, H=64, d=128, K=K, Hg=Hg, steps=m, seed=34,
                                 k_dtype=k_dtype, device="cuda")
    k, ks = prob["k"], prob["k_scale"]
    S_cap = k.shape[1]
    first = [P - 5, P + 3, 2000, S_cap - m + 1]          # keys the first window query sees
    seq_len = torch.tensor([n + m - 1 for n in first], dtype=torch.int32, device="cuda")
    q = prob["q_steps"].transpose(0, 1).reshape(Bs * m, 64, 128).contiguous()
    w = prob["w_steps"].transpose(0, 1).reshape(Bs * m, 64).contiguous()
    qbar, wbar = inputs.mean_pool_group_queries(q.float(), w, G, Hg)
    qbar = qbar.to(torch.bfloat16).contiguous()
    idx, sc, banks = indexer.index_mtp(q, w, k, seq_len, qbar, wbar, m, G, P, K, k_scale=ks,
                                       with_scores=True, with_banks=True)
    idx, sc, banks = idx.cpu().numpy(), sc.cpu().numpy(), banks.cpu().numpy()
    q64, w64, qb64, wb64 = f64(q), w.double().cpu().numpy(), f64(qbar), wbar.double().cpu().numpy()
    caches = [f64(k[b, :int(n)], None if ks is None else ks[b, :int(n)])
              for b, n in enumerate(seq_len.tolist())]
    ref = ox.mtp_topk(q64, w64, caches, qb64, wb64, seq_len.tolist(), m, G, P, K)
    gps, tol = m // G, RTOL[k_dtype]
    for b, n in enumerate(seq_len.tolist()):
        keys = caches[b]
        for g in range(gps):
            a = n - m + g * G
            row = banks[b * gps + g]
            if first[b] <= P:       # window-level fallback: the plain indexer
                assert row[:a + G].tolist() == list(range(a + G))
                assert np.all(row[a + G:] == -1)
                cands = [np.arange(n - m + j + 1) for j in range(g * G, g * G + G)]
            else:
                sb = ox.score_keys(qb64[b * gps + g], wb64[b * gps + g], keys[:a + 1])
                check_topk(row[:P], np.arange(a + 1), sb,
                           score_floor(qb64[b * gps + g], wb64[b * gps + g], keys[:a + 1]), P,
                           tol, what=f"mtp bank {b}/{g}")
                assert row[P:P + G - 1].tolist() == list(range(a + 1, a + G))
                assert np.all(row[P + G - 1:] == -1)
                bank = row[:P][row[:P] >= 0]
                cands = [np.union1d(bank, np.arange(a + 1, n - m + j + 1))
                         for j in range(g * G, g * G + G)]
                exact = set(bank.tolist()) == set(np.asarray(ox.token_bank(
                    qb64[b * gps + g], wb64[b * gps + g], keys,
                    ox.GroupPlan("bank", (), a, scan_n=a + 1, bank_k=P))).tolist())
            for j, cand in zip(range(g * G, g * G + G), cands):
                r = b * m + j
                cs = ox.score_keys(q64[r], w64[r], keys[cand])
                check_topk(idx[r], cand, cs, score_floor(q64[r], w64[r], keys[cand]), K, tol,
                           sc[r], f"mtp row {b}/{j}")
                if first[b] <= P or exact:  # same candidates as the oracle's own procedure
                    assert set(ref[r]) == set(ox.topk(cs, K, positions=cand).tolist())


# ---------------------------------------------------------------------------------------
# full-size workloads, sampled rows, in the configuration bench.py times
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_full_size_flat_prefill_sampled(dtype):
    T, K = 16384, 2048
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=1, device="cuda", dtype=dtype)
    idx, sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K, p["q_scale"], p["k_scale"],
                                       with_scores=True)
    _check_flat(p, idx, sc, _rows_sample(T, K, n=24, seed=3), f"full {dtype}")


def test_full_size_decode_sampled():
    Bs, S, K = 32, 131072, 2048
    prob = inputs.decode_problem(Bs=Bs, S=S, H=64, d=128, K=K, Hg=16, steps=1, seed=3,
                                 device="cuda")
    seq = inputs.decode_seq_len(prob, 0)
    q, w = prob["q_steps"][0], prob["w_steps"][0]
    idx, sc = indexer.index_decode(q, w, prob["k"], seq, K, k_scale=prob["k_scale"],
                                   with_scores=True)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    q64, w64 = f64(q), w.double().cpu().numpy()
    for b in (0, 17, 31):
        keys = f64(prob["k"][b], prob["k_scale"][b])
        check_topk(idx[b], np.arange(S), ox.score_keys(q64[b], w64[b], keys),
                   score_floor(q64[b], w64[b], keys), K, RTOL["e4m3"], sc[b], f"dfull {b}")


@pytest.mark.parametrize("q_pos0", [4096, 8192])
def test_bank_rows_starting_past_a_select_class(q_pos0):
    """Bank scan rows grow by G per group; when the first one is just longer than a select
    class holds (4097 and 8193 keys here), it must still go to a class that holds it. The
    key at the last scanned position is planted far above the rest, so a bank that drops
    it fails."""
    G, B, Hg, T = 64, 512, 16, 3 * 64
    S = q_pos0 + T
    p = _to_cuda(inputs.anchor_prefill(T, H=64, d=128, K=B, seed=24, S=S, q_pos0=q_pos0))
    qbar, wbar = inputs.mean_pool_group_queries(p["q"].float(), p["w"], G, Hg)
    qbar = qbar.to(torch.bfloat16).contiguous()
    qb64, wb64 = f64(qbar), wbar.double().cpu().numpy()
    base = ox.score_keys(qb64[0], wb64[0], f64(p["k"][:q_pos0]))
    p["k"][q_pos0] = (p["k"][int(np.argmax(base))].float() * 4).to(torch.bfloat16)
    bank = indexer.group_bank(qbar, wbar, p["k"], G, B, "paper", q_pos0=q_pos0)
    bank = bank.cpu().numpy()
    k64 = f64(p["k"])
    assert q_pos0 in bank[0, :B].tolist()
    for g, plan in enumerate(ox.plan_groups(T, q_pos0, G, B, "paper")):
        assert plan.kind == "bank" and plan.bank_k == B
        keys = k64[:plan.scan_n]
        check_topk(bank[g, :B], np.arange(plan.scan_n), ox.score_keys(qb64[g], wb64[g], keys),
                   score_floor(qb64[g], wb64[g], keys), B, RTOL["bf16"], what=f"bank {g}")


@pytest.mark.parametrize("mode,dtype", [("window", "bf16"), ("paper", "bf16"),
                                        ("window", "e4m3"), ("paper", "e4m3")])
def test_group_mode_on_a_later_chunk(mode, dtype):
    """Group mode for one query chunk of a longer prefix (q_pos0 > 0), as chunked prefill
    runs it; includes an incomplete trailing group; bf16 and e4m3 operands."""
    S, T, q_pos0, G, B, K, Hg = 3000, 64 * 9 + 21, 2300, 64, 512, 128, 16
    p = _to_cuda(inputs.anchor_prefill(T, H=64, d=128, K=K, seed=23, S=S, q_pos0=q_pos0))
    qbar, wbar = inputs.mean_pool_group_queries(p["q"].float(), p["w"], G, Hg)
    qbs = None
    if dtype == "e4m3":
        p.update(inputs.as_operands(p["q"].float(), p["k"].float(), "e4m3"))
        qbar, qbs = inputs.quantize_e4m3_rows(qbar)
    else:
        qbar = qbar.to(torch.bfloat16).contiguous()
    bank = indexer.group_bank(qbar, wbar, p["k"], G, B, mode, qbar_scale=qbs,
                              k_scale=p["k_scale"], q_pos0=q_pos0)
    idx, sc = indexer.bank_refine(p["q"], p["w"], p["k"], bank, G, B, mode, K,
                                  q_scale=p["q_scale"], k_scale=p["k_scale"], q_pos0=q_pos0,
                                  with_scores=True)
    torch.cuda.synchronize()
    q64, k64 = f64(p["q"], p["q_scale"]), f64(p["k"], p["k_scale"])
    w64 = p["w"].double().cpu().numpy()
    qb64, wb64 = f64(qbar, qbs), wbar.double().cpu().numpy()
    rtol = RTOL[dtype]
    bank, idx, sc = bank.cpu().numpy(), idx.cpu().numpy(), sc.cpu().numpy()
    plans = ox.plan_groups(T, q_pos0, G, B, mode)
    for g in range(T // G):
        plan = plans[g]
        assert plan.kind == "bank"      # every anchor here sees more than B keys
        bank_k, lo = plan.bank_k, plan.post_lo
        keys = k64[:plan.scan_n]
        check_topk(bank[g, :bank_k], np.arange(plan.scan_n),
                   ox.score_keys(qb64[g], wb64[g], keys), score_floor(qb64[g], wb64[g], keys),
                   bank_k, rtol, what=f"bank {g}")
        scan_part = bank[g, :bank_k][bank[g, :bank_k] >= 0]
        for r in range(g * G, g * G + G, 5):
            i = q_pos0 + r
            cand = np.union1d(scan_part, np.arange(lo, i + 1))
            cand = cand[cand <= i]
            check_topk(idx[r], cand, ox.score_keys(q64[r], w64[r], k64[cand]),
                       score_floor(q64[r], w64[r], k64[cand]), K, rtol, sc[r],
                       f"refine row {r}")
    for r in range(T // G * G, T):
        n = q_pos0 + r + 1
        check_topk(idx[r], np.arange(n), ox.score_keys(q64[r], w64[r], k64[:n]),
                   score_floor(q64[r], w64[r], k64[:n]), K, rtol, sc[r], f"tail {r}")


# ---------------------------------------------------------------------------------------
# training-free group queries (the PIVOT proxy)
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("G,Hg", [(64, 16), (4, 64), (16, 16), (1, 8)])
def test_group_query_mean(dtype, G, Hg):
    """bf16 output of an fp32 member sum: within half a bf16 step of the exact mean plus the
    fp32 accumulation error relative to the members' magnitudes."""
    T = 1000
    p = inputs.anchor_prefill(T, H=64, d=128, K=64, seed=26, device="cuda", dtype=dtype)
    qbar, wbar = indexer.group_query_mean(p["q"], p["w"], G, Hg, q_scale=p["q_scale"])
    q64, w64 = f64(p["q"], p["q_scale"]), p["w"].double().cpu().numpy()
    rq, rw = ox.mean_pool_group(q64, w64, G, Hg)
    ng = T // G
    mag = np.abs(q64[:ng * G, :Hg]).reshape(ng, G, Hg, -1).mean(axis=1)
    got = f64(qbar)
    assert got.shape == rq.shape
    assert np.all(np.abs(got - rq) <= 2.0 ** -8 * np.abs(rq) + 2.0 ** -20 * (mag + 1e-30))
    assert np.allclose(wbar.cpu().double().numpy(), rw, rtol=1e-6, atol=0)


@pytest.mark.parametrize("T,G,rope_dim,q_pos0,d_c,d_h,H_S", [
    (16 * 4 + 3, 4, 64, 0, 192, 320, 4), (8 * 16 + 15, 16, 64, 100000, 192, 320, 4),
    (5 * 64, 64, 0, 7, 192, 320, 4), (3 * 8, 8, 128, 262143, 192, 320, 4),
    # two column blocks per group, the first holding latent and hidden-state columns
    (6 * 16 + 5, 16, 64, 65536, 1536, 2048, 16)])
def test_group_indexer_queries(T, G, rope_dim, q_pos0, d_c, d_h, H_S):
    """Eqs. (6)-(7) on the library's tcgen05 GEMM + the pooling and RoPE kernels against the
    oracle in fp64. The path rounds the pooled mean, h-bar, c-bar and q-bar to bf16 (relative
    2^-9 each), so a
    head's error is a few 2^-9 of its rms plus q-bar's own rounding; the gates see h-bar's
    rounding through a sigmoid of slope at most 1/4."""
    p = inputs.group_indexer_problem(T, d_c=d_c, d_h=d_h, H_S=H_S, d=128, seed=28, device="cuda")
    qbar, wbar = indexer.group_indexer_queries(p["cq"], p["h"], p["w_pool"], p["w_q"], p["w_g"],
                                               G, H_S, 128, q_pos0=q_pos0, rope_dim=rope_dim)
    cpu = {k: (v.double().cpu().numpy() if torch.is_tensor(v) else v) for k, v in p.items()}
    rq, rw = ox.group_indexer_queries(cpu["cq"], cpu["h"], cpu["w_pool"], cpu["w_q"],
                                      cpu["w_g"], G, H_S, 128, q_pos0=q_pos0, rope_dim=rope_dim)
    got = f64(qbar)
    assert got.shape == rq.shape == (T // G, H_S, 128)
    rms = np.sqrt((rq ** 2).mean(axis=2, keepdims=True))
    assert np.all(np.abs(got - rq) <= 2.0 ** -6 * rms + 2.0 ** -8 * np.abs(rq))
    assert np.abs(wbar.cpu().double().numpy() - rw).max() <= 2.0 ** -8


def test_group_mode_on_kernel_group_queries():
    """Group mode end to end with the group queries built by the library itself."""
    T, G, B, K, Hg = 64 * 12, 64, 256, 128, 16
    p = _to_cuda(inputs.anchor_prefill(T, H=64, d=128, K=K, seed=27))
    qbar, wbar = indexer.group_query_mean(p["q"], p["w"], G, Hg)
    bank = indexer.group_bank(qbar, wbar, p["k"], G, B, "paper")
    idx, sc = indexer.bank_refine(p["q"], p["w"], p["k"], bank, G, B, "paper", K,
                                  with_scores=True)
    q64, k64, w64 = f64(p["q"]), f64(p["k"]), p["w"].double().cpu().numpy()
    qb64, wb64 = f64(qbar), wbar.double().cpu().numpy()
    bank, idx, sc = bank.cpu().numpy(), idx.cpu().numpy(), sc.cpu().numpy()
    for g in range(T // G):
        a = g * G
        keys = k64[:a + 1]
        check_topk(bank[g, :B], np.arange(a + 1), ox.score_keys(qb64[g], wb64[g], keys),
                   score_floor(qb64[g], wb64[g], keys), B, RTOL["bf16"], what=f"bank {g}")
        part = bank[g, :B][bank[g, :B] >= 0]
        for r in range(a, a + G, 9):
            cand = np.union1d(part, np.arange(a + 1, r + 1)) if a + 1 > B else np.arange(r + 1)
            cand = cand[cand <= r]
            check_topk(idx[r], cand, ox.score_keys(q64[r], w64[r], k64[cand]),
                       score_floor(q64[r], w64[r], k64[cand]), K, RTOL["bf16"], sc[r],
                       f"refine row {r}")


# ---------------------------------------------------------------------------------------
# host buffers (copies overlapped with the indexing, chunk by chunk)
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_host_buffer_prefill_equals_device_path(dtype):
    """Chunking only changes how the rows are partitioned: every row's scores and Top-K are
    the same as on the device-buffer path, bit for bit."""
    T, K = 5000, 300
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=28, device="cuda", dtype=dtype, S=5300)
    ref_idx, ref_sc, _ = indexer.index_prefill(p["q"], p["w"], p["k"], K, p["q_scale"],
                                               p["k_scale"], q_pos0=p["q_pos0"], with_scores=True)
    host = {n: (None if p[n] is None else p[n].cpu().pin_memory())
            for n in ("q", "w", "k", "q_scale", "k_scale")}
    idx, sc = indexer.index_prefill_host(host["q"], host["w"], host["k"], K, host["q_scale"],
                                         host["k_scale"], q_pos0=p["q_pos0"],
                                         rows_per_chunk=1024, with_scores=True)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref_idx.cpu())
    assert torch.equal(sc, ref_sc.cpu())


# ---------------------------------------------------------------------------------------
# HISA: block filter, then token refinement
# ---------------------------------------------------------------------------------------

def _check_hisa_row(t, p, q64, w64, k64, kbar64, blocks, idx, sc, n_blocks, K, rtol_blk, rtol,
                    S):
    """Row t at position p: the kernel's kept blocks must be the visible blocks (when they
    fit) or the forced pair plus a valid Top-(n_blocks - 2) of the other visible blocks under
    the oracle's block scores; its Top-K must be a valid Top-K of those blocks' visible
    tokens under the oracle's token scores."""
    cur = p // ox.HISA_BLOCK
    nvis = cur + 1
    got = blocks[t][blocks[t] >= 0]
    assert np.all(blocks[t][len(got):] == -1) and len(set(got.tolist())) == len(got)
    if nvis <= n_blocks:
        assert sorted(got.tolist()) == list(range(nvis)), f"row {t}: blocks"
    else:
        forced = {0, cur}
        assert forced <= set(got.tolist()) and len(got) == n_blocks, f"row {t}: forced blocks"
        rest = np.array([b for b in range(nvis) if b not in forced])
        chosen = np.array([b for b in got.tolist() if b not in forced])
        full = np.concatenate([chosen, -np.ones(0, np.int64)])
        check_topk(full, rest, ox.score_keys(q64[t], w64[t], kbar64[rest]),
                   score_floor(q64[t], w64[t], kbar64[rest]), n_blocks - len(forced), rtol_blk,
                   what=f"row {t} blocks")
    cand = ox.hisa_candidates(sorted(got.tolist()), p, S)
    check_topk(idx[t], cand, ox.score_keys(q64[t], w64[t], k64[cand]),
               score_floor(q64[t], w64[t], k64[cand]), K, rtol, sc[t], f"row {t} tokens")


@pytest.mark.parametrize("T,S,q_pos0,n_blocks,K,dtype", [
    (1500, 1500, 0, 5, 200, "bf16"), (700, 1900, 1200, 6, 640, "bf16"),
    (1300, 1300, 0, 64, 256, "bf16"),
    # a last group of rows shorter than the 4 that share a union, e4m3 operands, and the
    # smallest budget (the two forced blocks only)
    (1501, 1501, 0, 4, 300, "bf16"), (1203, 1203, 0, 5, 256, "e4m3"),
    (1027, 1400, 373, 2, 200, "bf16"),
    # block rows longer than the one-warp select holds (1329 blocks): forced by a kernel
    (8, 170000, 169992, 64, 2048, "bf16"),
    # the largest budget (255 blocks: the union of 4 rows sorts 1020 entries)
    (11, 40000, 39989, 255, 4096, "bf16")])
def test_hisa_prefill(T, S, q_pos0, n_blocks, K, dtype):
    """Prefill: 12 to 15 blocks with a partial last one, a chunk whose rows start at
    q_pos0 > 0, a budget that holds every block (the flat indexer then), ragged row groups,
    e4m3 operands (block keys bf16 for both formats; the block choice at the operands' own
    tolerance)."""
    p = inputs.anchor_prefill(T, H=64, d=128, K=K, seed=48, device="cuda", S=S, q_pos0=q_pos0,
                              dtype=dtype)
    kbar, _ = indexer.hisa_block_keys(p["q"], p["w"], p["k"], q_scale=p["q_scale"],
                                      k_scale=p["k_scale"], q_pos0=q_pos0)
    assert kbar.dtype == torch.bfloat16
    idx, sc, blocks = indexer.index_hisa(p["q"], p["w"], p["k"], kbar, K, n_blocks=n_blocks,
                                         q_scale=p["q_scale"], k_scale=p["k_scale"],
                                         q_pos0=q_pos0, with_scores=True, with_blocks=True)
    q64, w64 = f64(p["q"], p["q_scale"]), p["w"].double().cpu().numpy()
    k64 = f64(p["k"], p["k_scale"])
    ref_bar = ox.hisa_block_keys(k64[:q_pos0 + T])
    got_bar = f64(kbar)[:ref_bar.shape[0]]
    # bf16 rounding of an fp32 mean, whatever the key format
    assert np.all(np.abs(got_bar - ref_bar) <= 2.0 ** -8 * np.abs(ref_bar) + 1e-6)
    idx, sc, blocks = idx.cpu().numpy(), sc.cpu().numpy(), blocks.cpu().numpy()
    rows = sorted(set(range(0, T, 37)) | {0, T - 1, T - 2, T - 3, T // 2})
    rtol = RTOL[dtype]
    for t in rows:
        _check_hisa_row(t, q_pos0 + t, q64, w64, k64, got_bar, blocks, idx, sc, n_blocks, K,
                        rtol, rtol, S)


def test_hisa_decode_e4m3_and_last_block_update():
    """e4m3 caches of four lengths; the block keys (bf16 means of the decoded keys) of the next
    step, updated in place for the last block only, equal a full recomputation (bit for bit)
    and index the same way. Block choice at the e4m3 tolerance."""
    Bs, S, n_blocks, K = 4, 3100, 6, 300
    prob = inputs.decode_problem(Bs=Bs, S=S, H=64, d=128, K=K, Hg=16, steps=2, seed=49,
                                 device="cuda")
    k, ks = prob["k"], prob["k_scale"]
    S_cap = k.shape[1]
    seq_len = torch.tensor([S, 2049, 130, 1], dtype=torch.int32, device="cuda")
    q, w = prob["q_steps"][0], prob["w_steps"][0]
    kbar, _ = indexer.hisa_block_keys(q, w, k, k_scale=ks, seq_len=seq_len)
    idx, sc, blocks = indexer.index_hisa(q, w, k, kbar, K, n_blocks=n_blocks, k_scale=ks,
                                         seq_len=seq_len, with_scores=True, with_blocks=True)
    q64, w64 = f64(q), w.double().cpu().numpy()
    k64 = f64(k.reshape(-1, 128), ks.reshape(-1)).reshape(Bs, S_cap, 128)
    kb64 = f64(kbar.reshape(-1, 128)).reshape(Bs, -1, 128)
    idx_h, sc_h, blocks_h = idx.cpu().numpy(), sc.cpu().numpy(), blocks.cpu().numpy()
    for b, n in enumerate(seq_len.tolist()):
        ref = ox.hisa_block_keys(k64[b, :n])
        got = kb64[b, :ref.shape[0]]
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)
        _check_hisa_row(b, n - 1, q64, w64, k64[b], got, blocks_h, idx_h, sc_h, n_blocks, K,
                        RTOL["e4m3"], RTOL["e4m3"], S_cap)
    # next step: one more key per sequence, block keys refreshed for the last block only
    seq2 = seq_len + 1
    indexer.hisa_block_keys(q, w, k, k_scale=ks, seq_len=seq2, last_only=True, out=(kbar, None))
    full, _ = indexer.hisa_block_keys(q, w, k, k_scale=ks, seq_len=seq2)
    for b, n in enumerate(seq2.tolist()):
        nb = (n + 127) // 128
        assert torch.equal(kbar[b, :nb], full[b, :nb])
    q2, w2 = prob["q_steps"][1], prob["w_steps"][1]
    a = indexer.index_hisa(q2, w2, k, kbar, K, n_blocks=n_blocks, k_scale=ks, seq_len=seq2)[0]
    bb = indexer.index_hisa(q2, w2, k, full, K, n_blocks=n_blocks, k_scale=ks, seq_len=seq2)[0]
    assert torch.equal(a, bb)
