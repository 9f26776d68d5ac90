"""The parity checker the GPU tests use (`tests/parity.py`), run on the CPU against the
oracle's own results with mistakes planted in them: it must accept the oracle's Top-K and
scores (and a swap at a near-tie, which the tolerance allows), and reject every kind of wrong
answer a kernel could give - a key swapped for one well below the K-th score, a duplicate, a
key the row cannot see, too few or too many keys, padding that is not -1, and scores off by
more than the tolerance."""

import numpy as np
import pytest

from oracle import indexer as ox
from parity import RTOL, check_scores, check_topk, score_floor


def _row(seed=0, H=4, d=16, p=300, K=32):
    """One query at position p over random keys: its candidates, oracle scores and floors."""
    rng = np.random.default_rng(seed)
    q, w = rng.standard_normal((H, d)), rng.random(H)
    k = rng.standard_normal((p + 40, d))
    cand = np.arange(p + 1)
    sc = ox.score_keys(q, w, k[cand])
    fl = score_floor(q, w, k[cand])
    ref = ox.topk(sc, K, cand)
    return cand, sc, fl, ref, K


def test_accepts_the_oracle_topk_in_any_order_with_its_scores():
    cand, sc, fl, ref, K = _row()
    got = np.concatenate([ref[::-1], np.full(8, -1)])  # order carries no meaning; -1 padding
    check_topk(got, cand, sc, fl, K, RTOL["bf16"], got_scores=sc[ref[::-1]])


def test_accepts_a_swap_at_a_near_tie():
    cand, sc, fl, ref, K = _row(1)
    order = np.lexsort((cand, -sc))
    kth, nxt = order[K - 1], order[K]
    sc = sc.copy()
    sc[nxt] = sc[kth] - 1e-9 * max(1.0, abs(sc[kth]))  # the (K+1)-th a hair below the K-th
    got = ref.copy()
    got[got == cand[kth]] = cand[nxt]
    check_topk(got, cand, sc, fl, K, RTOL["bf16"])


def test_rejects_a_key_swapped_for_a_low_scoring_one():
    cand, sc, fl, ref, K = _row(2)
    low = cand[np.argmin(sc)]
    got = ref.copy()
    got[0] = low
    with pytest.raises(AssertionError, match="not within"):
        check_topk(got, cand, sc, fl, K, RTOL["bf16"])


def test_rejects_a_duplicate():
    cand, sc, fl, ref, K = _row(3)
    got = ref.copy()
    got[1] = got[0]
    with pytest.raises(AssertionError, match="duplicate"):
        check_topk(got, cand, sc, fl, K, RTOL["bf16"])


def test_rejects_a_key_the_row_cannot_see():
    cand, sc, fl, ref, K = _row(4)
    got = ref.copy()
    got[0] = cand[-1] + 5  # a future position
    with pytest.raises(AssertionError, match="outside the candidate set"):
        check_topk(got, cand, sc, fl, K, RTOL["bf16"])


def test_rejects_too_few_and_too_many_keys():
    cand, sc, fl, ref, K = _row(5)
    with pytest.raises(AssertionError, match="expected"):
        check_topk(np.concatenate([ref[:-1], [-1]]), cand, sc, fl, K, RTOL["bf16"])
    extra = next(int(c) for c in cand if c not in set(ref.tolist()))
    with pytest.raises(AssertionError, match="expected"):
        check_topk(np.concatenate([ref, [extra]]), cand, sc, fl, K, RTOL["bf16"])


def test_rejects_padding_that_is_not_minus_one_and_keys_after_padding():
    cand, sc, fl, ref, _ = _row(6, p=20, K=32)  # 21 visible keys: 11 slots of padding
    got = np.concatenate([ref, np.full(11, -1)])
    check_topk(got, cand, sc, fl, 32, RTOL["bf16"])
    bad = got.copy()
    bad[-1] = -7
    with pytest.raises(AssertionError):
        check_topk(bad, cand, sc, fl, 32, RTOL["bf16"])
    moved = np.concatenate([ref[:-1], [-1], ref[-1:], np.full(10, -1)])  # a key after a -1
    with pytest.raises(AssertionError, match="padding"):
        check_topk(moved, cand, sc, fl, 32, RTOL["bf16"])


def test_rejects_reported_scores_out_of_tolerance():
    cand, sc, fl, ref, K = _row(7)
    gs = sc[ref].copy()
    gs[3] += 3 * RTOL["bf16"] * max(abs(gs[3]), fl[ref[3]])
    with pytest.raises(AssertionError, match="out of tolerance"):
        check_topk(ref, cand, sc, fl, K, RTOL["bf16"], got_scores=gs)


def test_score_tolerance_is_relative_with_a_floor():
    ref = np.array([100.0, 1e-6, -50.0])
    floor = np.array([10.0, 10.0, 10.0])
    check_scores(ref * (1 + 0.019), ref, floor, 2e-2)            # within 2 %
    check_scores(ref + 0.19, ref, floor, 2e-2)                   # the floor admits 0.2 absolute
    with pytest.raises(AssertionError):
        check_scores(ref * (1 + 0.03), ref, floor, 2e-2)         # 3 % of 100 is out
    with pytest.raises(AssertionError):
        check_scores(ref + np.array([0.0, 0.25, 0.0]), ref, floor, 2e-2)  # past the floor
