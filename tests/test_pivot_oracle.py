"""Pins of the proxy-query page selection oracle (oracle/pivot.py) against things other than itself:
a hand-worked example, an exact brute force in Python integers (the dense indexer that PIVOT-Refine
matches when the candidate set holds every visible page: PIVOT, Abstract), and special cases that
reduce one variant to another."""
import numpy as np
import pytest

from oracle.pivot import pivot_select


def _dense_topk(q, keys, pos, T, P, K):
    """Exact dense per-query top-K in Python integers: every visible page scored by its own query."""
    Nq, Hkv, d = q.shape
    out = np.full((Hkv, Nq, K), -1, np.int32)
    for h in range(Hkv):
        for i in range(Nq):
            vis = min(P - 1, int(pos[i]) // T)
            sc = {p: sum(int(q[i, h, t]) * int(keys[p, h, t]) for t in range(d)) for p in range(vis + 1)}
            sel = sorted(sc, key=lambda p: (-sc[p], p))[:K]
            out[h, i, :len(sel)] = sel
    return out


def _int_case(seed, Nq=23, Hkv=2, d=8, P=13, T=16, lo=-3, hi=4, pos0=40):
    rng = np.random.default_rng(seed)
    q = rng.integers(lo, hi, size=(Nq, Hkv, d)).astype(np.float32)
    keys = rng.integers(lo, hi, size=(P, Hkv, d)).astype(np.float32)
    pos = pos0 + np.sort(rng.choice(P * T - pos0, size=Nq, replace=False)).astype(np.int64)
    return q, keys, pos, T, P


def test_hand_worked_example():
    # one KV head, d = 2, pages of 4 tokens; queries at positions 5 and 9 (own pages 1 and 2)
    keys = np.array([[[1, 0]], [[0, 1]], [[1, 1]], [[5, 5]]], np.float32)  # page 3 is in the future
    q = np.array([[[2, 1]], [[1, 3]]], np.float32)
    pos = np.array([5, 9])
    # Refine, groups of one: query 0 sees pages 0, 1 with scores 2, 1 -> [0, 1];
    # query 1 sees pages 0, 1, 2 with scores 1, 3, 4 -> [2, 1]
    got = pivot_select(q, keys, pos, 4, 4, group_size=1, n_cand=4, K=2, refine=True, g=1)
    assert got[0].tolist() == [[0, 1], [2, 1]]
    # one group of two: proxy = (1.5, 2), sees pages 0..2 with scores 1.5, 2, 3.5 -> candidates
    # [2, 1, 0]; Reuse gives each query the visible candidates in proxy order
    got = pivot_select(q, keys, pos, 4, 4, group_size=2, n_cand=4, K=2, refine=False, g=1)
    assert got[0].tolist() == [[1, 0], [2, 1]]
    # n_cand = 1 keeps only page 2: query 0 cannot see it and gets nothing
    got = pivot_select(q, keys, pos, 4, 4, group_size=2, n_cand=1, K=2, refine=True, g=1)
    assert got[0].tolist() == [[-1, -1], [2, -1]]


@pytest.mark.parametrize("seed,G", [(1, 1), (2, 4), (3, 7), (4, 32)])
def test_refine_with_every_page_as_candidate_is_the_dense_indexer(seed, G):
    q, keys, pos, T, P = _int_case(seed)
    K = 5
    got = pivot_select(q, keys, pos, T, P, group_size=G, n_cand=P, K=K, refine=True, g=3)
    want = _dense_topk(q, keys, pos, T, P, K)
    assert got.shape == (q.shape[1] * 3, q.shape[0], K)
    assert np.array_equal(got, np.repeat(want, 3, axis=0))


def test_reuse_with_groups_of_one_equals_refine():
    q, keys, pos, T, P = _int_case(5)
    a = pivot_select(q, keys, pos, T, P, group_size=1, n_cand=6, K=4, refine=False, g=1)
    b = pivot_select(q, keys, pos, T, P, group_size=1, n_cand=6, K=4, refine=True, g=1)
    assert np.array_equal(a, b)


def test_reuse_of_identical_queries_is_the_dense_top_k_of_that_query():
    # every member of a group has the same indexer query: the proxy is that query (mean of equal
    # vectors, exact), so Reuse with every page as candidate is the dense top-K
    q, keys, pos, T, P = _int_case(6, Nq=24)
    G = 8
    for g0 in range(0, q.shape[0], G):
        q[g0:g0 + G] = q[g0]
    got = pivot_select(q, keys, pos, T, P, group_size=G, n_cand=P, K=4, refine=False, g=1)
    assert np.array_equal(got, _dense_topk(q, keys, pos, T, P, 4))


def test_small_candidate_sets_stay_causal_distinct_and_inside_the_candidates():
    q, keys, pos, T, P = _int_case(7, Nq=40, P=29, T=8, pos0=10)
    G, C, K = 8, 6, 4
    got = pivot_select(q, keys, pos, T, P, group_size=G, n_cand=C, K=K, refine=True, g=1)
    for h in range(q.shape[1]):
        for i in range(q.shape[0]):
            row = [p for p in got[h, i] if p >= 0]
            assert len(set(row)) == len(row)
            assert all(p * T <= pos[i] for p in row)
            assert all(p == -1 for p in got[h, i][len(row):])
            # every selected page is among the group's C best proxy pages
            g0 = (i // G) * G
            members = range(g0, min(q.shape[0], g0 + G))
            proxy = sum(q[m, h].astype(np.float64) for m in members) / len(members)
            lim = min(P, max(int(pos[m]) for m in members) // T + 1)
            sc = {p: float(np.dot(proxy, keys[p, h].astype(np.float64))) for p in range(lim)}
            best = sorted(sc, key=lambda p: (-sc[p], p))[:C]
            assert set(row) <= set(best)


def test_float_scores_round_in_float32_sequentially():
    # values whose sum depends on the order: the oracle must add in t order, in float32
    keys = np.array([[[1e8, 1.0, -1e8]]], np.float32)
    q = np.array([[[1.0, 1.0, 1.0]]], np.float32)
    got = pivot_select(q, keys, np.array([0]), 4, 1, 1, 1, 1, True, 1)
    assert got[0, 0, 0] == 0
    from oracle.pivot import _score
    s = _score(q[0, 0], keys[:, 0, :])
    # ((1e8 + 1) rounded to 1e8) - 1e8 = 0 in float32 accumulation
    assert s[0] == np.float32(0.0)
