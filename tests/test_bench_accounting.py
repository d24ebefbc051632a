"""The benchmark's work accounting on the CPU: the selected-edge count E (the metric's numerator,
512 flop per edge) and the unique-page count, checked against a brute-force count written from
the support's definition (token t of page u is in A_i iff u is in the row's TopK set, t < kv_len
and t <= q_pos[i])."""
import numpy as np
import pytest

import bench
from query_union_paged_b200 import workloads as W


def _brute_edges(w):
    E = np.zeros((w.Hq, w.Nq), np.int64)
    for hq in range(w.Hq):
        for i in range(w.Nq):
            pages = {int(u) for u in w.topk[hq, i] if u >= 0}
            n = 0
            for u in pages:
                for t in range(u * w.T, (u + 1) * w.T):
                    if t < w.kv_len and t <= w.q_pos[i]:
                        n += 1
            E[hq, i] = n
    return E


@pytest.mark.parametrize("kw", [dict(seed=40), dict(seed=41, T=16, K=12), dict(seed=42, Nq=37, prefix=0, K=3)])
def test_selected_edges_match_brute_force(kw):
    w = W.random_small(**kw)
    assert np.array_equal(bench.selected_edges_per_row(w), _brute_edges(w))


def test_unique_pages_match_brute_force():
    w = W.random_small(43, Hq=8, Hkv=2)
    g = w.Hq // w.Hkv
    want = sum(len({int(u) for hq in range(h * g, (h + 1) * g) for u in w.topk[hq].ravel() if u >= 0})
               for h in range(w.Hkv))
    assert bench.unique_kv_pages(w) == want


def test_tiny_workload_edge_count_is_exact():
    # every row: page 0, its own page (up to its position) and 6 earlier full pages
    w = W.tiny_ref()
    E = bench.selected_edges_per_row(w)
    own_part = (w.q_pos % w.T) + 1
    assert np.array_equal(E[0], 7 * w.T + own_part)


def test_grouping_reference_over_windows_matches_the_single_call():
    """The windowed timing of the CPU grouping reference runs one call per query window; groups
    never cross a window, so the summed counters equal those of the single whole-workload call."""
    w = W.tiny_ref()
    r = bench.group_reference_sample(w, w.max_group, w.window, repeats=1)
    assert r["counters_match"]
    assert r["windows"] == -(-w.Nq // w.window)
    assert r["single_thread_us"] > 0 and r["threads_over_windows_us"] > 0
