"""Pins for the CPU grouping reference.

- the worked example of the PageWeaver page's Figure 2 (stored fixture);
- a pure-Python brute-force statement of the grouping rule (Python sets) on
  tiny inputs, which must agree group by group, page by page and bit by bit;
- partition invariants (every query once, at most max_group, union = member
  supports, masks = each row's own pages, counter identities);
- special cases: window = max_group gives fixed consecutive groups; identical
  supports give consecutive groups and no masked slots; the 128K block-union
  workload regroups into 64-query-block-aligned groups whose union is the
  block's union over the 4 heads of the KV group.
"""
import os

import numpy as np
import pytest

import oracle
from query_union_paged_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fig2_worked_example.txt")


def _read_fig2():
    topk, expect, meta = [], [], {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "topk":
                topk.append([int(v) for v in vals])
            elif key == "expect":
                expect.append(tuple(int(v) for v in vals))
            else:
                meta[key] = int(vals[0])
    return np.array(topk, np.int32)[None], expect, meta


def test_figure2_worked_example():
    topk, expect, meta = _read_fig2()
    assert len(expect) == 2
    for window, visits, masked_q, edges in expect:
        out = oracle.group(topk, 1, 1, meta["num_queries"], meta["num_pages"],
                           meta["max_group"], window)
        c = out["counters"][0]
        assert (c[0], c[2], c[3]) == (visits, masked_q, edges)
        assert c[1] == masked_q  # g = 1: rows are queries
    regroup = oracle.group(topk, 1, 1, 8, 4, 2, 8)
    groups = [list(regroup["members"][0, regroup["group_ptr"][0, k]:regroup["group_ptr"][0, k + 1]])
              for k in range(regroup["n_groups"][0])]
    assert groups == [[0, 2], [1, 3], [4, 6], [5, 7]]


# ----------------------------------------------------------- brute force

def py_group(topk, Hq, Hkv, Nq, max_group, window):
    """The grouping rule written with Python sets (no shared code with oracle.c)."""
    g = Hq // Hkv
    res = []
    for h in range(Hkv):
        rows = [[set(int(p) for p in topk[h * g + j, i] if p != -1) for j in range(g)]
                for i in range(Nq)]
        S = [set().union(*r) for r in rows]
        groups = []
        for w0 in range(0, Nq, window):
            left = list(range(w0, min(Nq, w0 + window)))
            while left:
                seed = min(left)
                left.remove(seed)
                mem, U = [seed], set(S[seed])
                while len(mem) < max_group and left:
                    c = min(left, key=lambda q: (len(S[q] - U), q))
                    left.remove(c)
                    mem.append(c)
                    U |= S[c]
                mem.sort()
                upages = sorted(U)
                masks = []
                for p in upages:
                    m = 0
                    for rank, q in enumerate(mem):
                        for j in range(g):
                            if p in rows[q][j]:
                                m |= 1 << (rank * g + j)
                    masks.append(m)
                groups.append((mem, upages, masks,
                               sum(len(U) - len(rows[q][j]) for q in mem for j in range(g)),
                               sum(len(U) - len(S[q]) for q in mem)))
        res.append((groups, sum(len(s) for s in S)))
    return res


def _groups_of(out, h):
    gp = out["group_ptr"][h]
    up = out["union_ptr"][h]
    res = []
    for k in range(out["n_groups"][h]):
        mem = [int(x) for x in out["members"][h, gp[k]:gp[k + 1]]]
        pages = [int(x) for x in out["union_pages"][up[k]:up[k + 1]]]
        masks = [int(x) for x in out["row_mask"][up[k]:up[k + 1]]]
        res.append((mem, pages, masks))
    return res


@pytest.mark.parametrize("seed", range(10))
def test_matches_python_brute_force(seed):
    rng = np.random.default_rng(seed)
    Hkv = int(rng.integers(1, 3))
    g = int(rng.choice([1, 2, 4]))
    Hq = Hkv * g
    Nq = int(rng.integers(1, 40))
    K = int(rng.integers(1, 6))
    P = int(rng.integers(2, 20))
    max_group = int(rng.choice([1, 2, 3, 4, 8]))
    window = max_group * int(rng.integers(1, 5))
    topk = rng.integers(-1, P, size=(Hq, Nq, K)).astype(np.int32)
    out = oracle.group(topk, Hq, Hkv, Nq, P, max_group, window)
    ref = py_group(topk, Hq, Hkv, Nq, max_group, window)
    for h in range(Hkv):
        groups, edges = ref[h]
        got = _groups_of(out, h)
        assert [x[:3] for x in groups] == [tuple(x) for x in got] or \
            [list(x[:3]) for x in groups] == [list(x) for x in got]
        c = out["counters"][h]
        assert c[0] == sum(len(x[1]) for x in groups)
        assert c[1] == sum(x[3] for x in groups)
        assert c[2] == sum(x[4] for x in groups)
        assert c[3] == edges


def check_partition_invariants(out, topk, Hq, Hkv, Nq, max_group):
    g = Hq // Hkv
    for h in range(Hkv):
        seen = np.zeros(Nq, int)
        for mem, pages, masks in _groups_of(out, h):
            assert 1 <= len(mem) <= max_group and mem == sorted(mem)
            seen[mem] += 1
            assert pages == sorted(set(pages))
            rowsets = [[set(int(p) for p in topk[h * g + j, q] if p != -1) for j in range(g)]
                       for q in mem]
            assert set(pages) == set().union(*[s for r in rowsets for s in r])
            for p, m in zip(pages, masks):
                for rank in range(len(mem)):
                    for j in range(g):
                        assert bool((m >> (rank * g + j)) & 1) == (p in rowsets[rank][j])
                assert m >> (len(mem) * g) == 0
        assert np.all(seen == 1)


def test_partition_invariants_random_workload():
    w = W.random_small(3, Hq=8, Hkv=2, Nq=150, K=8, max_group=8, window=64)
    out = oracle.group(w.topk, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, 8, 64)
    check_partition_invariants(out, w.topk, w.Hq, w.Hkv, w.Nq, 8)


def test_window_equal_to_max_group_gives_fixed_consecutive_groups():
    w = W.random_small(4, Hq=4, Hkv=1, Nq=37, K=5)
    out = oracle.group(w.topk, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, 8, 8)
    got = [x[0] for x in _groups_of(out, 0)]
    assert got == [list(range(s, min(37, s + 8))) for s in range(0, 37, 8)]


def test_identical_supports_have_no_masked_query_slots():
    topk = np.tile(np.array([3, 1, 4, 1, 5], np.int32), (2, 20, 1))
    out = oracle.group(topk, 2, 1, 20, 8, 8, 64)
    assert [x[0] for x in _groups_of(out, 0)] == [list(range(0, 8)), list(range(8, 16)),
                                                    list(range(16, 20))]
    assert out["counters"][0, 2] == 0 and out["counters"][0, 1] == 0
    assert out["counters"][0, 0] == 3 * 4 and out["counters"][0, 3] == 20 * 4


def test_block_union_workload_groups_align_with_query_blocks():
    w = W.block_union_128k()
    out = oracle.group(w.topk, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, 8, 64)
    g = w.g
    for h in range(w.Hkv):
        for mem, pages, masks in _groups_of(out, h):
            blocks = {q // 64 for q in mem}
            assert len(blocks) == 1
            b = blocks.pop()
            union = set()
            for j in range(g):
                union |= set(int(p) for p in w.topk[h * g + j, b * 64] if p != -1)
            assert set(pages) == union
    # every row keeps exactly its own block row, so masked row slots are the
    # union minus each head's row, and members of one block share their support
    assert np.all(out["counters"][:, 2] == 0)


# ----------------------------------------------------------- bundles

def py_bundle(out, Hq, Hkv, Nq, max_group, wb=64):
    """The bundling rule written with Python sets: greedy over group unions (pick key: new pages
    minus twice the shared pages, ties to the smallest index)."""
    g = Hq // Hkv
    rs = 1
    while rs < max_group * g:
        rs *= 2
    slots = 128 // rs
    wb = max(slots, (wb // slots) * slots)
    res = []
    for h in range(Hkv):
        groups = _groups_of(out, h)
        bundles = []
        for w0 in range(0, len(groups), wb):
            left = list(range(w0, min(len(groups), w0 + wb)))
            while left:
                seed = left.pop(0)
                U, b = set(groups[seed][1]), [seed]
                while len(b) < slots and left:
                    # fewest new pages, counted against the pages already shared with the bundle
                    c = min(left, key=lambda q: (len(set(groups[q][1]) - U) - 2 * len(set(groups[q][1]) & U), q))
                    left.remove(c)
                    b.append(c)
                    U |= set(groups[c][1])
                b.sort()
                pages = sorted(U)
                masks = []
                for p in pages:
                    m = 0
                    for j, gi in enumerate(b):
                        mem, gp, gm = groups[gi]
                        if p in gp:
                            m |= gm[gp.index(p)] << (j * rs)
                    masks.append(m)
                qids = [-1] * (128 // g)
                for j, gi in enumerate(b):
                    for k, q in enumerate(groups[gi][0]):
                        qids[j * (rs // g) + k] = q
                bundles.append((b, pages, masks, qids))
        res.append(bundles)
    return res


@pytest.mark.parametrize("seed", range(6))
def test_bundles_match_python_brute_force(seed):
    rng = np.random.default_rng(50 + seed)
    Hkv = int(rng.integers(1, 3))
    g = int(rng.choice([1, 2, 4]))
    max_group = int(rng.choice([1, 2, 4, 8]))
    Hq, Nq, K, P = Hkv * g, int(rng.integers(1, 200)), int(rng.integers(1, 6)), int(rng.integers(2, 60))
    topk = rng.integers(-1, P, size=(Hq, Nq, K)).astype(np.int32)
    out = oracle.group(topk, Hq, Hkv, Nq, P, max_group, max_group * 4)
    b = oracle.bundle(out, Hq, Hkv, Nq, max_group)
    ref = py_bundle(out, Hq, Hkv, Nq, max_group)
    for h in range(Hkv):
        assert b["n_bundles"][h] == len(ref[h])
        for k, (grp, pages, masks, qids) in enumerate(ref[h]):
            bp = b["bundle_ptr"][h]
            assert list(b["bundle_groups"][h, bp[k]:bp[k + 1]]) == grp
            up = b["bunion_ptr"][h]
            assert list(b["bunion_pages"][up[k]:up[k + 1]]) == pages
            words = b["bunion_mask"][up[k]:up[k + 1]].astype(np.uint64)
            got = [int(w[0]) | int(w[1]) << 32 | int(w[2]) << 64 | int(w[3]) << 96 for w in words]
            assert got == masks
            assert list(b["bundle_qid"][h, k]) == qids
        assert b["bcounters"][h, 0] == sum(len(x[1]) for x in ref[h])


def test_bundles_partition_groups_and_keep_row_supports():
    w = W.random_small(8, Hq=8, Hkv=2, Nq=200, K=6)
    out = oracle.group(w.topk, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, 8, 64)
    b = oracle.bundle(out, w.Hq, w.Hkv, w.Nq, 8)
    g = w.g
    for h in range(w.Hkv):
        seen = np.zeros(out["n_groups"][h], int)
        for k in range(b["n_bundles"][h]):
            bp, up = b["bundle_ptr"][h], b["bunion_ptr"][h]
            seen[b["bundle_groups"][h, bp[k]:bp[k + 1]]] += 1
            assert bp[k + 1] - bp[k] <= 128 // 32
            for e in range(up[k], up[k + 1]):
                p = b["bunion_pages"][e]
                m = int(b["bunion_mask"][e][0]) | int(b["bunion_mask"][e][1]) << 32 | \
                    int(b["bunion_mask"][e][2]) << 64 | int(b["bunion_mask"][e][3]) << 96
                for row in range(128):
                    q = b["bundle_qid"][h, k, row // g]
                    want = q >= 0 and p in set(w.topk[h * g + row % g, q].tolist())
                    assert bool((m >> row) & 1) == want
        assert np.all(seen == 1)
