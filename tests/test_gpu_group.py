"""GPU grouping (qup_sparse_group through the C ABI) vs the CPU reference: bit-exact."""
import numpy as np
import pytest

import oracle
import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

from helpers import assert_bundles_equal, assert_groups_equal, groups_to_host, workload

pytestmark = pytest.mark.gpu


def _run(topk_np, Hq, Hkv, P, max_group, window):
    import torch
    topk = torch.from_numpy(np.ascontiguousarray(topk_np, dtype=np.int32)).cuda()
    gr = qup.sparse_group(topk, Hq, Hkv, P, max_group, window)
    assert qup.get_error() == 0
    return groups_to_host(gr)


@pytest.mark.parametrize("seed", range(8))
def test_random_small_bitexact(seed):
    rng = np.random.default_rng(100 + seed)
    Hkv = int(rng.integers(1, 4))
    g = int(rng.choice([1, 2, 4]))
    max_group = int(rng.choice([1, 2, 4, 8])) if g < 8 else 4
    max_group = min(max_group, 32 // g)
    window = max_group * int(rng.integers(1, 9))
    window = min(window, 256 // max_group * max_group)
    Nq = int(rng.integers(1, 300))
    K = int(rng.integers(1, 20))
    P = int(rng.integers(1, 700))
    topk = rng.integers(-1, P, size=(Hkv * g, Nq, K)).astype(np.int32)
    got = _run(topk, Hkv * g, Hkv, P, max_group, window)
    ref = oracle.group(topk, Hkv * g, Hkv, Nq, P, max_group, window)
    assert_groups_equal(got, ref)
    assert_bundles_equal(got, oracle.bundle(ref, Hkv * g, Hkv, Nq, max_group))


@pytest.mark.parametrize("cfg", ["1", "2", "3", "4a", "4b", "4c", "5"])
@pytest.mark.parametrize("window", [64, 8, 128, 256])
def test_workload_bitexact(cfg, window):
    w = workload(cfg)
    got = _run(w.topk, w.Hq, w.Hkv, w.num_logical_pages, 8, window)
    ref = oracle.group(w.topk, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, 8, window)
    assert_groups_equal(got, ref)
    assert_bundles_equal(got, oracle.bundle(ref, w.Hq, w.Hkv, w.Nq, 8))


def test_chunk16k_bitexact():
    """The 16K-query chunk: grouping workspace, groups and the 16,384-query bundle walk bit-exact."""
    w = workload("6")
    got = _run(w.topk, w.Hq, w.Hkv, w.num_logical_pages, 8, w.window)
    ref = oracle.group(w.topk, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, 8, w.window)
    assert_groups_equal(got, ref)
    assert_bundles_equal(got, oracle.bundle(ref, w.Hq, w.Hkv, w.Nq, 8))


@pytest.mark.parametrize("seed", range(6))
def test_large_windows_small_universe_bitexact(seed):
    """Windows of 65..256 queries whose pages fit 8 words: the whole-CTA greedy."""
    rng = np.random.default_rng(300 + seed)
    Hkv, g = int(rng.integers(1, 3)), int(rng.choice([1, 2, 4]))
    max_group = min(int(rng.choice([1, 2, 4, 8])), 32 // g)
    window = max_group * int(rng.integers(65 // max_group + 1, 256 // max_group + 1))
    Nq = int(rng.integers(window // 2, 700))
    K = int(rng.integers(1, 12))
    P = int(rng.integers(8, 250))
    topk = rng.integers(-1, P, size=(Hkv * g, Nq, K)).astype(np.int32)
    got = _run(topk, Hkv * g, Hkv, P, max_group, window)
    ref = oracle.group(topk, Hkv * g, Hkv, Nq, P, max_group, window)
    assert_groups_equal(got, ref)
    assert_bundles_equal(got, oracle.bundle(ref, Hkv * g, Hkv, Nq, max_group))


def test_figure2_example_on_gpu():
    topk = np.array([[0, 1], [2, 3]] * 4, np.int32)[None]
    adj = _run(topk, 1, 1, 4, 2, 2)
    reg = _run(topk, 1, 1, 4, 2, 8)
    assert tuple(adj["counters"][0][[0, 2, 3]]) == (16, 16, 16)
    assert tuple(reg["counters"][0][[0, 2, 3]]) == (8, 0, 16)


def test_max_window_and_large_page_range():
    rng = np.random.default_rng(5)
    P = 5000
    topk = rng.integers(-1, P, size=(8, 600, 24)).astype(np.int32)
    got = _run(topk, 8, 2, P, 8, 256)
    ref = oracle.group(topk, 8, 2, 600, P, 8, 256)
    assert_groups_equal(got, ref)
    assert_bundles_equal(got, oracle.bundle(ref, 8, 2, 600, 8))


def test_bundles_of_a_given_partition_match_reference():
    import query_union_paged_b200 as qup
    rng = np.random.default_rng(9)
    Hq, Hkv, Nq, P = 8, 2, 150, 90
    topk = rng.integers(-1, P, size=(Hq, Nq, 7)).astype(np.int32)
    part = []
    for _ in range(Hkv):
        perm = rng.permutation(Nq)
        groups, i = [], 0
        while i < Nq:
            k = int(rng.integers(1, 9))
            groups.append(sorted(int(x) for x in perm[i:i + k]))
            i += k
        part.append(groups)
    ref = oracle.build_unions(topk, Hq, Hkv, Nq, P, part)
    gr = qup.groups_from_host(ref, Hq, Hkv, P, 8)
    assert qup.get_error() == 0
    assert_bundles_equal(groups_to_host(gr), oracle.bundle(ref, Hq, Hkv, Nq, 8))


def test_out_of_range_page_id_sets_error_bit():
    import torch
    topk = torch.tensor([[[0, 1, 9]]], dtype=torch.int32, device="cuda")
    qup.sparse_group(topk, 1, 1, 4, 8, 8)
    assert qup.get_error() & qup.ERR["PAGE_ID"]
    assert qup.get_error() == 0  # cleared by the read
