"""GPU union attention (qup_sparse_prefill_attn through the C ABI) vs the fp64 oracle.

Bounds (max abs, mean abs): bf16 and fp32 inputs 2e-2 / 2e-3; E4M3 KV 6e-2 / 6e-3.
Every case, the full-size workloads in the launch configuration the bench
times included, is compared on every output element.
"""
import numpy as np
import pytest

import oracle
import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

from helpers import check_close, out_to_f64, permute_queries, to_device, workload

pytestmark = pytest.mark.gpu


def _attn(w, dev, groups, want_lse=False):
    import torch
    lse = torch.full((w.Nq, w.Hq), float("nan"), device="cuda") if want_lse else None
    O = qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"], dev["page_table"], groups, dev["q_pos"],
                                w.kv_len, k_scale=dev["k_scale"], v_scale=dev["v_scale"],
                                topk=dev["topk"], lse=lse, num_logical_pages=w.num_logical_pages)
    code = qup.get_error()
    assert code == 0, f"device error {code}"
    return (O, lse) if want_lse else O


def _gpu_groups(w, dev, max_group=8, window=None):
    """Groups as the bench forms them: the workload's own window unless one is given."""
    return qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, max_group,
                            w.window if window is None else window)


def _perm_groups(w, seed, max_group=8):
    """A random partition of each KV head's queries into groups of <= max_group."""
    rng = np.random.default_rng(seed)
    part = []
    for _ in range(w.Hkv):
        perm = rng.permutation(w.Nq)
        groups = []
        i = 0
        while i < w.Nq:
            k = int(rng.integers(1, max_group + 1))
            groups.append(sorted(int(x) for x in perm[i:i + k]))
            i += k
        part.append(groups)
    return oracle.build_unions(w.topk, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, part)


SMALL = [
    dict(seed=0),
    dict(seed=1, T=32, prefix=1000),
    dict(seed=2, T=128, prefix=700, Nq=150),
    dict(seed=3, T=16, prefix=300, K=12),
    dict(seed=4, q_dtype=W.DT_F32, kv_dtype=W.DT_F32),
    dict(seed=5, q_dtype=W.DT_F32, kv_dtype=W.DT_F32, Hq=2, Hkv=2, T=32),
    dict(seed=6, kv_dtype=W.DT_E4M3, T=128, prefix=900),
    dict(seed=7, kv_dtype=W.DT_E4M3, T=64),
    dict(seed=8, Hq=8, Hkv=1, max_group=4, window=32),
    dict(seed=9, Hq=2, Hkv=1, Nq=37, prefix=0, K=3),
]


@pytest.mark.parametrize("kw", SMALL, ids=lambda k: f"s{k['seed']}")
def test_small_full_output_three_groupings(kw):
    w = W.random_small(**kw)
    ref = oracle.sparse_attn_workload(w)
    dev = to_device(w)
    mg = w.max_group
    for name, gr in (("online", _gpu_groups(w, dev, mg, w.window)),
                     ("fixed", _gpu_groups(w, dev, mg, mg)),
                     ("random", qup.groups_from_host(_perm_groups(w, kw["seed"], mg), w.Hq, w.Hkv,
                                                     w.num_logical_pages, mg))):
        got = out_to_f64(_attn(w, dev, gr))
        check_close(got, ref, w.kv_dtype, f"{w.name}/{name}")


def test_lse_matches_oracle():
    w = W.random_small(11, Hq=4, Hkv=2, Nq=90)
    ref, ref_lse = oracle.sparse_attn_workload(w, want_lse=True)
    dev = to_device(w)
    O, lse = _attn(w, dev, _gpu_groups(w, dev), want_lse=True)
    check_close(out_to_f64(O), ref, w.kv_dtype, "lse case")
    assert np.max(np.abs(lse.cpu().numpy() - ref_lse)) < 2e-3


def test_tiny_ref_fp32_full():
    w = W.tiny_ref()
    ref = oracle.sparse_attn_workload(w)
    dev = to_device(w)
    got = out_to_f64(_attn(w, dev, _gpu_groups(w, dev)))
    check_close(got, ref, w.kv_dtype, w.name)


def test_non_finite_bytes_past_kv_len_are_never_used():
    w = W.random_small(12, prefix=1000, Nq=77, T=64)  # kv_len = 1077: last page partly filled
    last_phys = w.page_table[w.num_logical_pages - 1]
    fill = w.kv_len % w.T
    assert fill != 0
    w.Kc[last_phys, :, fill:, :] = 0x7FC0  # bf16 NaN
    w.Vc[last_phys, :, fill:, :] = 0x7FC0
    ref = oracle.sparse_attn_workload(w)
    dev = to_device(w)
    got = out_to_f64(_attn(w, dev, _gpu_groups(w, dev)))
    check_close(got, ref, w.kv_dtype, "nan tail")


def test_empty_support_rows_give_zero_and_neg_inf_lse():
    w = W.random_small(13, Hq=2, Hkv=1, Nq=40)
    w.topk[:, 5, :] = -1          # no pages at all
    w.topk[:, 9, :] = -1
    w.topk[:, 9, 0] = w.num_logical_pages - 1  # only a page after the query: causally empty
    w.q_pos[9] = 3
    ref, ref_lse = oracle.sparse_attn_workload(w, want_lse=True)
    dev = to_device(w)
    O, lse = _attn(w, dev, _gpu_groups(w, dev), want_lse=True)
    got = out_to_f64(O)
    check_close(got, ref, w.kv_dtype, "empty rows")
    assert np.all(got[5] == 0) and np.all(got[9] == 0)
    assert np.all(np.isneginf(lse.cpu().numpy()[[5, 9]]))


def test_identity_page_table_and_single_member_groups():
    w = W.random_small(14, identity_pages=True, max_group=1, window=1)
    ref = oracle.sparse_attn_workload(w)
    dev = to_device(w)
    got = out_to_f64(_attn(w, dev, _gpu_groups(w, dev, 1, 1)))
    check_close(got, ref, w.kv_dtype, "groups of one")


@pytest.mark.parametrize("cfg", ["2", "3", "4a", "4b", "4c", "5"])
def test_full_size_every_element(cfg):
    """The whole output of each full-size workload, grouped as the bench groups it."""
    w = workload(cfg)
    dev = to_device(w)
    O = out_to_f64(_attn(w, dev, _gpu_groups(w, dev)))
    ref = oracle.sparse_attn_workload(w)
    check_close(O, ref, w.kv_dtype, w.name, report=True)


def test_chunk16k_rows_of_every_block():
    """The 16K-query chunk (the pages' base capture shape): one row per (Q head, 32-query block),
    so every bundle of the grouping is compared, in the launch configuration the bench times.
    (The oracle needs minutes for the whole output of this workload.)"""
    w = workload("6")
    dev = to_device(w)
    O = out_to_f64(_attn(w, dev, _gpu_groups(w, dev)))
    assert np.all(np.isfinite(O))
    rng = np.random.default_rng(66)
    blocks = np.arange(w.Hq * w.Nq // 32, dtype=np.int64)
    rows = blocks * 32 + rng.integers(0, 32, size=blocks.size)
    ref = oracle.sparse_attn_workload(w, rows=rows)
    hq, i = rows // w.Nq, rows % w.Nq
    check_close(O[i, hq], ref, w.kv_dtype, w.name + " (one row per head and 32-query block)", report=True)


def _shuffled_positions(w, seed, max_back):
    """Query IDs in random order, and each position moved back by up to max_back tokens (gaps,
    repeats, out of order): rows may then hold pages past their query, which the causal limit
    empties."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(w.Nq)
    pos = np.maximum(w.q_pos[perm] - rng.integers(0, max_back + 1, size=w.Nq), 0)
    return permute_queries(w, perm, q_pos=pos, name_suffix=f"shuffled{seed}")


SHUFFLED = [
    dict(seed=20),
    dict(seed=21, T=128, prefix=700, Nq=150, kv_dtype=W.DT_E4M3),
    dict(seed=22, T=32, prefix=1000, Hq=8, Hkv=2),
    dict(seed=23, q_dtype=W.DT_F32, kv_dtype=W.DT_F32, T=64),
]


@pytest.mark.parametrize("kw", SHUFFLED, ids=lambda k: f"s{k['seed']}")
def test_positions_out_of_id_order(kw):
    """Positions carried by the query IDs in any order (shuffled, gapped, repeated)."""
    w = _shuffled_positions(W.random_small(**kw), kw["seed"], 3 * W.random_small(**kw).T)
    ref = oracle.sparse_attn_workload(w)
    dev = to_device(w)
    for name, gr in (("online", _gpu_groups(w, dev)), ("fixed", _gpu_groups(w, dev, w.max_group, w.max_group))):
        check_close(out_to_f64(_attn(w, dev, gr)), ref, w.kv_dtype, f"{w.name}/{name}", report=True)


@pytest.mark.parametrize("cfg", ["2", "4b"])
def test_full_size_positions_out_of_id_order(cfg):
    """A full-size workload with its query IDs shuffled and positions moved back by up to a page."""
    w0 = workload(cfg)
    w = _shuffled_positions(w0, 31, w0.T)
    dev = to_device(w)
    O = out_to_f64(_attn(w, dev, _gpu_groups(w, dev)))
    ref = oracle.sparse_attn_workload(w)
    check_close(O, ref, w.kv_dtype, w.name, report=True)


@pytest.mark.parametrize("T", [64, 128])
def test_e4m3_ragged_kv_len_with_nan_bytes(T):
    """E4M3 KV with the last page partly filled and NaN bytes (0x7F) past kv_len."""
    w = W.random_small(40 + T, kv_dtype=W.DT_E4M3, T=T, prefix=1000, Nq=77, Hq=8, Hkv=2)
    fill = w.kv_len % w.T
    assert fill != 0
    last_phys = w.page_table[w.num_logical_pages - 1]
    w.Kc[last_phys, :, fill:, :] = 0x7F
    w.Vc[last_phys, :, fill:, :] = 0x7F
    ref = oracle.sparse_attn_workload(w)
    dev = to_device(w)
    got = out_to_f64(_attn(w, dev, _gpu_groups(w, dev)))
    check_close(got, ref, w.kv_dtype, f"e4m3 nan tail T={T}", report=True)


@pytest.mark.parametrize("cfg", ["2", "4b"])
def test_outputs_do_not_depend_on_grouping(cfg):
    w = workload(cfg)
    dev = to_device(w)
    a = out_to_f64(_attn(w, dev, _gpu_groups(w, dev, 8, 64)))
    b = out_to_f64(_attn(w, dev, _gpu_groups(w, dev, 8, 8)))
    tmax, tmean = (2e-2, 2e-3) if w.kv_dtype != W.DT_E4M3 else (6e-2, 6e-3)
    assert np.max(np.abs(a - b)) <= tmax and np.mean(np.abs(a - b)) <= tmean
