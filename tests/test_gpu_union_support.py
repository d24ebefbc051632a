"""Union as support (qup_union_support; CompactAttention: Accelerating Chunked Prefill with
Block-Union KV Selection): after the call every row of a group attends to the whole union of its
group.  The expected result is the oracle's definition with each query's TopK row replaced by its
group's union pages (built here from the groups), so the oracle itself is unchanged."""
import dataclasses

import numpy as np
import pytest

import oracle
import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

from helpers import check_close, groups_to_host, out_to_f64, to_device, workload

pytestmark = pytest.mark.gpu


def _union_topk(w, gh):
    """[Hq][Nq][Kmax]: for every query, the union pages of its group (its KV head's), -1 padded."""
    g = w.Hq // w.Hkv
    rows = {}
    kmax = 1
    for h in range(w.Hkv):
        gp, up = gh["group_ptr"][h], gh["union_ptr"][h]
        for k in range(int(gh["n_groups"][h])):
            pages = gh["union_pages"][up[k]:up[k + 1]]
            kmax = max(kmax, pages.size)
            for m in gh["members"][h, gp[k]:gp[k + 1]]:
                rows[(h, int(m))] = pages
    topk = np.full((w.Hq, w.Nq, kmax), -1, np.int32)
    for (h, m), pages in rows.items():
        topk[h * g:(h + 1) * g, m, :pages.size] = pages
    return topk


def _run(w, window):
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, w.max_group, window)
    gh = groups_to_host(gr)
    qup.union_support(gr, w.Hq, w.Hkv, w.Nq, w.num_logical_pages, w.max_group)
    O = qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"], dev["page_table"], gr, dev["q_pos"], w.kv_len,
                                k_scale=dev["k_scale"], v_scale=dev["v_scale"],
                                num_logical_pages=w.num_logical_pages)
    assert qup.get_error() == 0
    tu = _union_topk(w, gh)
    return out_to_f64(O), dataclasses.replace(w, topk=tu, K=tu.shape[-1])


def test_union_support_small_full_output():
    w = W.random_small(31, Hq=8, Hkv=2, Nq=100)
    got, wu = _run(w, 64)
    check_close(got, oracle.sparse_attn_workload(wu), w.kv_dtype, "union support, small")
    # the supports grew, so the outputs moved away from the per-row result
    own = oracle.sparse_attn_workload(w)
    assert np.max(np.abs(got - own)) > 1e-2


def test_union_support_block_union_workload_sampled_rows():
    w = workload("5")
    got, wu = _run(w, w.window)
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(w.Hq * w.Nq, size=2048, replace=False)).astype(np.int64)
    ref = oracle.sparse_attn_workload(wu, rows=rows)
    hq, i = rows // w.Nq, rows % w.Nq
    check_close(got[i, hq], ref, w.kv_dtype, "union support, block-union workload")
