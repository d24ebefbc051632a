"""Proxy-query page selection on the device (qup_pivot_select) against the oracle
(oracle/pivot.py): the selected page IDs are integers decided by float32 scores that both sides
compute with the same rounded operations in the same order, so they must agree exactly, including
the order of ties (integer-valued inputs make many)."""
import numpy as np
import pytest

import oracle.pivot as opivot
import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _device(x, bf16):
    import torch
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(x)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _run(inp, g, group_size, n_cand, K, refine, bf16=True):
    import torch
    q = _device(inp.q_bits if bf16 else inp.q, bf16)
    k = _device(inp.k_bits if bf16 else inp.k, bf16)
    pos = torch.from_numpy(inp.q_pos).cuda()
    got = qup.pivot_select(q, k, pos, g, inp.T, group_size, n_cand, K, refine=refine)
    torch.cuda.synchronize()
    assert qup.get_error() == 0
    return got.cpu().numpy()


CASES = [
    # seed, Nq, Hkv, d, prefix, T, g, G, C, K, refine, bf16, integer, shuffled
    (1, 100, 2, 128, 960, 64, 4, 16, 32, 8, True, True, False, False),
    (2, 100, 2, 128, 960, 64, 4, 16, 32, 8, False, True, False, False),
    (3, 77, 3, 64, 500, 16, 2, 8, 64, 16, True, True, True, False),      # ties, ragged last group
    (4, 77, 3, 64, 500, 16, 2, 8, 64, 16, False, True, True, True),      # ties, shuffled positions
    (5, 130, 1, 32, 0, 32, 1, 32, 20, 20, True, False, False, True),     # fp32, from position 0
    (6, 64, 2, 128, 4096, 128, 8, 64, 256, 32, True, True, False, False),  # candidates = every page
    (7, 50, 2, 16, 300, 64, 4, 1, 4, 4, True, True, True, False),        # groups of one
]


@pytest.mark.parametrize("case", CASES, ids=[f"s{c[0]}" for c in CASES])
def test_selection_matches_the_oracle_exactly(case):
    seed, Nq, Hkv, d, prefix, T, g, G, C, K, refine, bf16, integer, shuffled = case
    inp = W.indexer_inputs(seed, Nq, Hkv, d, prefix, T, bf16=bf16, integer=integer, shuffle_positions=shuffled,
                           extra_pages=3)
    want = opivot.pivot_select(inp.q, inp.k, inp.q_pos, T, inp.num_logical_pages, G, C, K, refine, g)
    got = _run(inp, g, G, C, K, refine, bf16)
    assert got.shape == want.shape
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} entries differ, first {bad[:3].tolist()}"


def test_selection_at_the_64k_workload_shape():
    """4096 queries after a 64K prefix, 8 KV heads of 4 query heads, 128-token pages, 128-wide index
    vectors, groups of 16, 64 candidates, Top16 (the shape of the 64K workloads' TopK rows)."""
    inp = W.indexer_inputs(11, 4096, 8, 128, 65536, 128)
    got = _run(inp, 4, 16, 64, 16, True)
    want = opivot.pivot_select(inp.q, inp.k, inp.q_pos, 128, inp.num_logical_pages, 16, 64, 16, True, 4)
    assert np.array_equal(got, want)


def test_selected_pages_feed_grouping_and_attention():
    """The device selection drives the grouping call and union attention; the result matches the fp64
    attention oracle on the same (oracle-selected, identical) TopK rows."""
    import torch
    import oracle
    from helpers import check_close, out_to_f64, to_device
    w = W.random_small(31, Hq=8, Hkv=2, Nq=96, T=64, prefix=960, K=8)
    inp = W.indexer_inputs(31, w.Nq, w.Hkv, 64, 960, w.T, extra_pages=w.num_logical_pages - (960 + w.Nq + 63) // 64)
    assert inp.num_logical_pages == w.num_logical_pages and np.array_equal(inp.q_pos, w.q_pos)
    g = w.Hq // w.Hkv
    topk = opivot.pivot_select(inp.q, inp.k, inp.q_pos, w.T, w.num_logical_pages, 16, 24, 8, True, g)
    w.topk = topk
    got_sel = _run(inp, g, 16, 24, 8, True)
    assert np.array_equal(got_sel, topk)
    dev = to_device(w)
    sel = torch.from_numpy(got_sel).cuda()
    gr = qup.sparse_group(sel, w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    out = qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"], dev["page_table"], gr, dev["q_pos"], w.kv_len,
                                  num_logical_pages=w.num_logical_pages)
    torch.cuda.synchronize()
    assert qup.get_error() == 0
    check_close(out_to_f64(out), oracle.sparse_attn_workload(w), w.kv_dtype, "selector -> group -> attention")
