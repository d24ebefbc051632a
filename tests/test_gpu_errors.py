"""Error paths on the GPU: bad inputs set device error bits; a bounded pipeline wait
that runs out (host-side fault injection: one ring stage is never loaded)
returns QUP_ERR_TIMEOUT and leaves the context usable. Nothing here faults,
traps or hangs the GPU: every wait in the kernel has a time limit.
"""
import numpy as np
import pytest

import oracle
import query_union_paged_b200 as qup
from query_union_paged_b200 import workloads as W

from helpers import check_close, out_to_f64, to_device

pytestmark = pytest.mark.gpu


def _call(w, dev, gr, page_table=None):
    return qup.sparse_prefill_attn(dev["Q"], dev["K"], dev["V"],
                                   dev["page_table"] if page_table is None else page_table, gr,
                                   dev["q_pos"], w.kv_len, k_scale=dev["k_scale"],
                                   v_scale=dev["v_scale"], num_logical_pages=w.num_logical_pages)


def test_bad_physical_page_sets_error_bit():
    w = W.random_small(21)
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    bad = dev["page_table"].clone()
    bad[3] = w.P_phys + 5
    _call(w, dev, gr, bad)
    assert qup.get_error() & qup.ERR["PHYS_PAGE"]


def test_bad_group_sets_error_bit():
    w = W.random_small(22)
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    gr.bundle_qid[0, 0, 0] = w.Nq + 3
    _call(w, dev, gr)
    assert qup.get_error() & qup.ERR["GROUP"]


def test_invalid_arguments_are_rejected_synchronously():
    w = W.random_small(23)
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    import torch
    with pytest.raises(qup.QupError):
        qup.sparse_prefill_attn(dev["Q"][:, :, :64].contiguous(), dev["K"][..., :64].contiguous(),
                                dev["V"][..., :64].contiguous(), dev["page_table"], gr, dev["q_pos"],
                                w.kv_len)
    with pytest.raises(qup.QupError):
        qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 9, 64)
    with pytest.raises(qup.QupError):
        qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 60)
    assert qup.get_error() == 0


def test_timeout_is_reported_and_context_stays_usable():
    w = W.random_small(24, Nq=120)
    dev = to_device(w)
    gr = qup.sparse_group(dev["topk"], w.Hq, w.Hkv, w.num_logical_pages, 8, 64)
    try:
        qup.set_debug(wait_limit_ms=50, skip_stage=2)
        _call(w, dev, gr)
        code = qup.get_error()
    finally:
        qup.set_debug(0, -1)
    assert code & qup.ERR["TIMEOUT"]
    got = out_to_f64(_call(w, dev, gr))
    assert qup.get_error() == 0
    check_close(got, oracle.sparse_attn_workload(w), w.kv_dtype, "after timeout")
